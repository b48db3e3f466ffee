// indexer_tc.cu -- lightning-indexer scores on tcgen05 tensor cores (bf16 in, fp32 out).
//
//   I(t,s) = sum_{j<16} w[t,j] * max(0, sum_{d<64} q_idx[t,j,d] * k_idx[s,d])
//
// (DSA ablation card, "Attention" bullet: a ReLU lightning indexer scores every key per
// query; one indexer key per token is shared by the heads.)
//
// Tiling.  Keys go on the UMMA M side (128 keys = the 128 TMEM lanes) and (query, head)
// pairs on the N side: N = QB * 16 with QB = 16 queries per block in prefill and QB = 1 in
// decode.  K = 64 is a single 128-byte swizzle atom, so one tile is 4 UMMAs of K = 16.
// With keys on lanes, the ReLU + head-weight reduction of a score is a sum over 16
// consecutive TMEM columns that stay inside one thread -- no shuffles.
//
// Warp roles (640 threads): warp 0 issues TMA loads (query block once per unit, key tiles
// through a ring of smem stages; for paged keys warps 2 and 3 issue the copies of two of
// every three stages), warp 1 issues UMMAs into a ring of TMEM accumulators (two of 256
// columns in prefill), warp 2 owns the TMEM allocation, warps 4..19 drain the
// accumulators: tcgen05.ld, ReLU, weight, reduce, causal mask, coalesced fp32 stores.  The
// drain is the longest stage per tile (16 max + 16 multiply-adds per score), so it gets
// four warps per TMEM lane quadrant, each on a quarter of the block's queries, and the
// weights are applied with packed fp32x2 FMAs (with at most two queries per warp their
// head weights stay in registers for the whole unit; eight-query blocks, which allow
// that, measured slower: less independent work per warp between the pipeline waits).  Tiles that lie wholly below the causal
// diagonal of a full block store without a per-score test.
//
// Work units are (query block, chunk of at most 32 key tiles): prefill blocks hold 16
// queries and their causal key range grows with the query position, so the range is cut
// into chunks to give every SM work even for a narrow window of query rows.  Decode units
// are (sequence, 2048-key chunk); key tiles are assembled from pages with one TMA load per
// page.  The query block and its head weights are double-buffered across units.
#include "dsa_common.cuh"
#include "launch.h"

namespace dsa {

namespace {

constexpr int kHI = 16;
constexpr int kDI = 64;
constexpr int kBM = 128;           // keys per tile (UMMA M)
// Key-tile ring: 6 stages of 16 KB (a 12-stage ring for the one-query decode blocks
// measured no faster).
template <int QB>
constexpr int stages_for() { return 6; }
constexpr int kThreads = 640;
constexpr int kEpiWarp0 = 4;       // first epilogue warp
constexpr int kEpiWarps = 16;      // four per TMEM lane quadrant
constexpr uint32_t kTileBytes = kBM * 128;  // 128 keys x 64 bf16
constexpr int kDecodeChunkTiles = 16;       // decode unit = 2048 keys
constexpr int kPrefillChunkTiles = 32;      // prefill unit: at most 4096 keys
constexpr int kPrefillQB = 16;              // prefill queries per block (UMMA N = 256)
// Paged (decode) key tiles are copied by three producer warps (0, 2 and 3), each issuing
// the copies of every third ring stage: one thread issuing TMA copies of 8 KB pages
// reaches ~4.7 TB/s, whatever the number of copies in flight.
constexpr int kDecodeProducers = 3;
static_assert(kPrefillChunkTiles * 128 == 4096, "filtered candidate lists are per 4096-key chunk");

template <int QB>
struct IdxSmem {
    static constexpr int kStages = stages_for<QB>();
    alignas(1024) uint8_t k[kStages][kTileBytes];
    alignas(1024) uint8_t q[2][QB * kHI * 128 < 1024 ? 1024 : QB * kHI * 128];
    alignas(16) float w[2][QB * kHI];  // head weights of the unit's queries
    uint64_t k_full[kStages];
    uint64_t k_empty[kStages];
    uint64_t q_full[2], q_empty[2];
    uint64_t acc_full[4], acc_empty[4];
    uint32_t tmem_base;
    int abort;
    int pages[kDecodeProducers][kDecodeChunkTiles * kBM / 16];  // decode: each producer's
                                                                // copy of the unit's pages
};

// What the prefill epilogue does with each score.
enum IdxMode : int {
    kDense = 0,    // store every causal score in a dense row
    kSample = 1,   // scores of every tile_stride-th key tile only, stored compactly
    kFilter = 2,   // append the keys at or above the row's threshold to candidate lists
                   // (no dense row)
};

struct IdxParams {
    const float* w;
    float* scores;
    long long ld;
    int tile_stride;          // physical key tile of logical tile j = j * tile_stride
    const int* guard;         // non-null: the launch does nothing unless *guard != 0
    // kFilter: a row's candidates are kept in one list per (4096-key chunk, TMEM lane
    // quadrant), so that each list has a single writer (one epilogue warp) and needs no
    // atomics: list (r, c, q) holds cq slots of {order key, key index} at
    // cand[((r * nchunk_max + c) * 4 + q) * cq] and its length (also past cq) in
    // ccount[(r * nchunk_max + c) * 4 + q]
    const uint32_t* tau;      // per row: threshold as an order key
    uint2* cand;
    uint32_t* ccount;
    int cq, nchunk_max;

    int q_begin, q_end;  // prefill query rows [q_begin, q_end)
    int S;               // prefill: key rows
    int num_units;
    int nb;              // prefill: query blocks in the window
    int nchunks;         // prefill: key chunks of the longest block
    // decode
    const int* page_table;
    const int* seq_lens;
    int max_pages, page_size, num_pages, max_len;
    unsigned* err;
};

// d0 += a0 * b0, d1 += a1 * b1 as one packed fp32x2 FMA (PTX fma.rn.f32x2, sm_100a): each
// lane is rounded once, exactly like fmaf
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 pa, pb, pc;\n\t"
        "mov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\tmov.b64 pc, {%0, %1};\n\t"
        "fma.rn.f32x2 pc, pa, pb, pc;\n\tmov.b64 {%0, %1}, pc;\n\t}"
        : "+f"(d0), "+f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Unit visited by this CTA at step i (snake order over rounds of gridDim.x units).
__device__ __forceinline__ int unit_at(int i) {
    const int G = gridDim.x, c = blockIdx.x;
    return (i & 1) ? i * G + (G - 1 - c) : i * G + c;
}

template <int QB, bool PAGED>
struct UnitInfo {
    int row0;       // prefill: first query t0; decode: sequence b
    int tile0;      // first key tile
    int ntiles;     // key tiles in this unit
    int len;        // decode: valid keys of the sequence
};

// Prefill: first query block whose causal key range reaches key chunk c (chunks count
// logical tiles, of which each is tile_stride physical tiles apart).
__host__ __device__ __forceinline__ int first_block_of_chunk(int c, int q_begin, int QB,
                                                            int tile_stride) {
    const long long need =
        (long long)c * kPrefillChunkTiles * kBM * tile_stride - q_begin - QB + 1;
    return need <= 0 ? 0 : (int)((need + QB - 1) / QB);
}

template <int QB, bool PAGED>
__device__ __forceinline__ UnitInfo<QB, PAGED> unit_info(const IdxParams& p, int u) {
    UnitInfo<QB, PAGED> x;
    if constexpr (!PAGED) {
        // units are enumerated chunk by chunk: chunk c covers blocks first_block(c)..nb-1
        int c = 0, rem = u, b = 0;
        for (; c < p.nchunks; ++c) {
            const int b0 = min(first_block_of_chunk(c, p.q_begin, QB, p.tile_stride), p.nb);
            const int cnt = p.nb - b0;
            if (rem < cnt) { b = b0 + rem; break; }
            rem -= cnt;
        }
        x.row0 = p.q_begin + b * QB;
        const int t_max = min(x.row0 + QB, p.q_end) - 1;
        const int total = t_max / (kBM * p.tile_stride) + 1;  // logical tiles reaching t_max
        x.tile0 = c * kPrefillChunkTiles;
        x.ntiles = max(0, min(kPrefillChunkTiles, total - x.tile0));
        x.len = min(x.row0 + QB, p.q_end) - x.row0;  // queries in the block
    } else {
        const int units_per_seq = (p.max_len + kBM * kDecodeChunkTiles - 1) / (kBM * kDecodeChunkTiles);
        x.row0 = u / units_per_seq;
        const int chunk = u % units_per_seq;
        int len = __ldg(p.seq_lens + x.row0);
        len = max(0, min(len, p.max_len));
        x.len = len;
        x.tile0 = chunk * kDecodeChunkTiles;
        const int tiles_total = (len + kBM - 1) / kBM;
        x.ntiles = max(0, min(kDecodeChunkTiles, tiles_total - x.tile0));
    }
    return x;
}

// One unit's copies, issued by a producer thread: the query block and its head weights
// (producer 0, once the previous user of the buffer is done), then the key tiles of the
// producer's ring stages (every stage in prefill; every kDecodeProducers-th, from stage
// pw on, for paged keys, whose pool rows come from the producer's sm.pages[pw]).  Returns
// false when a wait gave up.
template <int QB, bool PAGED>
__device__ __forceinline__ bool produce_unit(IdxSmem<QB>& sm, const IdxParams& p,
                                             const UnitInfo<QB, PAGED>& x, int ui, uint32_t& it,
                                             const CUtensorMap* tmap_q, const CUtensorMap* tmap_k,
                                             volatile int* abort, int pw) {
    const int qb = ui & 1;
    if (pw == 0) {
        if (!mbar_wait(&sm.q_empty[qb], ((ui >> 1) & 1) ^ 1, abort, p.err)) return false;
        // query block (TMA, swizzled) and its head weights (bulk copy) on one barrier
        const int nq = PAGED ? 1 : x.len;
        const uint32_t wbytes = (uint32_t)nq * kHI * 4;
        mbar_arrive_expect_tx(&sm.q_full[qb], (uint32_t)(QB * kHI * 128) + wbytes);
        tma_load_2d(sm.q[qb], tmap_q, 0, x.row0 * kHI, &sm.q_full[qb]);
        bulk_load(sm.w[qb], p.w + (long long)x.row0 * kHI, wbytes, &sm.q_full[qb]);
    }
    for (int j = 0; j < x.ntiles; ++j, ++it) {
        constexpr int kStages = IdxSmem<QB>::kStages;
        const int st = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (PAGED && st % kDecodeProducers != pw) continue;
        if (!mbar_wait(&sm.k_empty[st], ph ^ 1, abort, p.err)) return false;
        const int tile = (x.tile0 + j) * (PAGED ? 1 : p.tile_stride);
        if constexpr (!PAGED) {
            mbar_arrive_expect_tx(&sm.k_full[st], kTileBytes);
            tma_load_2d(sm.k[st], tmap_k, 0, tile * kBM, &sm.k_full[st]);
        } else {
            const int ps = p.page_size;
            const int per = kBM / ps;
            const int used = min(per, (x.len - tile * kBM + ps - 1) / ps);
            mbar_arrive_expect_tx(&sm.k_full[st], (uint32_t)(used * ps * 128));
            for (int q = 0; q < used; ++q)
                tma_load_2d(sm.k[st] + q * ps * 128, tmap_k, 0, sm.pages[pw][j * per + q] * ps,
                            &sm.k_full[st]);
        }
    }
    return true;
}

template <int QB, bool PAGED, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
indexer_tc_kernel(const __grid_constant__ CUtensorMap tmap_q,
                  const __grid_constant__ CUtensorMap tmap_k, const IdxParams p) {
    constexpr int BN = QB * kHI;                     // UMMA N
    constexpr uint32_t kAccCols = BN < 32 ? 32 : BN;  // TMEM columns per accumulator
    // as many accumulators (at most 4) as the 512 TMEM columns hold: the MMA warp runs
    // that many tiles ahead of the drain
    constexpr int kAcc = 512 / kAccCols >= 4 ? 4 : (int)(512 / kAccCols);
    constexpr uint32_t kTmemCols = kAcc * kAccCols <= 32 ? 32 : (kAcc * kAccCols <= 64 ? 64 : (kAcc * kAccCols <= 128 ? 128 : (kAcc * kAccCols <= 256 ? 256 : 512)));
    constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, BN, 0, 0);
    using Smem = IdxSmem<QB>;
    // One query per block (decode): the four query quarters of the epilogue take turns on
    // the tiles, each with an accumulator of its own, so four tiles drain at a time
    // instead of one tile by a quarter of the warps.
    constexpr bool kSplitTiles = QB == 1;
    static_assert(!kSplitTiles || kAcc == 4, "tile turns need one accumulator per quarter");

    static_assert(MODE == kDense || !PAGED, "decode stores dense rows");
    chained_launch_gate();
    if (p.guard != nullptr && *p.guard == 0) return;  // a fallback launch with nothing to do
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int* abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int i = 0; i < Smem::kStages; ++i) {
            mbar_init(&sm.k_full[i], 1);
            mbar_init(&sm.k_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.q_full[i], 1);
            mbar_init(&sm.q_empty[i], 1 + kEpiWarps);  // UMMA commit + epilogue warps
        }
        for (int i = 0; i < kAcc; ++i) {
            mbar_init(&sm.acc_full[i], 1);
            mbar_init(&sm.acc_empty[i], kSplitTiles ? 4 : kEpiWarps);
        }
        sm.abort = 0;
        fence_barrier_init();
    }
    if (warp == 2) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0 || (PAGED && (warp == 2 || warp == 3))) {
        // ---------------- TMA producer(s) ----------------
        const int pw = warp == 0 ? 0 : warp - 1;  // paged keys: producers 0, 1, 2
        // Lane 0 issues the copies.  For paged keys each producer warp reads a unit's
        // page-table entries into its own shared copy first (one round trip per unit, not a
        // dependent load before every tile's copies), and the next unit's entries are
        // loaded into registers while lane 0 issues this unit's copies, so that round trip
        // overlaps them.
        if (lane == 0) {
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_k);
        }
        constexpr int kPgLane = kDecodeChunkTiles * kBM / 16 / 32;  // entries per lane (pages >= 16)
        int pg_next[kPgLane];
        auto load_pages = [&](int u, int (&dst)[kPgLane]) {
            if constexpr (PAGED) {
                if (u < p.num_units) {
                    const UnitInfo<QB, PAGED> y = unit_info<QB, PAGED>(p, u);
                    const int per = kBM / p.page_size;
                    const int npg = min(y.ntiles * per, (y.len - y.tile0 * kBM + p.page_size - 1) / p.page_size);
                    const int* pt = p.page_table + (long long)y.row0 * p.max_pages + y.tile0 * per;
#pragma unroll
                    for (int i = 0; i < kPgLane; ++i) {
                        const int q = lane + 32 * i;
                        dst[i] = q < npg ? __ldg(pt + q) : 0;
                    }
                }
            }
        };
        load_pages(unit_at(0), pg_next);
        uint32_t it = 0;
        for (int i = 0, ui = 0;; ++i, ++ui) {
            const int u = unit_at(i);
            if (u >= p.num_units) break;
            const UnitInfo<QB, PAGED> x = unit_info<QB, PAGED>(p, u);
            if constexpr (PAGED) {
                const int per = kBM / p.page_size;
                const int npg = min(x.ntiles * per, (x.len - x.tile0 * kBM + p.page_size - 1) / p.page_size);
#pragma unroll
                for (int j = 0; j < kPgLane; ++j) {
                    const int q = lane + 32 * j;
                    if (q < npg) {
                        int pg = pg_next[j];
                        if (pg < 0 || pg >= p.num_pages) {
                            atomicOr(p.err, DSA_DEVERR_PAGE_RANGE);
                            pg = 0;
                        }
                        sm.pages[pw][q] = pg;
                    }
                }
                __syncwarp();
                load_pages(unit_at(i + 1), pg_next);
            }
            bool ok = true;
            if (lane == 0) ok = produce_unit<QB, PAGED>(sm, p, x, ui, it, &tmap_q, &tmap_k, abort, pw);
            ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
            __syncwarp();  // lane 0 has issued every copy that reads sm.pages
            if (!ok) break;
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- UMMA issuer ----------------
        uint32_t it = 0;
        for (int i = 0, ui = 0;; ++i, ++ui) {
            const int u = unit_at(i);
            if (u >= p.num_units) break;
            const UnitInfo<QB, PAGED> x = unit_info<QB, PAGED>(p, u);
            const int qb = ui & 1;
            if (!mbar_wait(&sm.q_full[qb], (ui >> 1) & 1, abort, p.err)) break;
            const uint32_t q_addr = smem_u32(sm.q[qb]);
            bool ok = true;
            for (int j = 0; j < x.ntiles; ++j, ++it) {
                const int st = it % Smem::kStages;
                const uint32_t ph = (it / Smem::kStages) & 1;
                const int ab = it % kAcc;
                const uint32_t aph = (it / kAcc) & 1;
                if (!mbar_wait(&sm.k_full[st], ph, abort, p.err)) { ok = false; break; }
                if (!mbar_wait(&sm.acc_empty[ab], aph ^ 1, abort, p.err)) { ok = false; break; }
                tc_fence_after();
                const uint64_t adesc = smem_desc(smem_u32(sm.k[st]), 16, 1024, kSwizzle128B);
                const uint64_t bdesc = smem_desc(q_addr, 16, 1024, kSwizzle128B);
#pragma unroll
                for (int kk = 0; kk < kDI / 16; ++kk)
                    umma_bf16(tmem + ab * kAccCols, adesc + 2 * kk, bdesc + 2 * kk, kIdesc, kk > 0);
                umma_commit(&sm.k_empty[st]);
                umma_commit(&sm.acc_full[ab]);
            }
            umma_commit(&sm.q_empty[qb]);
            if (!ok) break;
        }
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kEpiWarps) {
        // ---------------- epilogue ----------------
        const int ew = warp - kEpiWarp0;
        const int quad = warp & 3;              // TMEM lane quadrant this warp may access
        const int part = ew >> 2;               // which quarter of the queries
        constexpr int QPW = QB >= 4 ? QB / 4 : 1;  // queries per epilogue warp
        // with at most two queries per warp their 32 head weights stay in registers for
        // the whole unit; otherwise they are read from shared memory per tile
        constexpr bool kHoist = QPW <= 2;
        const bool active = QB >= 4 || kSplitTiles;
        const int qbase = kSplitTiles ? 0 : part * QPW;  // this warp's first query of the block
        uint32_t it = 0;
        for (int i = 0, ui = 0;; ++i, ++ui) {
            const int u = unit_at(i);
            if (u >= p.num_units) break;
            const UnitInfo<QB, PAGED> x = unit_info<QB, PAGED>(p, u);
            const int qb = ui & 1;
            if (!mbar_wait(&sm.q_full[qb], (ui >> 1) & 1, abort, p.err)) break;
            const float* wbuf = sm.w[qb] + qbase * kHI;  // this warp's queries' weights
            float wreg[kHoist ? QPW * kHI : 1];
            if constexpr (kHoist) {
#pragma unroll
                for (int h4 = 0; h4 < QPW * kHI / 4; ++h4) {
                    const float4 wv = reinterpret_cast<const float4*>(wbuf)[h4];
                    wreg[4 * h4] = wv.x;
                    wreg[4 * h4 + 1] = wv.y;
                    wreg[4 * h4 + 2] = wv.z;
                    wreg[4 * h4 + 3] = wv.w;
                }
            }
            float tau[QPW];      // kFilter: the thresholds of this warp's queries as floats
            uint32_t ncand[QPW]; // kFilter: candidates this warp appended per query
#pragma unroll
            for (int qi = 0; qi < QPW; ++qi) {
                const int r = x.row0 + qbase + qi - p.q_begin;
                // an order key >= tau[r] is exactly a score >= the float the key stands for
                const uint32_t tk =
                    (MODE == kFilter && qbase + qi < x.len) ? __ldg(p.tau + r) : 0u;
                tau[qi] = __uint_as_float((tk & 0x80000000u) ? (tk & 0x7FFFFFFFu) : ~tk);
                ncand[qi] = 0u;
            }
            const int chunk = x.tile0 / kPrefillChunkTiles;
            bool ok = true;
            for (int j = 0; j < x.ntiles; ++j, ++it) {
                const int ab = it % kAcc;
                const uint32_t aph = (it / kAcc) & 1;
                if (kSplitTiles && ab != part) continue;  // another quarter drains this tile
                if (!mbar_wait(&sm.acc_full[ab], aph, abort, p.err)) { ok = false; break; }
                tc_fence_after();
                const int lt = x.tile0 + j;  // logical tile
                const int tile_key0 = lt * (PAGED ? 1 : p.tile_stride) * kBM;
                const int s = tile_key0 + quad * 32 + lane;
                // every key of the tile precedes every query of the block: no causal test
                const bool below = !PAGED && tile_key0 + kBM - 1 <= x.row0 && x.len == QB;
                const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + ab * kAccCols;
                if (active) {
                    constexpr int QW = QPW < 2 ? QPW : 2;  // queries per TMEM load round
#pragma unroll
                    for (int qi = 0; qi < QPW; qi += QW) {
                        uint32_t r[QW][16];
                        const int i0 = qbase + qi;
#pragma unroll
                        for (int qq = 0; qq < QW; ++qq) tmem_ld16(tbase + (i0 + qq) * kHI, r[qq]);
                        tmem_wait_ld();
#pragma unroll
                        for (int qq = 0; qq < QW; ++qq) {
                            const int qidx = i0 + qq;
                            const int qo = qidx - qbase;
                            // even heads accumulate in acc0, odd heads in acc1
                            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                            for (int h4 = 0; h4 < 4; ++h4) {
                                float4 wv;
                                if constexpr (kHoist) {
                                    wv = make_float4(wreg[qo * kHI + 4 * h4], wreg[qo * kHI + 4 * h4 + 1],
                                                     wreg[qo * kHI + 4 * h4 + 2], wreg[qo * kHI + 4 * h4 + 3]);
                                } else {
                                    wv = reinterpret_cast<const float4*>(wbuf + qo * kHI)[h4];
                                }
                                const uint32_t* rv = r[qq] + 4 * h4;
                                ffma2(acc0, acc1, wv.x, wv.y, fmaxf(__uint_as_float(rv[0]), 0.f),
                                      fmaxf(__uint_as_float(rv[1]), 0.f));
                                ffma2(acc0, acc1, wv.z, wv.w, fmaxf(__uint_as_float(rv[2]), 0.f),
                                      fmaxf(__uint_as_float(rv[3]), 0.f));
                            }
                            const float score = acc0 + acc1;
                            if constexpr (PAGED) {
                                if (s < x.len) p.scores[(long long)x.row0 * p.ld + s] = score;
                            } else if constexpr (MODE == kDense) {
                                const int t = x.row0 + qidx;
                                if (below || (qidx < x.len && s <= t))
                                    p.scores[(long long)(t - p.q_begin) * p.ld + s] = score;
                            } else if constexpr (MODE == kSample) {
                                // compact sample row: logical tile lt at columns lt*128..
                                const int t = x.row0 + qidx;
                                if (qidx < x.len && s <= t)
                                    p.scores[(long long)(t - p.q_begin) * p.ld + lt * kBM +
                                             quad * 32 + lane] = score;
                            } else {
                                // the warp's 32 lanes are 32 consecutive keys: one ballot is
                                // one append batch of the (row, chunk, quadrant) list
                                const int t = x.row0 + qidx;
                                const long long r = t - p.q_begin;
                                const bool valid = qidx < x.len && s <= t;
                                const bool gt = valid && score >= tau[qo];
                                const unsigned gtm = __ballot_sync(0xffffffffu, gt);
                                if (gtm) {
                                    const uint32_t pos = ncand[qo] + __popc(gtm & ((1u << lane) - 1u));
                                    if (gt && pos < (uint32_t)p.cq)
                                        p.cand[((r * p.nchunk_max + chunk) * 4 + quad) * p.cq + pos] =
                                            make_uint2(float_order_key(score), (uint32_t)s);
                                    ncand[qo] += __popc(gtm);
                                }
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.acc_empty[ab]);
            }
            if (!ok) break;
            if constexpr (MODE == kFilter) {
                if (active && lane < QPW && qbase + lane < x.len) {
                    uint32_t nc = 0;
#pragma unroll
                    for (int qi = 0; qi < QPW; ++qi) nc = lane == qi ? ncand[qi] : nc;
                    const long long r = x.row0 + qbase + lane - p.q_begin;
                    p.ccount[(r * p.nchunk_max + chunk) * 4 + quad] = nc;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.q_empty[qb]);  // done with this unit's weights
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int QB, bool PAGED>
size_t indexer_smem_bytes() {
    return sizeof(IdxSmem<QB>) + 1024;
}

template <int QB, bool PAGED, int MODE>
cudaError_t launch_indexer_tc(const CUtensorMap& tq, const CUtensorMap& tk, const IdxParams& p,
                              int grid, cudaStream_t stream) {
    const size_t smem = indexer_smem_bytes<QB, PAGED>();
    cudaError_t e = cudaFuncSetAttribute(indexer_tc_kernel<QB, PAGED, MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_chained(indexer_tc_kernel<QB, PAGED, MODE>, dim3(grid), dim3(kThreads), smem, stream,
                       1, tq, tk, p);
    count_launch(DSA_KERNEL_INDEXER);
    return e;
}

// Prefill launch of any mode: tensor maps, the unit count of the window and the grid.
template <int MODE>
cudaError_t launch_prefill(const __nv_bfloat16* q_idx, const __nv_bfloat16* k_idx, int T, int S,
                           IdxParams p, cudaStream_t stream, const DevCtx& ctx) {
    constexpr int QB = kPrefillQB;
    CUtensorMap tq, tk;
    if (!make_tmap_bf16_2d(&tq, q_idx, (uint64_t)T * kHI, kDI, kDI * 2, QB * kHI, kDI))
        return cudaErrorInvalidValue;
    if (!make_tmap_bf16_2d(&tk, k_idx, (uint64_t)S, kDI, kDI * 2, kBM, kDI))
        return cudaErrorInvalidValue;
    const int rows = p.q_end - p.q_begin;
    p.S = S;
    p.nb = (rows + QB - 1) / QB;
    {
        const int t_max = p.q_end - 1;
        const int logical_tiles = t_max / (kBM * p.tile_stride) + 1;
        p.nchunks = (logical_tiles + kPrefillChunkTiles - 1) / kPrefillChunkTiles;
        long long units = 0;
        for (int c = 0; c < p.nchunks; ++c) {
            int b0 = first_block_of_chunk(c, p.q_begin, QB, p.tile_stride);
            units += p.nb - (b0 < p.nb ? b0 : p.nb);
        }
        p.num_units = (int)units;
    }
    p.err = ctx.err;
    const int grid = p.num_units < ctx.num_sms ? p.num_units : ctx.num_sms;
    if (grid <= 0) return cudaSuccess;
    return launch_indexer_tc<QB, false, MODE>(tq, tk, p, grid, stream);
}

}  // namespace

cudaError_t launch_indexer_bf16_prefill(const __nv_bfloat16* q_idx, const __nv_bfloat16* k_idx,
                                        const float* w, int T, int S, int q_begin, int rows,
                                        float* scores, long long ld, cudaStream_t stream,
                                        const DevCtx& ctx, const int* guard) {
    IdxParams p{};
    p.w = w;
    p.scores = scores;
    p.ld = ld;
    p.tile_stride = 1;
    p.guard = guard;
    p.q_begin = q_begin;
    p.q_end = q_begin + rows;
    return launch_prefill<kDense>(q_idx, k_idx, T, S, p, stream, ctx);
}

cudaError_t launch_indexer_bf16_sample(const __nv_bfloat16* q_idx, const __nv_bfloat16* k_idx,
                                       const float* w, int T, int S, int q_begin, int rows,
                                       int tile_stride, float* sample, long long ld_sample,
                                       cudaStream_t stream, const DevCtx& ctx) {
    IdxParams p{};
    p.w = w;
    p.scores = sample;
    p.ld = ld_sample;
    p.tile_stride = tile_stride;
    p.q_begin = q_begin;
    p.q_end = q_begin + rows;
    return launch_prefill<kSample>(q_idx, k_idx, T, S, p, stream, ctx);
}

cudaError_t launch_indexer_bf16_filter(const __nv_bfloat16* q_idx, const __nv_bfloat16* k_idx,
                                       const float* w, int T, int S, int q_begin, int rows,
                                       const uint32_t* tau, uint2* cand, uint32_t* ccount, int cq,
                                       int nchunk_max, cudaStream_t stream, const DevCtx& ctx) {
    IdxParams p{};
    p.w = w;
    p.tile_stride = 1;
    p.tau = tau;
    p.cand = cand;
    p.ccount = ccount;
    p.cq = cq;
    p.nchunk_max = nchunk_max;
    p.q_begin = q_begin;
    p.q_end = q_begin + rows;
    return launch_prefill<kFilter>(q_idx, k_idx, T, S, p, stream, ctx);
}

cudaError_t launch_indexer_bf16_decode(const __nv_bfloat16* q_idx, const __nv_bfloat16* k_pool,
                                       const float* w, int B, long long pool_rows,
                                       const int* page_table, int max_pages, int page_size,
                                       const int* seq_lens, int max_len, float* scores,
                                       long long ld, cudaStream_t stream, const DevCtx& ctx) {
    CUtensorMap tq, tk;
    if (!make_tmap_bf16_2d(&tq, q_idx, (uint64_t)B * kHI, kDI, kDI * 2, kHI, kDI))
        return cudaErrorInvalidValue;
    if (!make_tmap_bf16_2d(&tk, k_pool, (uint64_t)pool_rows, kDI, kDI * 2, page_size, kDI))
        return cudaErrorInvalidValue;
    IdxParams p{};
    p.w = w;
    p.scores = scores;
    p.ld = ld;
    p.page_table = page_table;
    p.seq_lens = seq_lens;
    p.max_pages = max_pages;
    p.page_size = page_size;
    p.num_pages = (int)(pool_rows / page_size);
    p.max_len = max_len;
    const int units_per_seq = (max_len + kBM * kDecodeChunkTiles - 1) / (kBM * kDecodeChunkTiles);
    p.num_units = B * units_per_seq;
    p.err = ctx.err;
    const int grid = p.num_units < ctx.num_sms ? p.num_units : ctx.num_sms;
    p.tile_stride = 1;
    return launch_indexer_tc<1, true, kDense>(tq, tk, p, grid, stream);
}

}  // namespace dsa
