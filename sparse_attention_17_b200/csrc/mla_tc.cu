// mla_tc.cu -- sparse absorbed-MLA attention on tcgen05 tensor cores (prefill and paged
// decode), plus the log-sum-exp merge of decode splits.
//
// For query n and head h (16 heads), over the selected keys I_n only:
//   logit_s  = scale * q[n,h,0:576] . C[s,0:576]          C = 576-dim latent row
//   out[n,h] = sum_s softmax(logit)_s * C[s,0:512]          value = first 512 latent dims
// (DSV2-Lite-IndexCache card: attention_mode="sparse" over the selected routes;
//  DeepSeek-V2-Lite-Chat SIQ card: MLA with kv_lora_rank 512 and 576 elements per token.)
//
// Design.  With 16 heads the natural GEMMs have M = 16, below the UMMA minimum, so both
// products are taken transposed, with keys or latent dims on the M side:
//   S^T[64 keys x 16 heads]   = C_blk[64 x 576]  . Q^T[576 x 16]     (M=64,  N=16, K=576)
//   O^T[512 dims x 16 heads] += C_blk^T[512 x 64] . P^T[64 x 16]     (M=128, N=16, K=64)
// The gathered block C_blk is written once into shared memory in the canonical K-major
// 128-byte-swizzled layout (9 chunks of 64 dims x 64 keys).  Read along the other axis the
// very same bytes are a valid MN-major operand (64 dims per 128-byte line, 8 keys per
// 1024-byte atom), so the PV product reuses the tile without any transpose or copy.
//
// Warp roles (288 threads):
//   warps 5..8  gather: each selected row (1152 B) is fetched with 16-byte cp.async copies
//               straight into the swizzled tile (invalid / padding rows are zero-filled);
//               completion arrives on an mbarrier.  Warp 5 also TMA-loads the 16x576 query.
//   warp 4      TMEM owner and UMMA issuer: QK of block j+1 is issued before PV of block j.
//   warps 0..3  softmax (one per TMEM lane quadrant): block max per head, running max
//               with lazy rescaling (O is rescaled in TMEM only when a head's max grows by
//               more than 2^8), P = exp2(.) in bf16 to shared memory, per-thread partial
//               row sums; at the end of a query they normalise O and write out / lse.
// Two smem stages of 64 keys (2 x 72 KB) keep the next gather in flight during softmax
// and PV.  Decode splits the selected keys of a sequence over several CTAs; their
// normalised partial outputs and log-sum-exps are merged by mla_combine_kernel.
#include "dsa_common.cuh"
#include "launch.h"

namespace dsa {

namespace {

constexpr int kH = 16;
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kBK = 64;                       // keys per block / stage
constexpr int kChunks = kDqk / 64;            // 9 chunks of 64 dims (128 B)
constexpr uint32_t kChunkBytes = kBK * 128;   // 8 KB
constexpr uint32_t kStageBytes = kChunks * kChunkBytes;  // 72 KB
constexpr uint32_t kQChunkBytes = kH * 128;   // 2 KB
constexpr uint32_t kQBytes = kChunks * kQChunkBytes;      // 18 KB
constexpr uint32_t kPBytes = kH * 128;        // 16 heads x 64 keys bf16
constexpr int kThreads = 288;
constexpr int kMmaWarp = 4;
constexpr int kGatherWarp0 = 5;
constexpr int kGatherThreads = 128;
constexpr int kIdxCap = 2048;                 // index entries of one unit held in smem
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kOCol = 0;                 // O^T: 4 M-tiles x 16 columns
constexpr uint32_t kSCol = 64;                // S^T of stage s at kSCol + 16 s
constexpr float kRescaleThreshold = 8.0f;     // log2 units

constexpr uint32_t kIdescQK = idesc_bf16_f32(64, kH, 0, 0);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, kH, 1, 0);

struct MlaSmem {
    alignas(1024) uint8_t a[2][kStageBytes];
    alignas(1024) uint8_t q[2][kQBytes];
    alignas(1024) uint8_t p[2][kPBytes];
    alignas(16) int idx[2][kIdxCap];  // the unit's selected indices (bulk-copied with Q)
    alignas(16) float red[2][4][kH];
    float lred[8][kH];
    uint64_t a_full[2], s_full[2], p_full[2], pv_done[2];
    uint64_t q_full[2], q_empty[2];
    uint64_t o_free;
    uint64_t red_bar[2];   // softmax warps exchange block maxima (bounded-wait barrier)
    uint64_t epi_bar;      // softmax warps exchange row sums at the end of a unit
    uint32_t tmem_base;
    int abort;
};

struct MlaParams {
    const __nv_bfloat16* kv;
    long long kv_rows;
    const int* page_table;  // NULL = prefill
    int max_pages, page_size, num_pages;
    const int* seq_lens;
    const int* idx;
    int k_sel;
    long long ld_idx;
    int num_q;
    int splits;      // decode: key ranges per sequence (1 in prefill)
    int chunk;       // decode: index entries per split (multiple of kBK)
    int num_units;
    float scale_log2;
    __nv_bfloat16* out;
    float* lse;
    float* o_part;
    float* lse_part;
    unsigned* err;
};

struct Unit {
    int n;       // query (prefill) or sequence (decode)
    int sp;      // split
    int e0, e1;  // index entries [e0, e1) of row n
    int nb;      // 64-key blocks
    int len;     // decode: valid length of the sequence
};

__device__ __forceinline__ Unit unit_of(const MlaParams& p, int u) {
    Unit x;
    if (p.page_table == nullptr) {
        x.n = u;
        x.sp = 0;
        x.e0 = 0;
        x.e1 = p.k_sel;
        x.len = 0;
    } else {
        x.n = u / p.splits;
        x.sp = u % p.splits;
        x.e0 = x.sp * p.chunk;
        x.e1 = min(p.k_sel, x.e0 + p.chunk);
        // keys beyond the page table's capacity cannot be addressed
        x.len = min(__ldg(p.seq_lens + x.n), p.max_pages * p.page_size);
    }
    x.nb = x.e1 > x.e0 ? (x.e1 - x.e0 + kBK - 1) / kBK : 0;
    return x;
}

// Row of the latent cache for index entry e of unit x, or -1 (padding / invalid).
// `uidx` holds the unit's entries e0..e1-1 (shared memory).  Out-of-range entries are
// recorded in the error word when `report` is set.
__device__ __forceinline__ long long resolve_row(const MlaParams& p, const Unit& x,
                                                 const int* uidx, int e, bool report) {
    if (e >= x.e1) return -1;
    const int s = uidx[e - x.e0];
    if (s < 0) return -1;
    if (p.page_table == nullptr) {
        if (s >= p.kv_rows) {
            if (report) atomicOr(p.err, DSA_DEVERR_INDEX_RANGE);
            return -1;
        }
        return s;
    }
    if (s >= x.len) {
        if (report) atomicOr(p.err, DSA_DEVERR_INDEX_RANGE);
        return -1;
    }
    const int pg = __ldg(p.page_table + (long long)x.n * p.max_pages + s / p.page_size);
    if (pg < 0 || pg >= p.num_pages) {
        if (report) atomicOr(p.err, DSA_DEVERR_PAGE_RANGE);
        return -1;
    }
    return (long long)pg * p.page_size + s % p.page_size;
}

// Inverse of float_order_key.
__device__ __forceinline__ float order_key_to_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

__global__ void __launch_bounds__(kThreads, 1)
sparse_mla_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const MlaParams p) {
    extern __shared__ uint8_t smem_raw[];
    MlaSmem& sm = *reinterpret_cast<MlaSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int* abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.a_full[i], kGatherThreads);
            mbar_init(&sm.s_full[i], 1);
            mbar_init(&sm.p_full[i], 4);
            mbar_init(&sm.pv_done[i], 1);
            mbar_init(&sm.q_full[i], 1);
            mbar_init(&sm.q_empty[i], 1 + 4 + 4);  // UMMA commit + gather + softmax warps
        }
        mbar_init(&sm.o_free, 4);
        mbar_init(&sm.red_bar[0], 4);
        mbar_init(&sm.red_bar[1], 4);
        mbar_init(&sm.epi_bar, 4);
        sm.abort = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp >= kGatherWarp0) {
        // ============================ gather ============================
        const int gw = warp - kGatherWarp0;  // keys gw*16 .. gw*16+15 of each block
        const bool q_leader = (gw == 0 && lane == 0);
        if (q_leader) tma_prefetch_desc(&tmap_q);
        // The leader issues each unit's query (TMA) and index entries (bulk copy) into the
        // double buffer as soon as the buffer is free, one unit ahead where possible.
        int issued = 0;
        auto issue_unit_loads = [&](bool blocking) {
            const int u2 = blockIdx.x + issued * gridDim.x;
            if (u2 >= p.num_units) return;
            const int qb2 = issued & 1;
            const uint32_t par = ((issued >> 1) & 1) ^ 1;
            const bool free = blocking ? mbar_wait(&sm.q_empty[qb2], par, abort, p.err)
                                       : mbar_try_wait(&sm.q_empty[qb2], par);
            if (!free) return;
            const Unit y = unit_of(p, u2);
            const uint32_t ibytes = (uint32_t)(y.e1 - y.e0) * 4u;
            mbar_arrive_expect_tx(&sm.q_full[qb2], kQBytes + ibytes);
            for (int c = 0; c < kChunks; ++c)
                tma_load_2d(sm.q[qb2] + c * kQChunkBytes, &tmap_q, c * 64, y.n * kH,
                            &sm.q_full[qb2]);
            if (ibytes)
                bulk_load(sm.idx[qb2], p.idx + (long long)y.n * p.ld_idx + y.e0, ibytes,
                          &sm.q_full[qb2]);
            ++issued;
        };
        uint32_t G = 0;
        for (int ui = 0;; ++ui) {
            const int u = blockIdx.x + ui * gridDim.x;
            if (u >= p.num_units) break;
            const Unit x = unit_of(p, u);
            const int qb = ui & 1;
            if (q_leader) {
                while (issued <= ui && !*abort) issue_unit_loads(true);
                issue_unit_loads(false);  // prefetch the next unit if its buffer is free
            }
            if (!mbar_wait(&sm.q_full[qb], (ui >> 1) & 1, abort, p.err)) break;
            const int* uidx = sm.idx[qb];
            bool ok = true;
            for (int j = 0; j < x.nb; ++j, ++G) {
                const int s = G & 1;
                const uint32_t ph = (G >> 1) & 1;
                if (!mbar_wait(&sm.pv_done[s], ph ^ 1, abort, p.err)) { ok = false; break; }
                long long row = -1;
                if (lane < 16) row = resolve_row(p, x, uidx, x.e0 + j * kBK + gw * 16 + lane, true);
                // lane l copies the 16-byte units l, l+32 and (l < 8) l+64 of each of the warp's
                // 16 rows; unit u of row r goes to chunk u/8, line r, slot (u%8) ^ (r%8)
                const uint32_t a_lane = smem_u32(sm.a[s]) + (lane >> 3) * kChunkBytes;
                const char* kvb = reinterpret_cast<const char*>(p.kv) + lane * 16;
#pragma unroll 4
                for (int kl = 0; kl < 16; ++kl) {
                    const long long rr = __shfl_sync(0xffffffffu, row, kl);
                    const int r = gw * 16 + kl;
                    const uint32_t dst = a_lane + r * 128 + (((lane & 7) ^ (r & 7)) << 4);
                    if (rr >= 0) {
                        const char* src = kvb + rr * (kDqk * 2);
                        cp_async_16(dst, src);
                        cp_async_16(dst + 4 * kChunkBytes, src + 512);
                        if (lane < 8) cp_async_16(dst + 8 * kChunkBytes, src + 1024);
                    } else {
                        cp_async_16_zero(dst, p.kv);
                        cp_async_16_zero(dst + 4 * kChunkBytes, p.kv);
                        if (lane < 8) cp_async_16_zero(dst + 8 * kChunkBytes, p.kv);
                    }
                }
                cp_async_mbar_arrive(&sm.a_full[s]);
                if (q_leader && issued == ui + 1) issue_unit_loads(false);
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.q_empty[qb]);  // done with this unit's indices
        }
        // let this thread's copies land before the CTA can exit
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp == kMmaWarp) {
        // ============================ UMMA ============================
        if (lane == 0) {
            uint32_t G = 0;
            int units_with_blocks = 0;
            // Descriptors are built once; per UMMA only a constant start-address offset
            // (in 16-byte units) is added.
            // (stage 1 / buffer 1 follow stage 0 / buffer 0 at a fixed distance)
            const uint64_t a_desc_k0 = smem_desc(smem_u32(sm.a[0]), 16, 1024, kSwizzle128B);
            const uint64_t a_desc_mn0 = smem_desc(smem_u32(sm.a[0]), kChunkBytes, 1024, kSwizzle128B);
            const uint64_t q_desc0 = smem_desc(smem_u32(sm.q[0]), 16, 1024, kSwizzle128B);
            const uint64_t p_desc0 = smem_desc(smem_u32(sm.p[0]), 16, 1024, kSwizzle128B);
            constexpr uint32_t kAStep = (uint32_t)(sizeof(MlaSmem::a[0]) >> 4);
            constexpr uint32_t kQStep = (uint32_t)(sizeof(MlaSmem::q[0]) >> 4);
            constexpr uint32_t kPStep = (uint32_t)(sizeof(MlaSmem::p[0]) >> 4);
            auto issue_pv_now = [&](uint32_t Gp, bool first) {
                const int s = Gp & 1;
                tc_fence_after();
                // K-step outer, M-tile inner: consecutive UMMAs go to different accumulators
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk) {
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        umma_bf16(tmem + kOCol + 16 * m,
                                  a_desc_mn0 + s * kAStep + ((2 * m * kChunkBytes + kk * 2048) >> 4),
                                  p_desc0 + s * kPStep + ((kk * 32) >> 4), kIdescPV,
                                  !(first && kk == 0));
                }
                umma_commit(&sm.pv_done[s]);
            };
            // PV of block Gp may start once its P is in smem (and, for the first block of
            // a unit, once the previous unit's epilogue has read O out of TMEM).
            auto pv_ready = [&](uint32_t Gp, bool first, int prior_units) -> bool {
                if (!mbar_try_wait(&sm.p_full[Gp & 1], (Gp >> 1) & 1)) return false;
                return !(first && prior_units > 0) ||
                       mbar_try_wait(&sm.o_free, (prior_units - 1) & 1);
            };
            auto issue_pv = [&](uint32_t Gp, bool first, int prior_units) -> bool {
                if (!mbar_wait(&sm.p_full[Gp & 1], (Gp >> 1) & 1, abort, p.err)) return false;
                if (first && prior_units > 0)
                    if (!mbar_wait(&sm.o_free, (prior_units - 1) & 1, abort, p.err)) return false;
                issue_pv_now(Gp, first);
                return true;
            };
            bool ok = true;
            for (int ui = 0; ok; ++ui) {
                const int u = blockIdx.x + ui * gridDim.x;
                if (u >= p.num_units) break;
                const Unit x = unit_of(p, u);
                const int qb = ui & 1;
                if (!mbar_wait(&sm.q_full[qb], (ui >> 1) & 1, abort, p.err)) break;
                for (int j = 0; j < x.nb; ++j, ++G) {
                    const int s = G & 1;
                    const uint32_t ph = (G >> 1) & 1;
                    // While block G's gather is in flight, start PV of block G-1 if its P is
                    // ready, so that stage G-1 is released as early as possible.
                    bool pv_prev_issued = j == 0;
                    if (!pv_prev_issued) {
                        for (uint32_t spin = 0; !mbar_try_wait(&sm.a_full[s], ph); ++spin) {
                            if (pv_ready(G - 1, j - 1 == 0, units_with_blocks)) {
                                issue_pv_now(G - 1, j - 1 == 0);
                                pv_prev_issued = true;
                                break;
                            }
                            if ((spin & 1023u) == 1023u && *abort) { ok = false; break; }
                        }
                        if (!ok) break;
                    }
                    if (!mbar_wait(&sm.a_full[s], ph, abort, p.err)) { ok = false; break; }
                    fence_proxy_async_smem();
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kDqk / 16; ++kk) {
                        const int c = kk >> 2, sub = kk & 3;
                        umma_bf16(tmem + kSCol + 16 * s,
                                  a_desc_k0 + s * kAStep + ((c * kChunkBytes + sub * 32) >> 4),
                                  q_desc0 + qb * kQStep + ((c * kQChunkBytes + sub * 32) >> 4),
                                  kIdescQK, kk > 0);
                    }
                    umma_commit(&sm.s_full[s]);
                    if (!pv_prev_issued && !issue_pv(G - 1, j - 1 == 0, units_with_blocks)) {
                        ok = false;
                        break;
                    }
                }
                umma_commit(&sm.q_empty[qb]);
                if (!ok) break;
                if (x.nb > 0) {
                    if (!issue_pv(G - 1, x.nb == 1, units_with_blocks)) break;
                    ++units_with_blocks;
                }
            }
        }
    } else {
        // ======================= softmax + epilogue =======================
        const int quad = warp;  // TMEM lanes 32*quad .. 32*quad+31
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        uint32_t G = 0;
        uint32_t epi_phase = 0;
        for (int ui = 0;; ++ui) {
            const int u = blockIdx.x + ui * gridDim.x;
            if (u >= p.num_units) break;
            const Unit x = unit_of(p, u);
            const int qb = ui & 1;
            if (!mbar_wait(&sm.q_full[qb], (ui >> 1) & 1, abort, p.err)) break;
            const int* uidx = sm.idx[qb];
            // l_part: sums of the bf16 probabilities fed to the PV product (normalises O);
            // l_lse: the same sums before rounding (for the log-sum-exp output)
            float m_ref[kH], l_part[kH], l_lse[kH];
#pragma unroll
            for (int h = 0; h < kH; ++h) { m_ref[h] = -INFINITY; l_part[h] = 0.f; l_lse[h] = 0.f; }
            bool ok = true;
            for (int j = 0; j < x.nb; ++j, ++G) {
                const int s = G & 1;
                const uint32_t ph = (G >> 1) & 1;
                // validity of this thread's key slot (M=64 layout: lanes 0..15 of each quadrant)
                const int r = quad * 16 + lane;
                const bool valid = lane < 16 && resolve_row(p, x, uidx, x.e0 + j * kBK + r, false) >= 0;
                if (!mbar_wait(&sm.s_full[s], ph, abort, p.err)) { ok = false; break; }
                tc_fence_after();
                uint32_t sr[16];
                tmem_ld16(tmem + lane_base + kSCol + 16 * s, sr);
                tmem_wait_ld();
                float xs[kH];
#pragma unroll
                for (int h = 0; h < kH; ++h)
                    xs[h] = valid ? __uint_as_float(sr[h]) * p.scale_log2 : -INFINITY;
                // block max per head: one redux per head over the warp, then across the 4
                // warps through shared memory (vector stores / loads, no branches)
                float wmax[kH];
#pragma unroll
                for (int h = 0; h < kH; ++h)
                    wmax[h] = order_key_to_float(
                        __reduce_max_sync(0xffffffffu, float_order_key(xs[h])));
                if (lane == 0) {
                    float4* dst = reinterpret_cast<float4*>(sm.red[s][quad]);
#pragma unroll
                    for (int h4 = 0; h4 < kH / 4; ++h4)
                        dst[h4] = make_float4(wmax[4 * h4], wmax[4 * h4 + 1], wmax[4 * h4 + 2],
                                              wmax[4 * h4 + 3]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.red_bar[s]);
                if (!mbar_wait(&sm.red_bar[s], ph, abort, p.err)) { ok = false; break; }
                float mb[kH];
#pragma unroll
                for (int h4 = 0; h4 < kH / 4; ++h4) {
                    const float4 a = reinterpret_cast<const float4*>(sm.red[s][0])[h4];
                    const float4 b = reinterpret_cast<const float4*>(sm.red[s][1])[h4];
                    const float4 c = reinterpret_cast<const float4*>(sm.red[s][2])[h4];
                    const float4 d = reinterpret_cast<const float4*>(sm.red[s][3])[h4];
                    mb[4 * h4 + 0] = fmaxf(fmaxf(a.x, b.x), fmaxf(c.x, d.x));
                    mb[4 * h4 + 1] = fmaxf(fmaxf(a.y, b.y), fmaxf(c.y, d.y));
                    mb[4 * h4 + 2] = fmaxf(fmaxf(a.z, b.z), fmaxf(c.z, d.z));
                    mb[4 * h4 + 3] = fmaxf(fmaxf(a.w, b.w), fmaxf(c.w, d.w));
                }
                // lazy reference: a head's reference moves only when its block max exceeds
                // it by more than 2^8 (or when it had no valid key yet); the decision is the
                // same in every thread because all read the same maxima
                bool rescale = false;
                float new_ref[kH];
#pragma unroll
                for (int h = 0; h < kH; ++h) {
                    const bool empty = m_ref[h] == -INFINITY;
                    const bool grow = !empty && mb[h] > m_ref[h] + kRescaleThreshold;
                    rescale |= grow;
                    new_ref[h] = (empty || grow) ? mb[h] : m_ref[h];
                }
                if (rescale) {
                    float alpha[kH];
#pragma unroll
                    for (int h = 0; h < kH; ++h)
                        alpha[h] = m_ref[h] == -INFINITY ? 1.f : exp2f(m_ref[h] - new_ref[h]);
                    // all earlier PV products must have landed before O is scaled in place
                    const uint32_t Gp = G - 1;
                    if (!mbar_wait(&sm.pv_done[Gp & 1], (Gp >> 1) & 1, abort, p.err)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        uint32_t o[16];
                        tmem_ld16(tmem + lane_base + kOCol + 16 * m, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int h = 0; h < kH; ++h)
                            o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
                        tmem_st16(tmem + lane_base + kOCol + 16 * m, o);
                    }
                    tmem_wait_st();
#pragma unroll
                    for (int h = 0; h < kH; ++h) { l_part[h] *= alpha[h]; l_lse[h] *= alpha[h]; }
                }
#pragma unroll
                for (int h = 0; h < kH; ++h) m_ref[h] = new_ref[h];
                // P buffer s is free once the PV product of block G-2 has completed
                if (!mbar_wait(&sm.pv_done[s], ph ^ 1, abort, p.err)) { ok = false; break; }
                if (lane < 16) {
                    uint8_t* pb = sm.p[s];
#pragma unroll
                    for (int h = 0; h < kH; ++h) {
                        // invalid keys carry xs = -inf, so exp2 gives exactly 0
                        const float ref = m_ref[h] == -INFINITY ? 0.f : m_ref[h];
                        const float pv = exp2f(xs[h] - ref);
                        const __nv_bfloat16 b = __float2bfloat16_rn(pv);
                        l_part[h] += __bfloat162float(b);
                        l_lse[h] += pv;
                        const int off = (h >> 3) * 1024 + (h & 7) * 128 +
                                        ((((2 * r) >> 4) ^ (h & 7)) << 4) + ((2 * r) & 15);
                        *reinterpret_cast<__nv_bfloat16*>(pb + off) = b;
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.p_full[s]);
            }
            if (!ok) break;

            // -------- epilogue of this unit --------
            float L[kH], Lx[kH];
            if (x.nb > 0) {
                const uint32_t Gp = G - 1;
                if (!mbar_wait(&sm.pv_done[Gp & 1], (Gp >> 1) & 1, abort, p.err)) break;
                tc_fence_after();
#pragma unroll
                for (int h = 0; h < kH; ++h) {
                    float v = l_part[h];
                    v += __shfl_xor_sync(0xffffffffu, v, 8);
                    v += __shfl_xor_sync(0xffffffffu, v, 4);
                    v += __shfl_xor_sync(0xffffffffu, v, 2);
                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                    float e = l_lse[h];
                    e += __shfl_xor_sync(0xffffffffu, e, 8);
                    e += __shfl_xor_sync(0xffffffffu, e, 4);
                    e += __shfl_xor_sync(0xffffffffu, e, 2);
                    e += __shfl_xor_sync(0xffffffffu, e, 1);
                    if (lane == 0) { sm.lred[quad][h] = v; sm.lred[4 + quad][h] = e; }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.epi_bar);
                if (!mbar_wait(&sm.epi_bar, epi_phase, abort, p.err)) break;
                epi_phase ^= 1;
#pragma unroll
                for (int h = 0; h < kH; ++h) {
                    L[h] = sm.lred[0][h] + sm.lred[1][h] + sm.lred[2][h] + sm.lred[3][h];
                    Lx[h] = sm.lred[4][h] + sm.lred[5][h] + sm.lred[6][h] + sm.lred[7][h];
                }
            } else {
#pragma unroll
                for (int h = 0; h < kH; ++h) { L[h] = 0.f; Lx[h] = 0.f; }
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                uint32_t o[16];
                if (x.nb > 0) {
                    tmem_ld16(tmem + lane_base + kOCol + 16 * m, o);
                    tmem_wait_ld();
                }
                const int dim = m * 128 + quad * 32 + lane;
#pragma unroll
                for (int h = 0; h < kH; ++h) {
                    const float v = (x.nb > 0 && L[h] > 0.f) ? __uint_as_float(o[h]) / L[h] : 0.f;
                    if (p.page_table == nullptr)
                        p.out[((long long)x.n * kH + h) * kDv + dim] = __float2bfloat16_rn(v);
                    else
                        p.o_part[(((long long)x.n * p.splits + x.sp) * kH + h) * kDv + dim] = v;
                }
            }
            if (quad == 0 && lane < kH) {
                float mr = m_ref[0], Lh = Lx[0];
#pragma unroll
                for (int h = 1; h < kH; ++h)
                    if (lane == h) { mr = m_ref[h]; Lh = Lx[h]; }
                const float l = Lh > 0.f ? (mr + log2f(Lh)) * 0.69314718055994531f : -INFINITY;
                if (p.page_table == nullptr) {
                    if (p.lse != nullptr) p.lse[(long long)x.n * kH + lane] = l;
                } else {
                    p.lse_part[((long long)x.n * p.splits + x.sp) * kH + lane] = l;
                }
            }
            if (x.nb > 0) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.o_free);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.q_empty[qb]);  // done with this unit's indices
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Merge of decode splits: lse = log sum_i exp(lse_i); out = sum_i exp(lse_i - lse) o_i.
__global__ void mla_combine_kernel(const float* __restrict__ o_part,
                                   const float* __restrict__ lse_part, int splits,
                                   __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
    const int n = blockIdx.x;
    const int h = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const float* lp = lse_part + (long long)n * splits * kH;
    float mx = -INFINITY;
    for (int i = 0; i < splits; ++i) mx = fmaxf(mx, lp[i * kH + h]);
    float denom = 0.f;
    for (int i = 0; i < splits; ++i) {
        const float l = lp[i * kH + h];
        denom += l == -INFINITY ? 0.f : expf(l - mx);
    }
    float acc[kDv / 32];
#pragma unroll
    for (int d = 0; d < kDv / 32; ++d) acc[d] = 0.f;
    for (int i = 0; i < splits; ++i) {
        const float l = lp[i * kH + h];
        if (l == -INFINITY) continue;
        const float wgt = expf(l - mx) / denom;
        const float* op = o_part + (((long long)n * splits + i) * kH + h) * kDv;
#pragma unroll
        for (int d = 0; d < kDv / 32; ++d) acc[d] = fmaf(wgt, op[d * 32 + lane], acc[d]);
    }
    __nv_bfloat16* ob = out + ((long long)n * kH + h) * kDv;
#pragma unroll
    for (int d = 0; d < kDv / 32; ++d) ob[d * 32 + lane] = __float2bfloat16_rn(acc[d]);
    if (lse != nullptr && lane == 0)
        lse[(long long)n * kH + h] = denom > 0.f ? mx + logf(denom) : -INFINITY;
}

}  // namespace

int mla_decode_splits(int num_q, int k_sel, int num_sms) {
    const int blocks = (k_sel + kBK - 1) / kBK;
    int splits = (4 * num_sms + num_q - 1) / (num_q > 0 ? num_q : 1);
    if (splits < 1) splits = 1;
    if (splits > blocks) splits = blocks;
    const int chunk = ((k_sel + splits - 1) / splits + kBK - 1) / kBK * kBK;
    return (k_sel + chunk - 1) / chunk;
}

size_t mla_smem_bytes() { return sizeof(MlaSmem) + 1024; }

cudaError_t launch_sparse_mla_bf16(const __nv_bfloat16* q, const __nv_bfloat16* kv,
                                   long long kv_rows, const int* page_table, int max_pages,
                                   int page_size, const int* seq_lens, const int* idx,
                                   int k_sel, long long ld_idx, int num_q, float scale,
                                   int splits, __nv_bfloat16* out, float* lse, float* o_part,
                                   float* lse_part, cudaStream_t stream, const DevCtx& ctx) {
    CUtensorMap tq;
    if (!make_tmap_bf16_2d(&tq, q, (uint64_t)num_q * kH, kDqk, kDqk * 2, kH, 64))
        return cudaErrorInvalidValue;
    MlaParams p{};
    p.kv = kv;
    p.kv_rows = kv_rows;
    p.page_table = page_table;
    p.max_pages = max_pages;
    p.page_size = page_size > 0 ? page_size : 1;
    p.num_pages = page_table ? (int)(kv_rows / p.page_size) : 0;
    p.seq_lens = seq_lens;
    p.idx = idx;
    p.k_sel = k_sel;
    p.ld_idx = ld_idx;
    p.num_q = num_q;
    p.splits = page_table ? splits : 1;
    p.chunk = page_table ? ((k_sel + splits - 1) / splits + kBK - 1) / kBK * kBK : k_sel;
    p.num_units = num_q * p.splits;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.out = out;
    p.lse = lse;
    p.o_part = o_part;
    p.lse_part = lse_part;
    p.err = ctx.err;
    const size_t smem = mla_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(sparse_mla_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = p.num_units < ctx.num_sms ? p.num_units : ctx.num_sms;
    sparse_mla_tc_kernel<<<grid, kThreads, smem, stream>>>(tq, p);
    count_launch(DSA_KERNEL_ATTENTION);
    return cudaGetLastError();
}

cudaError_t launch_mla_combine(const float* o_part, const float* lse_part, int num_q, int splits,
                               __nv_bfloat16* out, float* lse, cudaStream_t stream) {
    mla_combine_kernel<<<num_q, kH * 32, 0, stream>>>(o_part, lse_part, splits, out, lse);
    count_launch(DSA_KERNEL_COMBINE);
    return cudaGetLastError();
}

}  // namespace dsa
