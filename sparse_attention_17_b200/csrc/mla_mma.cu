// mla_mma.cu -- sparse absorbed-MLA attention (prefill and paged decode) on warp-level
// tensor-core MMAs (mma.sync m16n8k16, bf16 in, fp32 accumulate), with the selected
// latent rows gathered by TMA bulk copies.
//
// For query n and head h (16 heads), over the selected keys I_n only:
//   logit_s  = scale * q[n,h,0:576] . C[s,0:576]          C = 576-dim latent row
//   out[n,h] = sum_s softmax(logit)_s * C[s,0:512]          value = first 512 latent dims
// (DSV2-Lite-IndexCache card: attention_mode="sparse" over the selected routes;
//  DeepSeek-V2-Lite-Chat SIQ card: MLA with kv_lora_rank 512 and 576 elements per token.)
//
// Why warp MMAs here.  With 16 heads every product has a 16-wide side.  On this B200 a
// tcgen05.mma with N <= 64 costs ~49 cycles per instruction whatever M is, so the 16-head
// products would be bound by UMMA issue, while m16n8k16 warp MMAs reach ~1,030 MAC/clk per
// SM.  The gather of the selected 1152-byte rows (about 2 KB of latent data per query and
// key block of 64 FLOP/B) is then the bound, as it should be for this operation.
//
// Why this shape (measured).  With one CTA per SM, every phase of a block (gather, QK,
// cross-warp exchanges, softmax, PV) ran back to back and the kernel reached ~5.3 TB/s of
// gathered rows whatever the split of the work.  Here two independent CTAs share each SM,
// so one CTA's exchanges and softmax overlap the other's MMAs, and the rows are fetched by
// TMA bulk copies, which take no load/store-unit issue slots from the compute warps.
//
// Per CTA (two per SM, persistent; one query -- or one split of a decode sequence -- per
// unit), 192 threads:
//   warps 4, 5   gather: each lane of 16 issues one 1152-byte bulk copy (TMA) of its
//                selected row into a 32-row stage (rows padded to 1168 B so that ldmatrix
//                reads are bank-conflict free) and records whether the row is valid;
//                completion is tracked by the stage's mbarrier transaction count.  Rows of
//                invalid or padding entries are not fetched: they keep finite stale data
//                and get probability exactly 0.  Warp 4 lane 0 also bulk-copies each
//                unit's 16x576 query.  Selected indices are read from global memory one
//                block ahead.
//   warps 0..3   compute.  QK: warp w takes K-quarter w (9 of the 36 K-steps) for all 32
//                keys of the block; its quarter of Q stays in registers for the whole
//                unit.  Partial scores are exchanged through shared memory so that warp w
//                sums the four quarters for keys 8w..8w+7, runs the online softmax on them
//                (exact running max shared through shared memory) and writes P in bf16.
//                PV: warp w owns 128 of the 512 output dims (O stays in registers).
// Two stages per CTA keep the next block's gather in flight while a block is computed.
//
// fp8 latent cache (DeepSeek-V2-Lite-Chat SIQ card: fp8 KV at 576 bytes per token).  The
// same kernel, instantiated with kFp8, reads E4M3 codes (one byte per latent element,
// value = kv_scale * code) and gathers 576-byte rows, so the shared-memory traffic per key
// -- the bound of the bf16 kernel -- halves.  The codes are widened to f16 in registers
// (cvt e4m3x2 -> f16x2 is exact) right after ldmatrix, and both products run as f16 warp
// MMAs: the query is carried in f16 (exact for bf16 values of magnitude 2^-14 .. 65504)
// and P is rounded to f16 instead of bf16.  Two tricks keep the conversion cheap:
//   QK  the reduction over latent dims may run in any order, so an ldmatrix of fp8 rows
//       (lane: 4 consecutive bytes of one key) feeds one m16n8k16 directly; the query
//       fragments use the same order of dims (k = 2t,2t+1 <-> dims 4t,4t+1 and
//       k = 2t+8,2t+9 <-> dims 4t+2,4t+3 of each 16-dim chunk).
//   PV  ldmatrix.trans of fp8 rows gives each lane the byte pairs of two keys; one byte
//       permute splits them into (key 2t, key 2t+1) pairs for an even and an odd dim, so
//       one 8x8 load feeds two n-tiles, whose output dims interleave (handled at the store).
// Four stages per CTA (the fp8 rows take half the space) keep more copies in flight.
// Decode splits a sequence's selected keys over several units; their normalised partials
// and log-sum-exps are merged by mla_combine_kernel.
#include <cuda_fp16.h>

#include "dsa_common.cuh"
#include "launch.h"

namespace dsa {

namespace {

constexpr int kH = 16;
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kComputeWarps = 4;
constexpr int kBK = 32;                        // keys per block / stage
constexpr int kCtasPerSm = 2;
constexpr int kNT = kBK / 8;                   // 8-key n-tiles per block (one per compute warp)
constexpr int kGatherWarps = kBK / 16;         // each gather warp copies 16 rows per stage
constexpr int kGatherWarp0 = kComputeWarps;
constexpr int kThreads = 32 * (kComputeWarps + kGatherWarps);
constexpr int kQPitch = 1168;                  // bytes per query head row
constexpr int kQBytes = kH * kQPitch;          // 18688
constexpr int kPPitch = kBK * 2 + 16;          // bytes per P row (bf16 keys + 16)
constexpr int kPBytes = kH * kPPitch;
constexpr int kKSteps = kDqk / 16;             // 36
constexpr int kKQuarter = kKSteps / kComputeWarps;  // K-steps of the QK product per warp
constexpr int kDvWarp = kDv / kComputeWarps;   // output dims per compute warp
constexpr int kPVTiles = kDvWarp / 8;          // 8-dim n-tiles per compute warp
static_assert(kNT == kComputeWarps, "each compute warp runs the softmax of one n-tile");
static_assert(kKSteps % kComputeWarps == 0, "the K-steps split evenly over the warps");
static_assert(kDvWarp % 32 == 0, "PV loads two n-tiles (bf16) or two 16-dim chunks (fp8) at a time");

// Layout of the staged cache rows: bf16 (1152 B) or E4M3 codes (576 B) per row, padded by
// 16 B so that the 8 rows of an ldmatrix phase hit distinct bank groups (pitch / 16 odd).
template <bool kFp8>
struct RowLayout {
    static constexpr int kRowBytes = kFp8 ? kDqk : kDqk * 2;
    static constexpr int kRowPitch = kRowBytes + 16;
    static constexpr int kStages = kFp8 ? 4 : 2;
    static constexpr int kStageBytes = kBK * kRowPitch;
    static_assert((kRowPitch / 16) % 2 == 1, "row pitch must be an odd number of 16-byte units");
    static_assert((kStages & (kStages - 1)) == 0, "stage count must be a power of two");
};

template <bool kFp8>
struct MmaSmem {
    using L = RowLayout<kFp8>;
    alignas(128) uint8_t stage[L::kStages][L::kStageBytes];
    alignas(128) uint8_t q[kQBytes];
    alignas(128) uint8_t p[L::kStages][kPBytes];
    alignas(16) int valid[L::kStages][kBK];  // 1: the staged row holds the key; -1: not fetched
    alignas(16) float spart[kComputeWarps][kNT][32][4];  // [from warp][n-tile] partial scores
    alignas(16) float red[L::kStages][kH][kComputeWarps];  // per head, per warp block maxima
    alignas(16) float lsum[2][kComputeWarps][kH];         // per warp row sums at the end of a unit
    uint64_t a_full[L::kStages], a_free[L::kStages];
    uint64_t q_full, q_empty;
    int abort;
};

// two CTAs per SM: each may use at most half of the SM's 228 KB less 1 KB per CTA
static_assert(sizeof(MmaSmem<false>) + 128 <= 113 * 1024, "bf16 CTA too large for two per SM");
static_assert(sizeof(MmaSmem<true>) + 128 <= 113 * 1024, "fp8 CTA too large for two per SM");

struct Params {
    const __nv_bfloat16* q;
    const uint8_t* kv;       // cache rows: bf16 [.., 576] or E4M3 codes [.., 576]
    long long kv_rows;
    const int* page_table;  // NULL = prefill
    int max_pages, page_size, num_pages;
    const int* seq_lens;
    const int* idx;
    int k_sel;
    long long ld_idx;
    int splits, chunk, num_units;
    float scale_log2;        // softmax scale (times kv_scale for fp8) in log2 units
    float out_scale;         // 1 (bf16) or kv_scale (fp8): multiplies the normalised output
    __nv_bfloat16* out;
    float* lse;
    float* o_part;
    float* lse_part;
    unsigned* err;
};

struct Unit {
    int n, sp, e0, e1, nb, len;
};

__device__ __forceinline__ Unit unit_of(const Params& p, int u) {
    Unit x;
    if (p.page_table == nullptr) {
        x.n = u; x.sp = 0; x.e0 = 0; x.e1 = p.k_sel; x.len = 0;
    } else {
        x.n = u / p.splits;
        x.sp = u % p.splits;
        x.e0 = x.sp * p.chunk;
        x.e1 = min(p.k_sel, x.e0 + p.chunk);
        x.len = min(__ldg(p.seq_lens + x.n), p.max_pages * p.page_size);
    }
    x.nb = x.e1 > x.e0 ? (x.e1 - x.e0 + kBK - 1) / kBK : 0;
    return x;
}

// Selected key of index entry e (-1 past the unit's entries).
__device__ __forceinline__ int load_index(const Params& p, const Unit& x, int e) {
    return e < x.e1 ? __ldg(p.idx + (long long)x.n * p.ld_idx + e) : -1;
}

// Cache row of selected key s (-1: padding or invalid; invalid keys are reported).
__device__ __forceinline__ long long resolve_row(const Params& p, const Unit& x, int s) {
    if (s < 0) return -1;
    if (p.page_table == nullptr) {
        if (s >= p.kv_rows) {
            atomicOr(p.err, DSA_DEVERR_INDEX_RANGE);
            return -1;
        }
        return s;
    }
    if (s >= x.len) {
        atomicOr(p.err, DSA_DEVERR_INDEX_RANGE);
        return -1;
    }
    const int pg = __ldg(p.page_table + (long long)x.n * p.max_pages + s / p.page_size);
    if (pg < 0 || pg >= p.num_pages) {
        atomicOr(p.err, DSA_DEVERR_PAGE_RANGE);
        return -1;
    }
    return (long long)pg * p.page_size + s % p.page_size;
}

// ---- warp MMA helpers (PTX ISA: ldmatrix, mma.sync m16n8k16 bf16) ----
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// The same with f16 operands (the fp8 cache path).
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                        uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Two E4M3 codes (bytes 0,1 or bytes 2,3 of v) -> f16x2 (low byte -> low half); exact.
// One cvt on a half of the register, with no repacking of the result.
__device__ __forceinline__ uint32_t e4m3x2_lo_to_f16x2(uint32_t v) {
    uint32_t r;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, lo;\n\t}"
        : "=r"(r) : "r"(v));
    return r;
}
__device__ __forceinline__ uint32_t e4m3x2_hi_to_f16x2(uint32_t v) {
    uint32_t r;
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, hi;\n\t}"
        : "=r"(r) : "r"(v));
    return r;
}
// bf16x2 -> f16x2 (round to nearest; exact for magnitudes 2^-14 .. 65504).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
    const __half2 h = __floats2half2_rn(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
    return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
// Barrier among the compute warps only (hardware named barrier 1).
__device__ __forceinline__ void compute_sync() { named_bar_sync(1, 32 * kComputeWarps); }

// Waits with a time limit; on a timeout it records the error and lets the caller carry on
// along the same control flow (results are then garbage but every barrier still matches).
__device__ __forceinline__ void wait_soft(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          unsigned* err) {
    (void)mbar_wait(bar, parity, abort, err);
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
sparse_mla_mma_kernel(const Params p) {
    using L = RowLayout<kFp8>;
    constexpr int kStages = L::kStages;
    constexpr int kRowPitch = L::kRowPitch;
    constexpr int kRowBytes = L::kRowBytes;
    extern __shared__ uint8_t smem_raw[];
    MmaSmem<kFp8>& sm =
        *reinterpret_cast<MmaSmem<kFp8>*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int* abort = &sm.abort;
    chained_launch_gate();

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            // one expect-tx arrival per gather warp (after it has written the stage's valid
            // flags); the phase completes when every issued row copy has landed
            mbar_init(&sm.a_full[i], kGatherWarps);
            mbar_init(&sm.a_free[i], kComputeWarps);
        }
        mbar_init(&sm.q_full, 1);
        mbar_init(&sm.q_empty, kComputeWarps);
        sm.abort = 0;
        fence_barrier_init();
    }
    // zero the stages once, so that rows never fetched hold finite values; the padding
    // columns are never read
    for (int i = threadIdx.x; i < (int)(sizeof(sm.stage) / 16); i += kThreads)
        reinterpret_cast<uint4*>(sm.stage)[i] = make_uint4(0, 0, 0, 0);
    __syncthreads();

    if (warp >= kGatherWarp0) {
        // ================================ gather ================================
        const int gw = warp - kGatherWarp0;
        const bool leader = gw == 0 && lane == 0;
        uint32_t G = 0;
        int units = 0;
        for (int ui = 0;; ++ui, ++units) {
            const int u = blockIdx.x + ui * gridDim.x;
            if (u >= p.num_units) break;
            const Unit x = unit_of(p, u);
            if (leader) {
                // the query of this unit, once the compute warps hold the previous one in
                // registers
                wait_soft(&sm.q_empty, (ui & 1) ^ 1, abort, p.err);
                mbar_arrive_expect_tx(&sm.q_full, kH * kDqk * 2);
                for (int h = 0; h < kH; ++h)
                    bulk_load(sm.q + h * kQPitch, p.q + ((long long)x.n * kH + h) * kDqk, kDqk * 2,
                              &sm.q_full);
            }
            // This lane's selected keys are read two blocks ahead of their copies and
            // resolved to cache rows (a page-table load in decode) one block ahead.
            const int e_lane = x.e0 + gw * 16 + lane;
            int s_ahead = lane < 16 ? load_index(p, x, e_lane + kBK) : -1;
            long long row_next = lane < 16 ? resolve_row(p, x, load_index(p, x, e_lane)) : -1;
            for (int j = 0; j < x.nb; ++j, ++G) {
                const int s = G % kStages;
                const long long row = row_next;
                if (lane < 16) {
                    const int s_far = load_index(p, x, e_lane + (j + 2) * kBK);
                    row_next = resolve_row(p, x, s_ahead);
                    s_ahead = s_far;
                }
                wait_soft(&sm.a_free[s], ((G / kStages) & 1) ^ 1, abort, p.err);
                if (lane < 16) sm.valid[s][gw * 16 + lane] = row >= 0 ? 1 : -1;
                const unsigned vmask = __ballot_sync(0xffffffffu, row >= 0);
                __syncwarp();
                if (lane == 0)
                    mbar_arrive_expect_tx(&sm.a_full[s], (uint32_t)__popc(vmask) * kRowBytes);
                __syncwarp();
                if (row >= 0)
                    bulk_load(sm.stage[s] + (gw * 16 + lane) * kRowPitch, p.kv + row * kRowBytes,
                              kRowBytes, &sm.a_full[s]);
            }
        }
        // The compute warps consume every block and query, but after a timed-out wait they
        // may not have: let the last copies land (time-bounded, whatever the abort flag
        // says) before the CTA can exit.
        volatile int keep_waiting = 0;
        for (uint32_t Gl = G >= kStages ? G - kStages : 0; Gl < G; ++Gl)
            (void)mbar_wait(&sm.a_full[Gl % kStages], (Gl / kStages) & 1, &keep_waiting, p.err);
        if (leader && units > 0) (void)mbar_wait(&sm.q_full, (units - 1) & 1, &keep_waiting, p.err);
    } else {
        // ================================ compute ===============================
        // warp w: K-quarter w of the QK product over all kBK keys, then the softmax of keys
        // 8w..8w+7 (n-tile w) and PV for output dims kDvWarp*w ..
        const int g = lane >> 2;    // fragment row group
        const int t = lane & 3;     // thread in group
        uint32_t G = 0;
        for (int ui = 0;; ++ui) {
            const int u = blockIdx.x + ui * gridDim.x;
            if (u >= p.num_units) break;
            const Unit x = unit_of(p, u);
            wait_soft(&sm.q_full, ui & 1, abort, p.err);
            uint32_t qa[kKQuarter][4];
            if constexpr (!kFp8) {
                const int head = (lane & 7) + ((lane >> 3) & 1) * 8;
                const uint32_t qrow = smem_u32(sm.q) + head * kQPitch + ((lane >> 4) & 1) * 16;
#pragma unroll
                for (int ks = 0; ks < kKQuarter; ++ks)
                    ldsm_x4(qrow + (warp * kKQuarter + ks) * 32, qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
            } else {
                // f16 fragments in the permuted order of dims of the fp8 QK (see the top)
#pragma unroll
                for (int ks = 0; ks < kKQuarter; ++ks) {
                    const int d0 = (warp * kKQuarter + ks) * 16 + 4 * t;
                    const uint2 lo = *reinterpret_cast<const uint2*>(sm.q + g * kQPitch + d0 * 2);
                    const uint2 hi = *reinterpret_cast<const uint2*>(sm.q + (g + 8) * kQPitch + d0 * 2);
                    qa[ks][0] = bf16x2_to_f16x2(lo.x);
                    qa[ks][1] = bf16x2_to_f16x2(hi.x);
                    qa[ks][2] = bf16x2_to_f16x2(lo.y);
                    qa[ks][3] = bf16x2_to_f16x2(hi.y);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.q_empty);
            float o[kPVTiles][4];
#pragma unroll
            for (int i = 0; i < kPVTiles; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
            float m_run[2] = {-INFINITY, -INFINITY};  // heads g, g+8 (log2 domain)
            float l_run[2] = {0.f, 0.f};              // this thread's partial row sums
            float l_lse[2] = {0.f, 0.f};              // the same before bf16 rounding

            for (int j = 0; j < x.nb; ++j, ++G) {
                const int s = G % kStages;
                wait_soft(&sm.a_full[s], (G / kStages) & 1, abort, p.err);
                const uint32_t st = smem_u32(sm.stage[s]);
                // ---- QK: S[16 heads x kBK keys] over this warp's K-quarter ----
                float acc[kNT][4];
#pragma unroll
                for (int i = 0; i < kNT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
                if constexpr (!kFp8) {
                    const int key = (lane & 7) + ((lane >> 4) & 1) * 8;
                    const uint32_t krow = st + key * kRowPitch + ((lane >> 3) & 1) * 16 + warp * kKQuarter * 32;
#pragma unroll
                    for (int ks = 0; ks < kKQuarter; ++ks) {
#pragma unroll
                        for (int n2 = 0; n2 < kNT / 2; ++n2) {
                            uint32_t b0, b1, b2, b3;
                            ldsm_x4(krow + n2 * 16 * kRowPitch + ks * 32, b0, b1, b2, b3);
                            mma_bf16(acc[2 * n2], qa[ks], b0, b1);
                            mma_bf16(acc[2 * n2 + 1], qa[ks], b2, b3);
                        }
                    }
                } else {
                    // one x4 load = the 16 code bytes of this K-step for all 32 keys; matrix
                    // j (lanes 8j..8j+7 address keys 8j..8j+7) is n-tile j
                    const uint32_t krow = st + lane * kRowPitch + warp * kKQuarter * 16;
#pragma unroll
                    for (int ks = 0; ks < kKQuarter; ++ks) {
                        uint32_t r[4];
                        ldsm_x4(krow + ks * 16, r[0], r[1], r[2], r[3]);
#pragma unroll
                        for (int nt = 0; nt < kNT; ++nt)
                            mma_f16(acc[nt], qa[ks], e4m3x2_lo_to_f16x2(r[nt]), e4m3x2_hi_to_f16x2(r[nt]));
                    }
                }
                // partial sums of the other warps' n-tiles go through shared memory
#pragma unroll
                for (int nt = 0; nt < kNT; ++nt)
                    if (nt != warp)
                        *reinterpret_cast<float4*>(sm.spart[warp][nt][lane]) =
                            make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
                compute_sync();
                float sc[4];
                {
                    float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int nt = 0; nt < kNT; ++nt)
                        if (nt == warp) { a4[0] = acc[nt][0]; a4[1] = acc[nt][1]; a4[2] = acc[nt][2]; a4[3] = acc[nt][3]; }
#pragma unroll
                    for (int w2 = 0; w2 < kComputeWarps; ++w2) {
                        if (w2 == warp) continue;
                        const float4 v = *reinterpret_cast<const float4*>(sm.spart[w2][warp][lane]);
                        a4[0] += v.x; a4[1] += v.y; a4[2] += v.z; a4[3] += v.w;
                    }
                    // fragment i: head g + 8*(i>>1), key 8*warp + 2t + (i&1)
                    const int2 vr = *reinterpret_cast<const int2*>(&sm.valid[s][warp * 8 + 2 * t]);
                    sc[0] = vr.x >= 0 ? a4[0] * p.scale_log2 : -INFINITY;
                    sc[1] = vr.y >= 0 ? a4[1] * p.scale_log2 : -INFINITY;
                    sc[2] = vr.x >= 0 ? a4[2] * p.scale_log2 : -INFINITY;
                    sc[3] = vr.y >= 0 ? a4[3] * p.scale_log2 : -INFINITY;
                }
                float mx0 = fmaxf(sc[0], sc[1]), mx1 = fmaxf(sc[2], sc[3]);
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
                if (t == 0) {
                    sm.red[s][g][warp] = mx0;
                    sm.red[s][g + 8][warp] = mx1;
                }
                compute_sync();
                float ref[2], alpha[2];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    static_assert(kComputeWarps == 4, "one 16-byte load of the warps' maxima");
                    const float4 wm = *reinterpret_cast<const float4*>(sm.red[s][g + 8 * r]);
                    const float bm = fmaxf(fmaxf(wm.x, wm.y), fmaxf(wm.z, wm.w));
                    const float mn = fmaxf(m_run[r], bm);
                    alpha[r] = m_run[r] == -INFINITY ? 0.f : exp2f(m_run[r] - mn);
                    m_run[r] = mn;
                    ref[r] = mn == -INFINITY ? 0.f : mn;  // no valid key yet: P = 0 anyway
                    l_run[r] *= alpha[r];
                    l_lse[r] *= alpha[r];
                }
                // P = exp2(s - m) in bf16; invalid keys (s = -inf) give exactly 0
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const float p0 = exp2f(sc[2 * r] - ref[r]);
                    const float p1 = exp2f(sc[2 * r + 1] - ref[r]);
                    uint32_t pk;
                    if constexpr (!kFp8) {
                        pk = pack_bf16(p0, p1);
                        const __nv_bfloat162 pr = *reinterpret_cast<const __nv_bfloat162*>(&pk);
                        l_run[r] += __bfloat162float(pr.x) + __bfloat162float(pr.y);
                    } else {
                        pk = pack_f16(p0, p1);
                        const __half2 pr = *reinterpret_cast<const __half2*>(&pk);
                        l_run[r] += __low2float(pr) + __high2float(pr);
                    }
                    l_lse[r] += p0 + p1;
                    *reinterpret_cast<uint32_t*>(sm.p[s] + (g + 8 * r) * kPPitch + (warp * 8 + 2 * t) * 2) = pk;
                }
#pragma unroll
                for (int n = 0; n < kPVTiles; ++n) {
                    o[n][0] *= alpha[0]; o[n][1] *= alpha[0];
                    o[n][2] *= alpha[1]; o[n][3] *= alpha[1];
                }
                compute_sync();  // P of this block is in shared memory
                // ---- PV: O[16 heads x kDvWarp dims of this warp] += P[16 x kBK keys] V ----
                {
                    const int head = (lane & 7) + ((lane >> 3) & 1) * 8;
                    const uint32_t prow = smem_u32(sm.p[s]) + head * kPPitch + ((lane >> 4) & 1) * 16;
                    const int vkey = (lane & 7) + ((lane >> 3) & 1) * 8;
                    if constexpr (!kFp8) {
                        const uint32_t vrow = st + vkey * kRowPitch + (warp * kDvWarp + ((lane >> 4) & 1) * 8) * 2;
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk) {
                            uint32_t pa[4];
                            ldsm_x4(prow + kk * 32, pa[0], pa[1], pa[2], pa[3]);
#pragma unroll
                            for (int n2 = 0; n2 < kPVTiles / 2; ++n2) {
                                uint32_t b0, b1, b2, b3;
                                ldsm_x4_t(vrow + kk * 16 * kRowPitch + n2 * 32, b0, b1, b2, b3);
                                mma_bf16(o[2 * n2], pa, b0, b1);
                                mma_bf16(o[2 * n2 + 1], pa, b2, b3);
                            }
                        }
                    } else {
                        // x4.trans: matrices (keys 0-7 | 8-15) x (chunk c | c+1) of 16 dims;
                        // lane (g,t) gets bytes [V(2t,2g) V(2t,2g+1) V(2t+1,2g) V(2t+1,2g+1)]
                        // of its chunk; the byte permute 3120 pairs them per dim.  n-tile
                        // 4*c2 + 2*(c&1) holds the even dims of chunk c, the next tile the
                        // odd dims.
                        const uint32_t vrow = st + vkey * kRowPitch + warp * kDvWarp + ((lane >> 4) & 1) * 16;
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk) {
                            uint32_t pa[4];
                            ldsm_x4(prow + kk * 32, pa[0], pa[1], pa[2], pa[3]);
#pragma unroll
                            for (int c2 = 0; c2 < kPVTiles / 4; ++c2) {
                                uint32_t r[4];
                                ldsm_x4_t(vrow + kk * 16 * kRowPitch + c2 * 32, r[0], r[1], r[2], r[3]);
#pragma unroll
                                for (int h = 0; h < 2; ++h) {
                                    const uint32_t x0 = __byte_perm(r[2 * h], 0u, 0x3120);
                                    const uint32_t x1 = __byte_perm(r[2 * h + 1], 0u, 0x3120);
                                    mma_f16(o[4 * c2 + 2 * h], pa, e4m3x2_lo_to_f16x2(x0), e4m3x2_lo_to_f16x2(x1));
                                    mma_f16(o[4 * c2 + 2 * h + 1], pa, e4m3x2_hi_to_f16x2(x0), e4m3x2_hi_to_f16x2(x1));
                                }
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.a_free[s]);  // stage and P buffer reusable
            }

            // ---- epilogue of the unit: row sums, normalise, write ----
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
                l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
                l_lse[r] += __shfl_xor_sync(0xffffffffu, l_lse[r], 1);
                l_lse[r] += __shfl_xor_sync(0xffffffffu, l_lse[r], 2);
            }
            if (t == 0) {
                sm.lsum[0][warp][g] = l_run[0];
                sm.lsum[0][warp][g + 8] = l_run[1];
                sm.lsum[1][warp][g] = l_lse[0];
                sm.lsum[1][warp][g + 8] = l_lse[1];
            }
            compute_sync();
            float L[2] = {0.f, 0.f}, Lx[2] = {0.f, 0.f};
#pragma unroll
            for (int i = 0; i < kComputeWarps; ++i) {
                L[0] += sm.lsum[0][i][g];
                L[1] += sm.lsum[0][i][g + 8];
                Lx[0] += sm.lsum[1][i][g];
                Lx[1] += sm.lsum[1][i][g + 8];
            }
            const float inv0 = (x.nb > 0 && L[0] > 0.f) ? p.out_scale / L[0] : 0.f;
            const float inv1 = (x.nb > 0 && L[1] > 0.f) ? p.out_scale / L[1] : 0.f;
            if constexpr (kFp8) {
                // chunk c of this warp: dims 16c + 4t + {0,1,2,3} are (even tile, odd tile)
                // x (column 0, column 1) -- see the PV comment
#pragma unroll
                for (int c = 0; c < kPVTiles / 2; ++c) {
                    const int te = 4 * (c >> 1) + 2 * (c & 1);
                    const int dim = warp * kDvWarp + 16 * c + 4 * t;
                    const float v0[4] = {o[te][0] * inv0, o[te + 1][0] * inv0, o[te][1] * inv0, o[te + 1][1] * inv0};
                    const float v1[4] = {o[te][2] * inv1, o[te + 1][2] * inv1, o[te][3] * inv1, o[te + 1][3] * inv1};
                    if (p.page_table == nullptr) {
                        __nv_bfloat16* o0 = p.out + ((long long)x.n * kH + g) * kDv + dim;
                        __nv_bfloat16* o1 = p.out + ((long long)x.n * kH + g + 8) * kDv + dim;
                        *reinterpret_cast<uint2*>(o0) = make_uint2(pack_bf16(v0[0], v0[1]), pack_bf16(v0[2], v0[3]));
                        *reinterpret_cast<uint2*>(o1) = make_uint2(pack_bf16(v1[0], v1[1]), pack_bf16(v1[2], v1[3]));
                    } else {
                        float* o0 = p.o_part + (((long long)x.n * p.splits + x.sp) * kH + g) * kDv + dim;
                        float* o1 = p.o_part + (((long long)x.n * p.splits + x.sp) * kH + g + 8) * kDv + dim;
                        *reinterpret_cast<float4*>(o0) = make_float4(v0[0], v0[1], v0[2], v0[3]);
                        *reinterpret_cast<float4*>(o1) = make_float4(v1[0], v1[1], v1[2], v1[3]);
                    }
                }
            }
#pragma unroll
            for (int n = 0; n < (kFp8 ? 0 : kPVTiles); ++n) {
                const int dim = warp * kDvWarp + n * 8 + 2 * t;
                if (p.page_table == nullptr) {
                    __nv_bfloat16* o0 = p.out + ((long long)x.n * kH + g) * kDv + dim;
                    __nv_bfloat16* o1 = p.out + ((long long)x.n * kH + g + 8) * kDv + dim;
                    *reinterpret_cast<uint32_t*>(o0) = pack_bf16(o[n][0] * inv0, o[n][1] * inv0);
                    *reinterpret_cast<uint32_t*>(o1) = pack_bf16(o[n][2] * inv1, o[n][3] * inv1);
                } else {
                    float* o0 = p.o_part + (((long long)x.n * p.splits + x.sp) * kH + g) * kDv + dim;
                    float* o1 = p.o_part + (((long long)x.n * p.splits + x.sp) * kH + g + 8) * kDv + dim;
                    *reinterpret_cast<float2*>(o0) = make_float2(o[n][0] * inv0, o[n][1] * inv0);
                    *reinterpret_cast<float2*>(o1) = make_float2(o[n][2] * inv1, o[n][3] * inv1);
                }
            }
            if (warp == 0 && t == 0) {
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int head = g + 8 * r;
                    const float l = (x.nb > 0 && Lx[r] > 0.f) ? (m_run[r] + log2f(Lx[r])) * 0.69314718055994531f
                                                           : -INFINITY;
                    if (p.page_table == nullptr) {
                        if (p.lse != nullptr) p.lse[(long long)x.n * kH + head] = l;
                    } else {
                        p.lse_part[((long long)x.n * p.splits + x.sp) * kH + head] = l;
                    }
                }
            }
            compute_sync();  // lsum is rewritten by the next unit
        }
    }
}

// Merge of decode splits: lse = log sum_i exp(lse_i); out = sum_i exp(lse_i - lse) o_i.
// Grid (sequences, kCombineParts): each CTA merges one part of the output dims for all 16
// heads (a warp per head), so that a decode batch spreads over the SMs and every lane has
// kDv / 32 / kCombineParts independent loads per split in flight.
constexpr int kCombineParts = 4;
constexpr int kCombineDims = kDv / kCombineParts;
__global__ void __launch_bounds__(kH * 32)
mla_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                   int splits, __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
    chained_launch_gate();
    const int n = blockIdx.x;
    const int d0 = blockIdx.y * kCombineDims;
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
    float acc[kCombineDims / 32];
#pragma unroll
    for (int d = 0; d < kCombineDims / 32; ++d) acc[d] = 0.f;
#pragma unroll 4
    for (int i = 0; i < splits; ++i) {
        const float l = lp[i * kH + h];
        if (l == -INFINITY) continue;
        const float wgt = expf(l - mx) / denom;
        const float* op = o_part + (((long long)n * splits + i) * kH + h) * kDv + d0;
#pragma unroll
        for (int d = 0; d < kCombineDims / 32; ++d) acc[d] = fmaf(wgt, op[d * 32 + lane], acc[d]);
    }
    __nv_bfloat16* ob = out + ((long long)n * kH + h) * kDv + d0;
#pragma unroll
    for (int d = 0; d < kCombineDims / 32; ++d) ob[d * 32 + lane] = __float2bfloat16_rn(acc[d]);
    if (lse != nullptr && lane == 0 && blockIdx.y == 0)
        lse[(long long)n * kH + h] = denom > 0.f ? mx + logf(denom) : -INFINITY;
}

}  // namespace

// Splits per decode sequence: the count that minimises the modelled time, waves of units
// over the CTA slots times (key blocks per unit + a per-unit start-up cost of about four
// blocks: the query copy and the first gather round trip); ties go to fewer splits.
int mla_decode_splits(int num_q, int k_sel, int num_sms) {
    constexpr int kUnitStartBlocks = 4;
    const int blocks = (k_sel + kBK - 1) / kBK;
    const long long slots = (long long)kCtasPerSm * num_sms;
    const int nq = num_q > 0 ? num_q : 1;
    int best = 1;
    long long best_cost = -1;
    for (int sp = 1; sp <= blocks; ++sp) {
        const int per_unit = (blocks + sp - 1) / sp;
        const int splits = (blocks + per_unit - 1) / per_unit;  // no empty split
        if (splits != sp) continue;
        const long long waves = ((long long)nq * splits + slots - 1) / slots;
        const long long cost = waves * (per_unit + kUnitStartBlocks);
        if (best_cost < 0 || cost < best_cost) {
            best = splits;
            best_cost = cost;
        }
    }
    return best;
}

size_t mla_mma_smem_bytes(bool fp8) {
    return (fp8 ? sizeof(MmaSmem<true>) : sizeof(MmaSmem<false>)) + 128;
}

namespace {
template <bool kFp8>
cudaError_t launch_mla_kernel(const Params& p, cudaStream_t stream, const DevCtx& ctx) {
    const size_t smem = mla_mma_smem_bytes(kFp8);
    cudaError_t e = cudaFuncSetAttribute(sparse_mla_mma_kernel<kFp8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // two CTAs per SM need most of the shared memory carve-out
    e = cudaFuncSetAttribute(sparse_mla_mma_kernel<kFp8>,
                             cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    const int slots = kCtasPerSm * ctx.num_sms;
    const int grid = p.num_units < slots ? p.num_units : slots;
    e = launch_chained(sparse_mla_mma_kernel<kFp8>, dim3(grid), dim3(kThreads), smem, stream, 1, p);
    count_launch(DSA_KERNEL_ATTENTION);
    return e;
}
}  // namespace

cudaError_t launch_sparse_mla_mma(const __nv_bfloat16* q, const void* kv, bool kv_fp8,
                                  float kv_scale, long long kv_rows, const int* page_table,
                                  int max_pages, int page_size, const int* seq_lens,
                                  const int* idx, int k_sel, long long ld_idx, int num_q,
                                  float scale, int splits, __nv_bfloat16* out, float* lse,
                                  float* o_part, float* lse_part, cudaStream_t stream,
                                  const DevCtx& ctx) {
    Params p{};
    p.q = q;
    p.kv = static_cast<const uint8_t*>(kv);
    p.kv_rows = kv_rows;
    p.page_table = page_table;
    p.max_pages = max_pages;
    p.page_size = page_size > 0 ? page_size : 1;
    p.num_pages = page_table ? (int)(kv_rows / p.page_size) : 0;
    p.seq_lens = seq_lens;
    p.idx = idx;
    p.k_sel = k_sel;
    p.ld_idx = ld_idx;
    p.splits = page_table ? splits : 1;
    p.chunk = page_table ? ((k_sel + splits - 1) / splits + kBK - 1) / kBK * kBK : k_sel;
    p.num_units = num_q * p.splits;
    p.scale_log2 = scale * (kv_fp8 ? kv_scale : 1.f) * 1.4426950408889634f;
    p.out_scale = kv_fp8 ? kv_scale : 1.f;
    p.out = out;
    p.lse = lse;
    p.o_part = o_part;
    p.lse_part = lse_part;
    p.err = ctx.err;
    return kv_fp8 ? launch_mla_kernel<true>(p, stream, ctx) : launch_mla_kernel<false>(p, stream, ctx);
}

cudaError_t launch_mla_combine(const float* o_part, const float* lse_part, int num_q, int splits,
                               __nv_bfloat16* out, float* lse, cudaStream_t stream) {
    const cudaError_t e = launch_chained(mla_combine_kernel, dim3(num_q, kCombineParts),
                                         dim3(kH * 32), 0, stream, 1, o_part, lse_part, splits,
                                         out, lse);
    count_launch(DSA_KERNEL_COMBINE);
    return e;
}

}  // namespace dsa
