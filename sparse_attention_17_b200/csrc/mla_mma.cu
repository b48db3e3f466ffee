// mla_mma.cu -- sparse absorbed-MLA attention (prefill and paged decode) on warp-level
// tensor-core MMAs (mma.sync m16n8k16, bf16 in, fp32 accumulate).
//
// For query n and head h (16 heads), over the selected keys I_n only:
//   logit_s  = scale * q[n,h,0:576] . C[s,0:576]          C = 576-dim latent row
//   out[n,h] = sum_s softmax(logit)_s * C[s,0:512]          value = first 512 latent dims
// (DSV2-Lite-IndexCache card: attention_mode="sparse" over the selected routes;
//  DeepSeek-V2-Lite-Chat SIQ card: MLA with kv_lora_rank 512 and 576 elements per token.)
//
// Why warp MMAs here.  With 16 heads every product has a 16-wide side.  On this B200 a
// tcgen05.mma with N <= 64 costs ~49 cycles per instruction whatever M is, so the 16-head
// products (52 UMMAs per 64 keys) would be bound at ~40 cycles per key by instruction
// issue, while m16n8k16 warp MMAs reach ~1,030 MAC/clk per SM -- about 17 cycles per key
// for the same work.  The gather of the selected 1152-byte latent rows (cp.async, ~32
// bytes/clk per SM from L2) is then the bound, as it should be for this operation.
//
// Per CTA (persistent; one query -- or one split of a decode sequence -- per unit):
//   warps 8..11  gather: 16-byte cp.async copies of each selected row into a 64-row stage
//                (rows padded to 1168 B so that ldmatrix reads are bank-conflict free);
//                invalid / padding rows are zero-filled; completion on an mbarrier.
//                Warp 8 lane 0 also bulk-copies the next unit's query and indices.
//   warps 0..7   compute.  QK: warp w takes keys 16*(w%4)..+15 and K-half w/4 (18 of the
//                36 K-steps); its half of Q stays in registers for the whole unit.  The
//                two K-halves are summed through shared memory, the K-half-0 warps run
//                the online softmax (exact running max, rescale of O in registers) and
//                write P in bf16; then every warp computes PV for its 64 output dims
//                (O stays in registers) and releases the stage.
// Two stages keep the next block's gather in flight while a block is computed.  Decode
// splits a sequence's selected keys over several units; their normalised partials and
// log-sum-exps are merged by mla_combine_kernel.
#include "dsa_common.cuh"
#include "launch.h"

namespace dsa {

namespace {

constexpr int kH = 16;
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kBK = 64;                        // keys per block / stage
constexpr int kRowPitch = 1168;                // bytes per staged key row (1152 + 16)
constexpr int kStageBytes = kBK * kRowPitch;   // 74752
constexpr int kQPitch = 1168;                  // bytes per query head row
constexpr int kQBytes = kH * kQPitch;          // 18688
constexpr int kPPitch = 144;                   // bytes per P row (64 keys bf16 + 16)
constexpr int kPBytes = kH * kPPitch;          // 2304
constexpr int kIdxCap = 2048;
constexpr int kComputeWarps = 8;
constexpr int kGatherWarp0 = 8;
constexpr int kGatherWarps = 4;
constexpr int kThreads = 32 * (kComputeWarps + kGatherWarps);  // 384
constexpr int kKSteps = kDqk / 16;             // 36
constexpr int kKHalf = kKSteps / 2;            // 18

struct MmaSmem {
    alignas(128) uint8_t stage[2][kStageBytes];
    alignas(128) uint8_t q[2][kQBytes];
    alignas(128) uint8_t p[2][kPBytes];
    alignas(16) int idx[2][kIdxCap];
    alignas(16) float spart[4][32][8];   // K-half-1 partial scores, per key group
    alignas(16) float red[4][kH];        // per key group, per head block maxima
    alignas(16) float alpha[kH];         // per head rescale factor of the current block
    alignas(16) float lsum[4][kH];       // per key group row sums at the end of a unit
    uint64_t a_full[2], a_free[2];
    uint64_t q_full[2], q_empty[2];
    int abort;
};

struct Params {
    const __nv_bfloat16* q;
    const __nv_bfloat16* kv;
    long long kv_rows;
    const int* page_table;  // NULL = prefill
    int max_pages, page_size, num_pages;
    const int* seq_lens;
    const int* idx;
    int k_sel;
    long long ld_idx;
    int splits, chunk, num_units;
    float scale_log2;
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

// Cache row of index entry e (-1: padding or invalid; invalid entries are reported).
__device__ __forceinline__ long long resolve_row(const Params& p, const Unit& x, const int* uidx,
                                                 int e, bool report) {
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

__global__ void __launch_bounds__(kThreads, 1)
sparse_mla_mma_kernel(const Params p) {
    extern __shared__ uint8_t smem_raw[];
    MmaSmem& sm = *reinterpret_cast<MmaSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    volatile int* abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.a_full[i], 32 * kGatherWarps);  // one cp.async arrival per gather thread
            mbar_init(&sm.a_free[i], kComputeWarps);
            mbar_init(&sm.q_full[i], 1);
            mbar_init(&sm.q_empty[i], kComputeWarps + kGatherWarps);
        }
        sm.abort = 0;
        fence_barrier_init();
    }
    // zero the stages once: rows of invalid keys are zero-filled by the gather anyway, and
    // the padding columns are never read
    for (int i = threadIdx.x; i < (int)(sizeof(sm.stage) / 16); i += kThreads)
        reinterpret_cast<uint4*>(sm.stage)[i] = make_uint4(0, 0, 0, 0);
    __syncthreads();

    if (warp >= kGatherWarp0) {
        // ================================ gather ================================
        const int gw = warp - kGatherWarp0;
        const bool leader = gw == 0 && lane == 0;
        int issued = 0;  // units whose query and indices have been requested
        auto issue_unit = [&](bool blocking) {
            const int u2 = blockIdx.x + issued * gridDim.x;
            if (u2 >= p.num_units) return;
            const int b2 = issued & 1;
            const uint32_t par = ((issued >> 1) & 1) ^ 1;
            if (!blocking && !mbar_try_wait(&sm.q_empty[b2], par)) return;
            if (blocking) wait_soft(&sm.q_empty[b2], par, abort, p.err);
            const Unit y = unit_of(p, u2);
            const uint32_t ibytes = (uint32_t)(y.e1 - y.e0) * 4u;
            mbar_arrive_expect_tx(&sm.q_full[b2], kH * kDqk * 2 + ibytes);
            for (int h = 0; h < kH; ++h)
                bulk_load(sm.q[b2] + h * kQPitch, p.q + ((long long)y.n * kH + h) * kDqk, kDqk * 2,
                          &sm.q_full[b2]);
            if (ibytes)
                bulk_load(sm.idx[b2], p.idx + (long long)y.n * p.ld_idx + y.e0, ibytes,
                          &sm.q_full[b2]);
            ++issued;
        };
        uint32_t G = 0;
        for (int ui = 0;; ++ui) {
            const int u = blockIdx.x + ui * gridDim.x;
            if (u >= p.num_units) break;
            const Unit x = unit_of(p, u);
            const int qb = ui & 1;
            if (leader) {
                while (issued <= ui) issue_unit(true);
                issue_unit(false);
            }
            wait_soft(&sm.q_full[qb], (ui >> 1) & 1, abort, p.err);
            const int* uidx = sm.idx[qb];
            for (int j = 0; j < x.nb; ++j, ++G) {
                const int s = G & 1;
                wait_soft(&sm.a_free[s], ((G >> 1) & 1) ^ 1, abort, p.err);
                long long row = -1;
                if (lane < 16) row = resolve_row(p, x, uidx, x.e0 + j * kBK + gw * 16 + lane, true);
                const uint32_t base = smem_u32(sm.stage[s]) + lane * 16;
                const char* kvb = reinterpret_cast<const char*>(p.kv) + lane * 16;
#pragma unroll 4
                for (int kl = 0; kl < 16; ++kl) {
                    const long long rr = __shfl_sync(0xffffffffu, row, kl);
                    const uint32_t dst = base + (gw * 16 + kl) * kRowPitch;
                    if (rr >= 0) {
                        const char* src = kvb + rr * (kDqk * 2);
                        cp_async_16(dst, src);
                        cp_async_16(dst + 512, src + 512);
                        if (lane < 8) cp_async_16(dst + 1024, src + 1024);
                    } else {
                        cp_async_16_zero(dst, p.kv);
                        cp_async_16_zero(dst + 512, p.kv);
                        if (lane < 8) cp_async_16_zero(dst + 1024, p.kv);
                    }
                }
                cp_async_mbar_arrive(&sm.a_full[s]);
                if (leader && issued == ui + 1) issue_unit(false);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.q_empty[qb]);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else {
        // ================================ compute ===============================
        const int kg = warp & 3;   // key group: keys 16*kg .. 16*kg+15 of a block
        const int kh = warp >> 2;  // K-half of the QK product
        const int g = lane >> 2;   // fragment row group
        const int t = lane & 3;    // thread in group
        uint32_t G = 0;
        for (int ui = 0;; ++ui) {
            const int u = blockIdx.x + ui * gridDim.x;
            if (u >= p.num_units) break;
            const Unit x = unit_of(p, u);
            const int qb = ui & 1;
            wait_soft(&sm.q_full[qb], (ui >> 1) & 1, abort, p.err);
            const int* uidx = sm.idx[qb];
            // this warp's K-half of Q as A fragments (16 heads x 16 dims per K-step)
            uint32_t qa[kKHalf][4];
            {
                const int head = (lane & 7) + ((lane >> 3) & 1) * 8;
                const uint32_t qrow = smem_u32(sm.q[qb]) + head * kQPitch + ((lane >> 4) & 1) * 16;
#pragma unroll
                for (int ks = 0; ks < kKHalf; ++ks)
                    ldsm_x4(qrow + (kh * kKHalf + ks) * 32, qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
            }
            float o[8][4];
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
            float m_run[2] = {-INFINITY, -INFINITY};  // heads g, g+8 (log2 domain)
            float l_run[2] = {0.f, 0.f};              // this thread's partial row sums
            float l_lse[2] = {0.f, 0.f};              // the same before bf16 rounding

            for (int j = 0; j < x.nb; ++j, ++G) {
                const int s = G & 1;
                wait_soft(&sm.a_full[s], (G >> 1) & 1, abort, p.err);
                const uint32_t st = smem_u32(sm.stage[s]);
                // ---- QK: S[16 heads x 16 keys] over this warp's K-half ----
                float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                {
                    const int key = kg * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
                    const uint32_t krow = st + key * kRowPitch + ((lane >> 3) & 1) * 16;
#pragma unroll
                    for (int ks = 0; ks < kKHalf; ++ks) {
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(krow + (kh * kKHalf + ks) * 32, b0, b1, b2, b3);
                        mma_bf16(acc[0], qa[ks], b0, b1);
                        mma_bf16(acc[1], qa[ks], b2, b3);
                    }
                }
                if (kh == 1) {
                    float4* dst = reinterpret_cast<float4*>(sm.spart[kg][lane]);
                    dst[0] = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
                    dst[1] = make_float4(acc[1][0], acc[1][1], acc[1][2], acc[1][3]);
                }
                compute_sync();
                if (kh == 0) {
                    const float4* src = reinterpret_cast<const float4*>(sm.spart[kg][lane]);
                    const float4 x0 = src[0], x1 = src[1];
                    acc[0][0] += x0.x; acc[0][1] += x0.y; acc[0][2] += x0.z; acc[0][3] += x0.w;
                    acc[1][0] += x1.x; acc[1][1] += x1.y; acc[1][2] += x1.z; acc[1][3] += x1.w;
                    // fragment (nt, i): head g + 8*(i>>1), key 16*kg + 8*nt + 2t + (i&1)
                    float sv[2][4];
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            const int e = x.e0 + j * kBK + kg * 16 + nt * 8 + 2 * t + c;
                            const bool valid = resolve_row(p, x, uidx, e, false) >= 0;
                            sv[nt][c] = valid ? acc[nt][c] * p.scale_log2 : -INFINITY;
                            sv[nt][2 + c] = valid ? acc[nt][2 + c] * p.scale_log2 : -INFINITY;
                        }
                    }
                    // per-head maximum over this warp's 16 keys (rows g and g+8)
                    float mx0 = fmaxf(fmaxf(sv[0][0], sv[0][1]), fmaxf(sv[1][0], sv[1][1]));
                    float mx1 = fmaxf(fmaxf(sv[0][2], sv[0][3]), fmaxf(sv[1][2], sv[1][3]));
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
                    if (t == 0) {
                        sm.red[kg][g] = mx0;
                        sm.red[kg][g + 8] = mx1;
                    }
                    named_bar_sync(2, 128);  // the four K-half-0 warps
                    float bm[2];
                    bm[0] = fmaxf(fmaxf(sm.red[0][g], sm.red[1][g]), fmaxf(sm.red[2][g], sm.red[3][g]));
                    bm[1] = fmaxf(fmaxf(sm.red[0][g + 8], sm.red[1][g + 8]),
                                  fmaxf(sm.red[2][g + 8], sm.red[3][g + 8]));
                    float alpha[2], ref[2];
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const float mn = fmaxf(m_run[r], bm[r]);
                        alpha[r] = m_run[r] == -INFINITY ? 0.f : exp2f(m_run[r] - mn);
                        m_run[r] = mn;
                        ref[r] = mn == -INFINITY ? 0.f : mn;  // no valid key yet: P = 0 anyway
                        l_run[r] *= alpha[r];
                        l_lse[r] *= alpha[r];
                    }
                    // P = exp2(s - m) in bf16; invalid keys (s = -inf) give exactly 0
                    uint8_t* pb = sm.p[s];
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                        for (int r = 0; r < 2; ++r) {
                            const float p0 = exp2f(sv[nt][2 * r] - ref[r]);
                            const float p1 = exp2f(sv[nt][2 * r + 1] - ref[r]);
                            const uint32_t pk = pack_bf16(p0, p1);
                            const __nv_bfloat162 pr = *reinterpret_cast<const __nv_bfloat162*>(&pk);
                            l_run[r] += __bfloat162float(pr.x) + __bfloat162float(pr.y);
                            l_lse[r] += p0 + p1;
                            const int head = g + 8 * r;
                            const int key = kg * 16 + nt * 8 + 2 * t;
                            *reinterpret_cast<uint32_t*>(pb + head * kPPitch + key * 2) = pk;
                        }
                    }
                    if (kg == 0 && t == 0) {
                        sm.alpha[g] = alpha[0];
                        sm.alpha[g + 8] = alpha[1];
                    }
                }
                compute_sync();  // P and alpha of this block are in shared memory
                // ---- PV: O[16 heads x 64 dims of this warp] += P[16 x 64 keys] V ----
                {
                    const float a0 = sm.alpha[g], a1 = sm.alpha[g + 8];
#pragma unroll
                    for (int n = 0; n < 8; ++n) {
                        o[n][0] *= a0; o[n][1] *= a0;
                        o[n][2] *= a1; o[n][3] *= a1;
                    }
                    const int head = (lane & 7) + ((lane >> 3) & 1) * 8;
                    const uint32_t prow = smem_u32(sm.p[s]) + head * kPPitch + ((lane >> 4) & 1) * 16;
                    const int vkey = (lane & 7) + ((lane >> 3) & 1) * 8;
                    const uint32_t vrow = st + vkey * kRowPitch + (warp * 64 + ((lane >> 4) & 1) * 8) * 2;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        uint32_t pa[4];
                        ldsm_x4(prow + kk * 32, pa[0], pa[1], pa[2], pa[3]);
#pragma unroll
                        for (int n2 = 0; n2 < 4; ++n2) {
                            uint32_t b0, b1, b2, b3;
                            ldsm_x4_t(vrow + kk * 16 * kRowPitch + n2 * 32, b0, b1, b2, b3);
                            mma_bf16(o[2 * n2], pa, b0, b1);
                            mma_bf16(o[2 * n2 + 1], pa, b2, b3);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.a_free[s]);  // stage and P buffer reusable
            }

            // ---- epilogue of the unit: row sums, normalise, write ----
            if (kh == 0) {
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
                    l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
                    l_lse[r] += __shfl_xor_sync(0xffffffffu, l_lse[r], 1);
                    l_lse[r] += __shfl_xor_sync(0xffffffffu, l_lse[r], 2);
                }
                if (t == 0) {
                    sm.lsum[kg][g] = l_run[0];
                    sm.lsum[kg][g + 8] = l_run[1];
                }
            }
            compute_sync();
            float L[2], Lx[2] = {0.f, 0.f};
            L[0] = sm.lsum[0][g] + sm.lsum[1][g] + sm.lsum[2][g] + sm.lsum[3][g];
            L[1] = sm.lsum[0][g + 8] + sm.lsum[1][g + 8] + sm.lsum[2][g + 8] + sm.lsum[3][g + 8];
            compute_sync();  // lsum is reused for the exact sums below
            if (kh == 0 && t == 0) {
                sm.lsum[kg][g] = l_lse[0];
                sm.lsum[kg][g + 8] = l_lse[1];
            }
            compute_sync();
            Lx[0] = sm.lsum[0][g] + sm.lsum[1][g] + sm.lsum[2][g] + sm.lsum[3][g];
            Lx[1] = sm.lsum[0][g + 8] + sm.lsum[1][g + 8] + sm.lsum[2][g + 8] + sm.lsum[3][g + 8];
            // m_run is only kept by the K-half-0 warps; broadcast it through alpha's slot
            compute_sync();
            if (kh == 0 && kg == 0 && t == 0) {
                sm.alpha[g] = m_run[0];
                sm.alpha[g + 8] = m_run[1];
            }
            compute_sync();
            const float mr[2] = {sm.alpha[g], sm.alpha[g + 8]};
            const float inv0 = (x.nb > 0 && L[0] > 0.f) ? 1.f / L[0] : 0.f;
            const float inv1 = (x.nb > 0 && L[1] > 0.f) ? 1.f / L[1] : 0.f;
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                const int dim = warp * 64 + n * 8 + 2 * t;
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
                    const float l = (x.nb > 0 && Lx[r] > 0.f) ? (mr[r] + log2f(Lx[r])) * 0.69314718055994531f
                                                           : -INFINITY;
                    if (p.page_table == nullptr) {
                        if (p.lse != nullptr) p.lse[(long long)x.n * kH + head] = l;
                    } else {
                        p.lse_part[((long long)x.n * p.splits + x.sp) * kH + head] = l;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.q_empty[qb]);
        }
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

size_t mla_mma_smem_bytes() { return sizeof(MmaSmem) + 128; }

cudaError_t launch_sparse_mla_mma(const __nv_bfloat16* q, const __nv_bfloat16* kv,
                                  long long kv_rows, const int* page_table, int max_pages,
                                  int page_size, const int* seq_lens, const int* idx, int k_sel,
                                  long long ld_idx, int num_q, float scale, int splits,
                                  __nv_bfloat16* out, float* lse, float* o_part, float* lse_part,
                                  cudaStream_t stream, const DevCtx& ctx) {
    Params p{};
    p.q = q;
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
    p.splits = page_table ? splits : 1;
    p.chunk = page_table ? ((k_sel + splits - 1) / splits + kBK - 1) / kBK * kBK : k_sel;
    p.num_units = num_q * p.splits;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.out = out;
    p.lse = lse;
    p.o_part = o_part;
    p.lse_part = lse_part;
    p.err = ctx.err;
    const size_t smem = mla_mma_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(sparse_mla_mma_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = p.num_units < ctx.num_sms ? p.num_units : ctx.num_sms;
    sparse_mla_mma_kernel<<<grid, kThreads, smem, stream>>>(p);
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
