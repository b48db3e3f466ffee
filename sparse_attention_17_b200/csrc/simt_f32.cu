// simt_f32.cu -- fp32 kernels for the small DSA layer of the DSA ablation model card
// (lightning indexer with 2 heads x dim 16, top-512, 4 attention heads of dim 32, context
// 3072).  The work is about 1 GFLOP in total, so these are plain SIMT kernels; the bf16
// paths for the 576-dim MLA layers are indexer_tc.cu (tcgen05) and mla_mma.cu.
#include "dsa_common.cuh"
#include "launch.h"

namespace dsa {

namespace {

constexpr int kIdxKeysPerBlock = 128;

// One block per (query row, 128-key tile): every thread scores one key.
//   I(t,s) = sum_j w[t,j] * max(0, q[t,j,:] . k[s,:])
__global__ void __launch_bounds__(kIdxKeysPerBlock)
indexer_scores_f32_kernel(const float* __restrict__ q_idx, const float* __restrict__ k_idx,
                          const float* __restrict__ w, int H_I, int D_I, int q_begin,
                          float* __restrict__ scores, long long ld) {
    extern __shared__ float sq[];  // [H_I * D_I] query vectors, then [H_I] weights
    const int r = blockIdx.x;
    const long long t = (long long)q_begin + r;
    const int s0 = blockIdx.y * kIdxKeysPerBlock;
    if (s0 > t) return;  // tile entirely above the diagonal
    const int HD = H_I * D_I;
    for (int i = threadIdx.x; i < HD; i += blockDim.x) sq[i] = q_idx[t * HD + i];
    for (int i = threadIdx.x; i < H_I; i += blockDim.x) sq[HD + i] = w[t * H_I + i];
    __syncthreads();
    const int s = s0 + threadIdx.x;
    if (s > t) return;
    const float4* kr = reinterpret_cast<const float4*>(k_idx + (long long)s * D_I);
    float acc = 0.f;
    for (int j = 0; j < H_I; ++j) {
        const float* qj = sq + j * D_I;
        float dot = 0.f;
        for (int d4 = 0; d4 < D_I / 4; ++d4) {
            const float4 kv = __ldg(kr + d4);
            dot = fmaf(qj[4 * d4 + 0], kv.x, dot);
            dot = fmaf(qj[4 * d4 + 1], kv.y, dot);
            dot = fmaf(qj[4 * d4 + 2], kv.z, dot);
            dot = fmaf(qj[4 * d4 + 3], kv.w, dot);
        }
        acc = fmaf(sq[HD + j], fmaxf(dot, 0.f), acc);
    }
    scores[(long long)r * ld + s] = acc;
}

// Sparse multi-head attention over the selected keys, fp32.  One block per query, one
// warp per head; lane l owns dims l and l+32.  Online softmax in the log2 domain.
__global__ void sparse_mha_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                                      const float* __restrict__ v, int H, int D,
                                      float scale_log2, long long kv_rows,
                                      const int* __restrict__ idx, int k_sel, long long ld_idx,
                                      float* __restrict__ out, float* __restrict__ lse,
                                      unsigned* __restrict__ err) {
    const int n = blockIdx.x;
    const int h = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (h >= H) return;
    const long long qoff = ((long long)n * H + h) * D;
    const float q0 = lane < D ? q[qoff + lane] : 0.f;
    const float q1 = lane + 32 < D ? q[qoff + lane + 32] : 0.f;
    float m = -INFINITY, l = 0.f, o0 = 0.f, o1 = 0.f;
    const int* sel = idx + (long long)n * ld_idx;
    bool bad = false;
    for (int i = 0; i < k_sel; ++i) {
        const int s = __ldg(sel + i);
        if (s < 0) continue;
        if (s >= kv_rows) { bad = true; continue; }
        const long long koff = ((long long)s * H + h) * D;
        float part = (lane < D ? q0 * k[koff + lane] : 0.f) +
                     (lane + 32 < D ? q1 * k[koff + lane + 32] : 0.f);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        const float x = part * scale_log2;
        const float m_new = fmaxf(m, x);
        const float alpha = exp2f(m - m_new);
        const float p = exp2f(x - m_new);
        l = l * alpha + p;
        o0 = o0 * alpha + p * (lane < D ? v[koff + lane] : 0.f);
        o1 = o1 * alpha + p * (lane + 32 < D ? v[koff + lane + 32] : 0.f);
        m = m_new;
    }
    if (bad && lane == 0) atomicOr(err, DSA_DEVERR_INDEX_RANGE);
    const float inv = l > 0.f ? 1.f / l : 0.f;
    if (lane < D) out[qoff + lane] = o0 * inv;
    if (lane + 32 < D) out[qoff + lane + 32] = o1 * inv;
    if (lse != nullptr && lane == 0)
        lse[(long long)n * H + h] = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace

cudaError_t launch_indexer_f32(const float* q_idx, const float* k_idx, const float* w, int H_I,
                               int D_I, int q_begin, int rows, float* scores, long long ld,
                               cudaStream_t stream) {
    const int max_key = q_begin + rows;  // keys 0 .. q_begin+rows-1
    dim3 grid(rows, (max_key + kIdxKeysPerBlock - 1) / kIdxKeysPerBlock);
    const size_t smem = sizeof(float) * (size_t)(H_I * D_I + H_I);
    indexer_scores_f32_kernel<<<grid, kIdxKeysPerBlock, smem, stream>>>(q_idx, k_idx, w, H_I,
                                                                         D_I, q_begin, scores, ld);
    count_launch(DSA_KERNEL_INDEXER);
    return cudaGetLastError();
}

cudaError_t launch_sparse_mha_f32(const float* q, const float* k, const float* v, int num_q,
                                  int H, int D, float scale, long long kv_rows, const int* idx,
                                  int k_sel, long long ld_idx, float* out, float* lse,
                                  cudaStream_t stream, const DevCtx& ctx) {
    const float scale_log2 = scale * 1.4426950408889634f;
    sparse_mha_f32_kernel<<<num_q, 32 * H, 0, stream>>>(q, k, v, H, D, scale_log2, kv_rows, idx,
                                                         k_sel, ld_idx, out, lse, ctx.err);
    count_launch(DSA_KERNEL_ATTENTION);
    return cudaGetLastError();
}

}  // namespace dsa
