// launch.h -- host-side launchers of the DSA kernels (internal to libdsa.so).
// The C ABI in capi.cu validates arguments and then calls these.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dsa.h"

namespace dsa {

// Per-device facts the launchers need.
struct DevCtx {
    int device;
    int num_sms;
    unsigned* err;  // device address of this device's error word
};

// Fills ctx for the current device (cached per device).
cudaError_t get_dev_ctx(DevCtx* ctx);

// Counts one launch of a kernel family (dsa_launch_count).
void count_launch(int kind);

// Launches a kernel whose first statement is chained_launch_gate() with programmatic
// dependent launch allowed: it is launched once the previous kernel of the stream has no
// CTA left running instead of once that kernel has completed, so that the launch overlaps
// the completion; the gate keeps every global memory access after the previous work has
// completed and is visible.  cluster > 1 adds a cluster dimension (x).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                  cudaStream_t stream, unsigned cluster, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// The calling thread's message for dsa_last_error: cleared on entry to every call, set
// (printf-style) with the status a call returns on failure.
void clear_last_error();
dsa_status fail_with(dsa_status st, const char* fmt, ...);

// Builds a 2-D bf16 tensor map (rows x cols, row pitch in bytes) with a box of
// box_rows x box_cols and 128-byte swizzle.  Returns false if the driver rejects it.
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint64_t row_pitch_bytes, uint32_t box_rows, uint32_t box_cols);

cudaError_t launch_indexer_f32(const float* q_idx, const float* k_idx, const float* w, int H_I,
                               int D_I, int q_begin, int rows, float* scores, long long ld,
                               cudaStream_t stream);

// Dense prefill scores of query rows [q_begin, q_begin+rows).  With `guard` non-null the
// launch does nothing unless *guard != 0 (the filtered path's fallback).
cudaError_t launch_indexer_bf16_prefill(const __nv_bfloat16* q_idx, const __nv_bfloat16* k_idx,
                                        const float* w, int T, int S, int q_begin, int rows,
                                        float* scores, long long ld, cudaStream_t stream,
                                        const DevCtx& ctx, const int* guard = nullptr);

// Scores of every tile_stride-th 128-key tile only, stored compactly: row r, logical tile j
// at sample[r * ld_sample + j * 128 ...] (causal entries only).
cudaError_t launch_indexer_bf16_sample(const __nv_bfloat16* q_idx, const __nv_bfloat16* k_idx,
                                       const float* w, int T, int S, int q_begin, int rows,
                                       int tile_stride, float* sample, long long ld_sample,
                                       cudaStream_t stream, const DevCtx& ctx);

// Filtered prefill scores: for row r, every causal key with order key >= tau[r] is
// appended to the list of its 4096-key chunk c and TMEM lane quadrant q (the key's bits
// 5..6): cand[((r * nchunk_max + c) * 4 + q) * cq ..] ({order key, key index}) with its
// length in ccount[(r * nchunk_max + c) * 4 + q] (also when past cq).
cudaError_t launch_indexer_bf16_filter(const __nv_bfloat16* q_idx, const __nv_bfloat16* k_idx,
                                       const float* w, int T, int S, int q_begin, int rows,
                                       const uint32_t* tau, uint2* cand, uint32_t* ccount, int cq,
                                       int nchunk_max, cudaStream_t stream, const DevCtx& ctx);

cudaError_t launch_indexer_bf16_decode(const __nv_bfloat16* q_idx, const __nv_bfloat16* k_pool,
                                       const float* w, int B, long long pool_rows,
                                       const int* page_table, int max_pages, int page_size,
                                       const int* seq_lens, int max_len, float* scores,
                                       long long ld, cudaStream_t stream, const DevCtx& ctx);

// Per-row top-k of dense score rows.  With row_mask non-null, only rows r with
// row_mask[r] != 0 are processed (the filtered path's fallback).  idx_offset is added to
// every selected key position (the first token of a packed sequence).
cudaError_t launch_topk(const float* scores, long long ld, int rows, int q_begin,
                        const int* row_len, int max_len, int k, int* idx, long long ld_idx,
                        cudaStream_t stream, const DevCtx& ctx, const int* row_mask = nullptr,
                        int idx_offset = 0);

// Sampled keys per row the threshold kernel holds at most (tiles x 128).
int topk_sample_max();

// Filtered path, step 2: per-row threshold tau (an order key) from the compact sampled
// scores of launch_indexer_bf16_sample (at most topk_sample_max() per row).  Clears
// *fb_any.
cudaError_t launch_topk_threshold(const float* sample, long long ld_sample, int q_begin, int rows,
                                  int tile_stride, int k, uint32_t* tau, int* fb_any,
                                  cudaStream_t stream);

// Filtered path, step 4: exact top-k of each row from its candidate lists (the output of
// launch_indexer_bf16_filter).  Rows it cannot settle (a list past cq, more candidates than
// the selection buffer holds, or fewer than k) get fb_row[r] = 1 and *fb_any = 1 and are
// left for the dense fallback.
cudaError_t launch_topk_candidates(const uint2* cand, const uint32_t* ccount, int cq,
                                   int nchunk_max, int q_begin, int rows, int max_len, int k,
                                   int* idx, long long ld_idx, int* fb_row, int* fb_any,
                                   cudaStream_t stream);

cudaError_t launch_sparse_mha_f32(const float* q, const float* k, const float* v, int num_q,
                                  int H, int D, float scale, long long kv_rows, const int* idx,
                                  int k_sel, long long ld_idx, float* out, float* lse,
                                  cudaStream_t stream, const DevCtx& ctx);

// Absorbed-MLA sparse attention (bf16 query, 16 heads, 576/512; bf16 latent cache, or E4M3
// codes times kv_scale when kv_fp8) on warp-level MMAs.  Prefill
// when page_table is NULL; otherwise decode with `splits` key ranges per sequence written
// to the partial buffers (o_part [num_q, splits, 16, 512] fp32, lse_part [num_q, splits,
// 16]) and merged by launch_mla_combine.
cudaError_t launch_sparse_mla_mma(const __nv_bfloat16* q, const void* kv, bool kv_fp8,
                                  float kv_scale, long long kv_rows, const int* page_table,
                                  int max_pages, int page_size, const int* seq_lens,
                                  const int* idx, int k_sel, long long ld_idx, int num_q,
                                  float scale, int splits, __nv_bfloat16* out, float* lse,
                                  float* o_part, float* lse_part, cudaStream_t stream,
                                  const DevCtx& ctx);

// dst[i] = E4M3(src[i] / kv_scale) (round to nearest even, finite saturation).
cudaError_t launch_latent_quantize_fp8(const __nv_bfloat16* src, long long n, float kv_scale,
                                       uint8_t* dst, cudaStream_t stream, const DevCtx& ctx);

// One CTA whose bounded mbarrier wait runs out (2 s); *gave_up <- 1 if it gave up.
cudaError_t launch_wait_timeout_selftest(int* gave_up, cudaStream_t stream, const DevCtx& ctx);

cudaError_t launch_mla_combine(const float* o_part, const float* lse_part, int num_q, int splits,
                               __nv_bfloat16* out, float* lse, cudaStream_t stream);

// Split count the decode path uses for this many sequences and selected keys.
int mla_decode_splits(int num_q, int k_sel, int num_sms);

}  // namespace dsa
