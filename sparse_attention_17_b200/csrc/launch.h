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

// Builds a 2-D bf16 tensor map (rows x cols, row pitch in bytes) with a box of
// box_rows x box_cols and 128-byte swizzle.  Returns false if the driver rejects it.
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint64_t row_pitch_bytes, uint32_t box_rows, uint32_t box_cols);

cudaError_t launch_indexer_f32(const float* q_idx, const float* k_idx, const float* w, int H_I,
                               int D_I, int q_begin, int rows, float* scores, long long ld,
                               cudaStream_t stream);

cudaError_t launch_indexer_bf16_prefill(const __nv_bfloat16* q_idx, const __nv_bfloat16* k_idx,
                                        const float* w, int T, int S, int q_begin, int rows,
                                        float* scores, long long ld, cudaStream_t stream,
                                        const DevCtx& ctx);

cudaError_t launch_indexer_bf16_decode(const __nv_bfloat16* q_idx, const __nv_bfloat16* k_pool,
                                       const float* w, int B, long long pool_rows,
                                       const int* page_table, int max_pages, int page_size,
                                       const int* seq_lens, int max_len, float* scores,
                                       long long ld, cudaStream_t stream, const DevCtx& ctx);

cudaError_t launch_topk(const float* scores, long long ld, int rows, int q_begin,
                        const int* row_len, int max_len, int k, int* idx, long long ld_idx,
                        cudaStream_t stream, const DevCtx& ctx);

cudaError_t launch_sparse_mha_f32(const float* q, const float* k, const float* v, int num_q,
                                  int H, int D, float scale, long long kv_rows, const int* idx,
                                  int k_sel, long long ld_idx, float* out, float* lse,
                                  cudaStream_t stream, const DevCtx& ctx);

// Absorbed-MLA sparse attention (bf16, 16 heads, 576/512) on warp-level MMAs.  Prefill
// when page_table is NULL; otherwise decode with `splits` key ranges per sequence written
// to the partial buffers (o_part [num_q, splits, 16, 512] fp32, lse_part [num_q, splits,
// 16]) and merged by launch_mla_combine.
cudaError_t launch_sparse_mla_mma(const __nv_bfloat16* q, const __nv_bfloat16* kv,
                                  long long kv_rows, const int* page_table, int max_pages,
                                  int page_size, const int* seq_lens, const int* idx, int k_sel,
                                  long long ld_idx, int num_q, float scale, int splits,
                                  __nv_bfloat16* out, float* lse, float* o_part, float* lse_part,
                                  cudaStream_t stream, const DevCtx& ctx);

cudaError_t launch_mla_combine(const float* o_part, const float* lse_part, int num_q, int splits,
                               __nv_bfloat16* out, float* lse, cudaStream_t stream);

// Split count the decode path uses for this many sequences and selected keys.
int mla_decode_splits(int num_q, int k_sel, int num_sms);

}  // namespace dsa
