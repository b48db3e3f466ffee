/*
 * dsa.h -- C ABI of the B200 (sm_100a) DeepSeek Sparse Attention hot path.
 *
 * The library computes, on one GPU, the three steps of DSA prefill and decode and the
 * IndexCache reuse of selected indices across layers:
 *
 *   dsa_indexer_scores   lightning-indexer scores  I(t,s) = sum_j w[t,j] * ReLU(q_idx[t,j] . k_idx[s])
 *   dsa_topk_select      per-row top-k of those scores (ties -> lower index), ascending, -1 padded
 *   dsa_sparse_mla_fwd   attention of each query over its selected keys only (absorbed MLA:
 *                        one 576-dim latent row per token shared by all heads, value = first
 *                        512 dims; or plain multi-head attention for the fp32 path)
 *   dsa_layer_stack      an F/S pattern of layers: F layers run indexer + top-k into one
 *                        index buffer, S layers reuse it (IndexCache)
 *   dsa_sparse_mla_fp8_fwd, dsa_latent_quantize_fp8
 *                        the same attention over an fp8 (E4M3) latent cache, and the
 *                        conversion of bf16 latent rows into such a cache
 *
 * Sources.  DSA ablation model card ("Attention" bullet: a ReLU lightning indexer picks the
 * top-k keys per query; closing note: prompts no longer than k attend densely);
 * DSV2-Lite-IndexCache-Sparse-1250 card (first paragraph: causal selection budget of 2048,
 * FSS pattern repeated nine times, full layers' routes reused by shared layers);
 * DeepSeek-V2-Lite-Chat SIQ card (MLA with kv_lora_rank 512, 576 B per token at fp8, i.e.
 * a 576-element latent); vLLM IndexCache docs ("Configuration Reference": index_topk_freq
 * and index_topk_pattern; "How It Works": F layers store top-k indices, S layers receive
 * them).  The indexer formula itself is not printed on those pages; this library takes the
 * standard DSA form above with one indexer key per token shared by all indexer heads.
 *
 * Conventions for every call:
 *   - All tensor arguments are DEVICE pointers owned by the caller; the library never
 *     allocates, frees or retains them.  Scratch memory is passed in as `workspace`.
 *   - Tensors are dense row-major ("C order") unless a leading dimension is given.
 *     Tensor pointers must be 16-byte aligned; leading dimensions are in elements.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream).  Results are valid once the stream has reached the call.  The indexer,
 *     top-k, attention and split-merge kernels are launched with programmatic dependent
 *     launch: one may start while the previous kernel of the stream drains, and waits
 *     (griddepcontrol) for that work to complete before touching memory, so stream order
 *     holds as for any launch.
 *   - Argument errors return DSA_ERR_INVALID_ARG / DSA_ERR_UNSUPPORTED before anything is
 *     launched; dsa_last_error() then describes the problem.  DSA_ERR_CUDA reports a
 *     failed launch or CUDA runtime call.
 *   - Indices handed to dsa_sparse_mla_fwd that fall outside the valid key range are
 *     skipped by the kernel and recorded in a per-device error word, which
 *     dsa_check_device_errors() reads and clears.  They never cause an out-of-bounds read.
 *   - Results are deterministic: no floating-point atomics; identical inputs give
 *     bit-identical outputs.
 *   - Thread safety: calls may be issued from several host threads on different streams.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dsa_stream_t; /* same type as cudaStream_t */

typedef enum {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1,  /* a pointer, size, stride or alignment is wrong */
    DSA_ERR_UNSUPPORTED = 2,  /* a valid request the library has no kernel for */
    DSA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required */
    DSA_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
    DSA_ERR_DEVICE_CHECK = 5  /* a kernel recorded an invalid input (see error bits) */
} dsa_status;

typedef enum { DSA_F32 = 0, DSA_BF16 = 1, DSA_FP8_E4M3 = 2 } dsa_dtype;
typedef enum { DSA_PREFILL = 0, DSA_DECODE = 1 } dsa_mode;

/* Bits of the per-device error word (dsa_check_device_errors). */
#define DSA_DEVERR_INDEX_RANGE 0x1u  /* a selected index outside [0, valid length) */
#define DSA_DEVERR_PAGE_RANGE  0x2u  /* a page-table entry outside the page pool */
#define DSA_DEVERR_TIMEOUT     0x4u  /* an internal pipeline wait gave up (kernel bug) */

/* Kernel families counted by dsa_launch_count(). */
typedef enum {
    DSA_KERNEL_INDEXER = 0,
    DSA_KERNEL_TOPK = 1,
    DSA_KERNEL_ATTENTION = 2,
    DSA_KERNEL_COMBINE = 3,
    DSA_KERNEL_QUANTIZE = 4,
    DSA_KERNEL_KINDS = 5
} dsa_kernel_kind;

/* Human-readable name of a status code (static storage). */
const char* dsa_status_string(int status);

/* Detail of the last error returned on the calling host thread ("" if none). */
const char* dsa_last_error(void);

/* ABI version of this header: (major << 16) | minor.  1.1 added dsa_index_select,
 * dsa_index_varlen, the fp8 cache calls, dsa_selftest_wait_timeout and
 * DSA_KERNEL_QUANTIZE. */
int dsa_version(void);

/*
 * dsa_indexer_scores -- lightning indexer scores (DSA ablation card, "Attention" bullet).
 *
 *   I(t,s) = sum_{j < H_I} w[t,j] * max(0, sum_{d < D_I} q_idx[t,j,d] * k_idx[s,d])
 *
 * mode DSA_PREFILL (causal, DSV2-Lite-IndexCache card: causal key selection):
 *   q_idx  [T, H_I, D_I]   dtype (bf16 or fp32), T >= q_begin + rows
 *   k_idx  [S, D_I]        dtype, S >= q_begin + rows
 *   w      [T, H_I]        fp32
 *   Row r of `scores` is query t = q_begin + r; columns s = 0..t hold I(t,s).  Columns
 *   t+1 .. ld_scores-1 are unspecified (the kernel may or may not write them).
 *   page_table, seq_lens must be NULL; max_pages, page_size are ignored.
 * mode DSA_DECODE (bf16 only; one new query per sequence, keys read through pages):
 *   q_idx  [B, H_I, D_I]   with B = rows, q_begin = 0
 *   k_idx  [num_pages, page_size, D_I] page pool; S = num_pages * page_size
 *   w      [B, H_I]
 *   page_table [B, max_pages] int32: token s of sequence b is pool row
 *              page_table[b, s / page_size] * page_size + s % page_size
 *   seq_lens   [B] int32: sequence b scores keys 0..seq_lens[b]-1 (the new token's key is
 *              already in the cache); 1 <= seq_lens[b] <= min(ld_scores, max_pages*page_size).
 *   Columns >= seq_lens[b] are unspecified.
 * scores [rows, ld_scores] fp32, ld_scores a multiple of 4 and >= q_begin + rows (prefill).
 * Supported: bf16 with H_I = 16, D_I = 64; fp32 (prefill only) with H_I * D_I <= 256 and
 * D_I a multiple of 4.  Page sizes: multiples of 16 (decode).
 */
dsa_status dsa_indexer_scores(int dtype, int mode, const void* q_idx, const void* k_idx,
                              const float* w, int H_I, int D_I, int q_begin, int rows, int S,
                              const int* page_table, int max_pages, int page_size,
                              const int* seq_lens, float* scores, long long ld_scores,
                              dsa_stream_t stream);

/*
 * dsa_topk_select -- per-row top-k (DSA ablation card: top-k keys per query; its closing
 * note: when a row has no more than k valid keys, all of them are selected).
 *
 * Row r has n_r valid scores in columns 0..n_r-1 of scores[r * ld_scores ...]:
 *   row_len == NULL:  n_r = q_begin + r + 1          (causal prefill rows)
 *   row_len != NULL:  n_r = row_len[r] (device int32) (decode rows)
 * and 1 <= n_r <= max_len <= ld_scores.  Selection: the k valid keys with the largest
 * scores; among equal scores the lower index wins (-0.0 and +0.0 are equal).  If n_r <= k
 * all n_r keys are selected.  idx[r * ld_idx + i], i < k, receives the selected key
 * positions in ascending order followed by -1 padding.  Scores must not be NaN.
 * Limits: 1 <= k <= 4096, max_len <= 262144, ld_idx >= k, ld_scores a multiple of 4
 * (rows start on 16-byte boundaries); scores, idx and row_len 16-byte aligned.
 */
dsa_status dsa_topk_select(const float* scores, long long ld_scores, int rows, int q_begin,
                           const int* row_len, int max_len, int k, int* idx,
                           long long ld_idx, dsa_stream_t stream);

/*
 * dsa_index_select -- lightning-indexer scores and the per-row top-k of causal prefill rows
 * in one call, without writing the dense score rows (DSA ablation card, "Attention" bullet:
 * every key is scored, the top-k keys are kept).  The result is identical to
 * dsa_indexer_scores (bf16, prefill) followed by dsa_topk_select on the same rows: the same
 * tensor-core scores, the same selection rule and ties, the same output layout.
 *
 * Method: per window of rows, one 128-key tile in 16 is scored first and each row gets a
 * threshold a few standard deviations below the score its k-th largest key is expected to
 * have; the full scoring pass then appends only the keys above the threshold to per-row
 * candidate lists and marks the keys equal to it in a bitmap; the exact top-k is taken among
 * those.  A row the candidates cannot settle (too many, or too few together with the
 * ties) is recomputed from dense scores of its window, so the result never depends on the
 * sample.
 *
 * q_idx [q_begin+rows, 16, 64] bf16 (query t in row t), k_idx [S, 64] bf16, w [q_begin+rows,
 * 16] fp32; query row t = q_begin + r has the n = t + 1 keys 0..t (q_begin + rows <= S <=
 * 262144).  idx [rows, ld_idx] int32 receives, per row, the selected key positions in
 * ascending order then -1 padding (1 <= k <= 4096, ld_idx >= k, a multiple of 4).
 * workspace: caller-owned device scratch, 256-byte aligned; rows are processed in windows
 * of the largest multiple of 16 rows (or all rows) for which
 * dsa_index_select_workspace_size(window, S) <= ws_bytes; fewer than 16 rows ->
 * DSA_ERR_WORKSPACE.  Supported: H_I = 16, D_I = 64 (else DSA_ERR_UNSUPPORTED).
 */
dsa_status dsa_index_select(const void* q_idx, const void* k_idx, const float* w, int H_I,
                            int D_I, int q_begin, int rows, int S, int k, int* idx,
                            long long ld_idx, void* workspace, size_t ws_bytes,
                            dsa_stream_t stream);

/* Scratch bytes dsa_index_select needs for a window of rows_window rows and S keys. */
size_t dsa_index_select_workspace_size(int rows_window, int S);

/*
 * dsa_sparse_mla_fwd -- attention over the selected keys only (DSV2-Lite-IndexCache card:
 * attention_mode="sparse"; its portable runtime is the same computation as masked SDPA).
 *
 * For query n, head h, with I_n the non-negative entries of idx[n * ld_idx + 0 .. k_sel-1]:
 *   logit_s = scale * q[n,h,:] . K(s)
 *   out[n,h,:] = sum_{s in I_n} softmax_s(logit) * V(s)
 *   lse[n,h]   = log sum_{s in I_n} exp(logit_s)            (natural log; -inf if I_n empty)
 * MLA (dtype DSA_BF16, num_kv_heads = 1, v = NULL): K(s) is the latent row kv[s, 0:D_qk]
 *   shared by all H heads and V(s) = kv[s, 0:D_v].  Supported: H = 16, D_qk = 576, D_v = 512.
 * MHA (dtype DSA_F32, num_kv_heads = H, v != NULL): K(s) = kv[s,h,:], V(s) = v[s,h,:],
 *   D_qk = D_v <= 64, H <= 16; prefill only.
 *
 * mode DSA_PREFILL:  q [num_q, H, D_qk]; kv [kv_rows, num_kv_heads, D_qk]; query n uses
 *   the rows named by idx directly (0 <= s < kv_rows is checked).  page_table, seq_lens NULL.
 * mode DSA_DECODE:   num_q = B sequences; kv is the page pool
 *   [kv_rows / page_size pages, page_size, D_qk]; token s of sequence n lives in pool row
 *   page_table[n, s / page_size] * page_size + s % page_size; only 0 <= s < seq_lens[n]
 *   is valid.  The decode path splits each sequence's keys over several CTAs and merges
 *   them with their log-sum-exp; it needs `workspace` of dsa_sparse_mla_workspace_size().
 * out [num_q, H, D_v] in dtype; lse [num_q, H] fp32 or NULL.
 * workspace may be NULL when dsa_sparse_mla_workspace_size() returns 0.
 */
dsa_status dsa_sparse_mla_fwd(int dtype, int mode, int num_q, int H, int num_kv_heads,
                              int D_qk, int D_v, float scale, const void* q, const void* kv,
                              const void* v, long long kv_rows, const int* page_table,
                              int max_pages, int page_size, const int* seq_lens,
                              const int* idx, int k_sel, long long ld_idx, void* out,
                              float* lse, void* workspace, size_t workspace_bytes,
                              dsa_stream_t stream);

/* Workspace bytes dsa_sparse_mla_fwd needs for this shape (0 for prefill). */
size_t dsa_sparse_mla_workspace_size(int mode, int num_q, int H, int D_v, int k_sel);

/*
 * dsa_sparse_mla_decode_noalloc -- the decode path of dsa_sparse_mla_fwd (bf16 absorbed
 * MLA, mode DSA_DECODE, same arguments and results) for callers that cannot allocate
 * device memory where they decode, e.g. inside a fixed-size memory pool or an
 * allocation-free serving loop.  The paper has no counterpart: this is a deployment
 * variant of the same computation.
 *
 * Instead of a caller workspace, the per-split partial results live in a 16 MiB device
 * array that belongs to the library; every GPU that loads the library holds it until
 * the process exits.  The call allocates nothing (no cudaMalloc, cudaFree or allocating
 * library routine).  Limits: num_q <= 511 sequences (fewer splits per sequence are used
 * when many sequences share the array); otherwise DSA_ERR_UNSUPPORTED, before anything is
 * launched.  The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream capture.
 * All calls share the one array: calls that overlap on the GPU (other streams, other host
 * threads) race and must be serialised by the caller.  Each call overwrites the parts of
 * the array it uses, so nothing has to be cleared between calls.  Errors: as for
 * dsa_sparse_mla_fwd; dsa_last_error() describes the failure.
 */
dsa_status dsa_sparse_mla_decode_noalloc(int num_q, int H, int D_qk, int D_v, float scale,
                                         const void* q, const void* kv, long long kv_rows,
                                         const int* page_table, int max_pages, int page_size,
                                         const int* seq_lens, const int* idx, int k_sel,
                                         long long ld_idx, void* out, float* lse,
                                         dsa_stream_t stream);

/*
 * dsa_index_varlen -- indexer + top-k for a batch of independent prefill sequences packed
 * along the token axis (batched prefill of unequal lengths; a left-padded batch [B, T] is
 * the packing with sequence b at rows b*T + pad_b .. (b+1)*T - 1 and the pads outside
 * every sequence).  DSV2-Lite-IndexCache card: causal selection per query, and batched
 * generation with left padding.
 *
 * Sequence b holds the tokens seq_start[b] .. seq_start[b] + seq_len[b] - 1 of
 *   q_idx [num_tokens, 16, 64] bf16, k_idx [num_tokens, 64] bf16, w [num_tokens, 16] fp32.
 * Token t of sequence b selects, exactly as dsa_indexer_scores + dsa_topk_select would for
 * that sequence alone, the top-k of I(t, s) over its own keys s = seq_start[b] .. t.
 * idx [num_tokens, ld_idx] int32: row t receives the selected keys as PACKED token rows
 * (so that dsa_sparse_mla_fwd in prefill mode reads them from the packed latent cache),
 * ascending, -1 padded.  Rows outside every sequence are not written.
 * seq_start, seq_len: HOST int32 arrays of num_seqs entries; sequences lie inside
 * [0, num_tokens), in increasing order, without overlap; lengths 0 .. 262144.
 * workspace: device memory for score rows, at least dsa_index_varlen_workspace_size(
 * longest sequence, 1) bytes; a larger workspace scores more rows per launch.
 * Launches one indexer and one top-k per sequence and window of rows; nothing is
 * synchronised.  Errors: as for dsa_indexer_scores / dsa_topk_select.
 */
dsa_status dsa_index_varlen(const void* q_idx, const void* k_idx, const float* w, int H_I,
                            int D_I, int num_tokens, int num_seqs, const int* seq_start,
                            const int* seq_len, int k, int* idx, long long ld_idx,
                            void* workspace, size_t workspace_bytes, dsa_stream_t stream);

/* Workspace bytes for dsa_index_varlen with windows of rows_window rows of the longest
 * sequence (0 = the library's default window, about 4 GB of scores). */
size_t dsa_index_varlen_workspace_size(int max_seq_len, int rows_window);

/*
 * dsa_sparse_mla_fp8_fwd -- dsa_sparse_mla_fwd (absorbed MLA, bf16 query, prefill or paged
 * decode) over an fp8 latent cache.  DeepSeek-V2-Lite-Chat SIQ card (what is quantized,
 * KV-cache bullet): fp8 KV at 576 bytes per token, one byte per latent element.
 *
 * Encoding (the card names only "fp8"; this is the reading used): each byte of `kv` is
 * an E4M3 code of the OCP 8-bit floating-point format (sign, 4 exponent bits with bias 7,
 * 3 mantissa bits, subnormals, 0x7f/0xff NaN, largest finite 448), and the latent element
 * is kv_scale * E4M3(code), with one fp32 kv_scale for the whole cache.  So
 *   logit_s = scale * kv_scale * q[n,h,:] . E4M3(kv[s,:])
 *   out[n,h,:] = kv_scale * sum_s softmax_s(logit) * E4M3(kv[s, 0:512])
 * kv [kv_rows, 576] uint8 (prefill) or [kv_rows / page_size, page_size, 576] (decode);
 * every other argument, the supported shapes (H = 16, D_qk = 576, D_v = 512), the
 * workspace (dsa_sparse_mla_workspace_size) and the error behaviour are those of
 * dsa_sparse_mla_fwd with dtype DSA_BF16.
 * Precision: the codes are widened exactly to f16 and the query is rounded to f16 for
 * the tensor-core products (bf16 query values must lie within +-65504; magnitudes below
 * 2^-14 keep f16's subnormal precision); probabilities are rounded to f16; fp32
 * accumulation; out rounded to bf16.  kv_scale must be finite and > 0.  NaN codes are
 * not supported.
 */
dsa_status dsa_sparse_mla_fp8_fwd(int mode, int num_q, int H, int D_qk, int D_v, float scale,
                                  float kv_scale, const void* q, const void* kv,
                                  long long kv_rows, const int* page_table, int max_pages,
                                  int page_size, const int* seq_lens, const int* idx,
                                  int k_sel, long long ld_idx, void* out, float* lse,
                                  void* workspace, size_t workspace_bytes,
                                  dsa_stream_t stream);

/*
 * dsa_latent_quantize_fp8 -- writes an fp8 latent cache for dsa_sparse_mla_fp8_fwd:
 *   dst[i] = E4M3(src[i] / kv_scale),  i = 0 .. n-1
 * src bf16 [n], dst uint8 [n] (both 16-byte aligned device pointers; n >= 0, any value).
 * The quotient is the fp32 IEEE division (round to nearest); the conversion rounds to the
 * nearest E4M3 value with ties to the even code, keeps the sign of values that round to
 * zero, and saturates finite magnitudes above 448 to +-448.  kv_scale finite and > 0.
 */
dsa_status dsa_latent_quantize_fp8(const void* src, long long n, float kv_scale, void* dst,
                                   dsa_stream_t stream);

/*
 * dsa_layer_stack -- IndexCache over an F/S layer pattern (vLLM IndexCache docs, "How It
 * Works"; DSV2-Lite-IndexCache card: "FSS" x 9).  Prefill, bf16 absorbed MLA.
 *
 * pattern: num_layers characters from {'F','S'}, pattern[0] == 'F'.
 * For layer l (arrays are HOST arrays of DEVICE pointers, length num_layers):
 *   'F': idx_buf <- top-k of the layer's own indexer scores
 *        (q_idx[l] [T,16,64] bf16, k_idx[l] [T,64] bf16, w[l] [T,16] fp32), computed in
 *        windows of query rows through `workspace`.
 *   'S': idx_buf is reused unchanged (no indexer or top-k launch; q_idx[l], k_idx[l],
 *        w[l] are not read and may be NULL).
 *   every layer: out[l] [T,16,512] <- sparse MLA of q[l] [T,16,576] over kv[l] [T,576]
 *        with the current idx_buf; lse[l] [T,16] fp32 if lse != NULL and lse[l] != NULL.
 * idx_buf [T, topk] int32 holds, on return, the indices of the last F layer.
 * workspace: at least dsa_layer_stack_workspace_size(T, 0) bytes; a larger workspace
 * processes more query rows per window.
 */
dsa_status dsa_layer_stack(const char* pattern, int num_layers, int T, int topk,
                           int H_I, int D_I, int H, int D_qk, int D_v, float scale,
                           const void* const* q_idx, const void* const* k_idx,
                           const float* const* w, const void* const* q,
                           const void* const* kv, void* const* out, float* const* lse,
                           int* idx_buf, void* workspace, size_t workspace_bytes,
                           dsa_stream_t stream);

/* Workspace bytes for dsa_layer_stack with windows of rows_window query rows
 * (0 = the library's default window). */
size_t dsa_layer_stack_workspace_size(int T, int rows_window);

/*
 * dsa_pattern_from_freq -- the pattern index_topk_freq describes (vLLM IndexCache docs,
 * "Configuration Reference": top-k computed every freq layers; freq 1 = every layer).
 * Layer i is 'F' iff i % freq == 0.  Writes num_layers characters and a NUL into
 * out[0 .. out_len-1]; out_len must be > num_layers.  Host-only.
 */
dsa_status dsa_pattern_from_freq(int freq, int num_layers, char* out, int out_len);

/*
 * dsa_selftest_wait_timeout -- runs the failure path of the kernels' pipeline waits: one
 * CTA waits on an mbarrier that nothing arrives on, with the same time-bounded wait every
 * kernel uses (2 s).  The wait gives up, records DSA_DEVERR_TIMEOUT in the device error
 * word (read it with dsa_check_device_errors) and the kernel exits; *gave_up (a device
 * int) receives 1.  No memory other than the error word and *gave_up is touched, and the
 * context stays usable.  Not part of the hot path: a check that a hung pipeline stage
 * becomes an error status instead of a hung GPU.
 */
dsa_status dsa_selftest_wait_timeout(int* gave_up, dsa_stream_t stream);

/* Reads and clears the current device's error word after synchronizing `stream`.
 * *error_bits (may be NULL) receives the DSA_DEVERR_* bits.  Returns
 * DSA_ERR_DEVICE_CHECK if any bit was set, DSA_OK otherwise. */
dsa_status dsa_check_device_errors(dsa_stream_t stream, unsigned* error_bits);

/* Number of kernels of a family this process has launched through the library (all
 * devices, all threads); used to check that S layers launch no indexer or top-k. */
long long dsa_launch_count(int kind);
void dsa_reset_launch_counts(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
