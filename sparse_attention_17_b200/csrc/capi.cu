// capi.cu -- the extern "C" boundary of libdsa.so (declared in include/dsa.h).
//
// Every entry point validates its arguments on the host and returns before launching
// anything when they are wrong; then it calls the launchers of the kernel files.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "dsa_common.cuh"
#include "launch.h"

#if defined(DSA_NVTX) && DSA_NVTX
#include <nvtx3/nvToolsExt.h>
#endif

namespace dsa {

// Per-device error word: kernels OR DSA_DEVERR_* bits into it; dsa_check_device_errors
// reads and clears it.  Each device that loads the library has its own copy.
__device__ unsigned g_device_error_word;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_ctx_mutex;
DevCtx g_ctx[kMaxDevices];
bool g_ctx_ready[kMaxDevices];

std::atomic<long long> g_launches[DSA_KERNEL_KINDS];

thread_local char g_last_error[512];

dsa_status fail(dsa_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

dsa_status cuda_fail(cudaError_t e, const char* where) {
    return fail(DSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

}  // namespace

cudaError_t get_dev_ctx(DevCtx* ctx) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_ctx_mutex);
    if (!g_ctx_ready[dev]) {
        DevCtx c{};
        c.device = dev;
        e = cudaDeviceGetAttribute(&c.num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        int major = 0, minor = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (major != 10 || minor != 0) return cudaErrorNoKernelImageForDevice;
        void* addr = nullptr;
        e = cudaGetSymbolAddress(&addr, g_device_error_word);
        if (e != cudaSuccess) return e;
        c.err = static_cast<unsigned*>(addr);
        g_ctx[dev] = c;
        g_ctx_ready[dev] = true;
    }
    *ctx = g_ctx[dev];
    return cudaSuccess;
}

void count_launch(int kind) {
    if (kind >= 0 && kind < DSA_KERNEL_KINDS) g_launches[kind].fetch_add(1);
}

void clear_last_error() { g_last_error[0] = 0; }

dsa_status fail_with(dsa_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint64_t row_pitch_bytes, uint32_t box_rows, uint32_t box_cols) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {row_pitch_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Validation shared by the calls.
// Tracing: an NVTX range for the lifetime of the object when the library is built with
// -DDSA_NVTX=1 (build.py --nvtx), so that timelines show each layer and index window; an
// empty object otherwise.
struct TraceRange {
#if defined(DSA_NVTX) && DSA_NVTX
    explicit TraceRange(const char* fmt, ...) {
        char name[96];
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(name, sizeof name, fmt, ap);
        va_end(ap);
        nvtxRangePushA(name);
    }
    ~TraceRange() { nvtxRangePop(); }
#else
    explicit TraceRange(const char*, ...) {}
#endif
};

dsa_status check_stream_device(DevCtx* ctx) {
    cudaError_t e = get_dev_ctx(ctx);
    if (e == cudaErrorNoKernelImageForDevice)
        return fail(DSA_ERR_UNSUPPORTED, "this library is built for sm_100a (B200) only");
    if (e != cudaSuccess) return cuda_fail(e, "device query");
    return DSA_OK;
}

}  // namespace dsa

using namespace dsa;

extern "C" {

const char* dsa_status_string(int status) {
    switch (status) {
        case DSA_OK: return "DSA_OK";
        case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
        case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
        case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
        case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
        case DSA_ERR_DEVICE_CHECK: return "DSA_ERR_DEVICE_CHECK";
        default: return "DSA_ERR_UNKNOWN";
    }
}

const char* dsa_last_error(void) { return g_last_error; }

int dsa_version(void) { return (1 << 16) | 1; }

dsa_status dsa_indexer_scores(int dtype, int mode, const void* q_idx, const void* k_idx,
                              const float* w, int H_I, int D_I, int q_begin, int rows, int S,
                              const int* page_table, int max_pages, int page_size,
                              const int* seq_lens, float* scores, long long ld_scores,
                              dsa_stream_t stream) {
    g_last_error[0] = 0;
    if (!q_idx || !k_idx || !w || !scores) return fail(DSA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(scores))
        return fail(DSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (H_I <= 0 || D_I <= 0 || rows < 0 || q_begin < 0 || S <= 0)
        return fail(DSA_ERR_INVALID_ARG, "sizes must be positive (H_I=%d D_I=%d rows=%d S=%d)",
                    H_I, D_I, rows, S);
    if (ld_scores <= 0 || (ld_scores & 3))
        return fail(DSA_ERR_INVALID_ARG, "ld_scores must be a positive multiple of 4");
    if (dtype != DSA_F32 && dtype != DSA_BF16) return fail(DSA_ERR_INVALID_ARG, "bad dtype");
    if (mode != DSA_PREFILL && mode != DSA_DECODE) return fail(DSA_ERR_INVALID_ARG, "bad mode");
    if (rows == 0) return DSA_OK;
    DevCtx ctx;
    dsa_status st = check_stream_device(&ctx);
    if (st != DSA_OK) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (mode == DSA_PREFILL) {
        if (page_table || seq_lens)
            return fail(DSA_ERR_INVALID_ARG, "prefill takes no page_table / seq_lens");
        if ((long long)q_begin + rows > S)
            return fail(DSA_ERR_INVALID_ARG, "causal keys 0..q_begin+rows-1 exceed S=%d", S);
        if (ld_scores < (long long)q_begin + rows)
            return fail(DSA_ERR_INVALID_ARG, "ld_scores < q_begin + rows");
        if (dtype == DSA_F32) {
            if (H_I * D_I > 256 || (D_I & 3))
                return fail(DSA_ERR_UNSUPPORTED, "fp32 indexer needs H_I*D_I <= 256, D_I %% 4 == 0");
            e = launch_indexer_f32(static_cast<const float*>(q_idx),
                                   static_cast<const float*>(k_idx), w, H_I, D_I, q_begin, rows,
                                   scores, ld_scores, cs);
        } else {
            if (H_I != 16 || D_I != 64)
                return fail(DSA_ERR_UNSUPPORTED, "bf16 indexer supports H_I=16, D_I=64 only");
            e = launch_indexer_bf16_prefill(static_cast<const __nv_bfloat16*>(q_idx),
                                            static_cast<const __nv_bfloat16*>(k_idx), w,
                                            q_begin + rows, S, q_begin, rows, scores, ld_scores,
                                            cs, ctx);
        }
        return e == cudaSuccess ? DSA_OK : cuda_fail(e, "indexer launch");
    }
    // decode
    if (dtype != DSA_BF16) return fail(DSA_ERR_UNSUPPORTED, "decode indexer is bf16 only");
    if (H_I != 16 || D_I != 64)
        return fail(DSA_ERR_UNSUPPORTED, "bf16 indexer supports H_I=16, D_I=64 only");
    if (!page_table || !seq_lens) return fail(DSA_ERR_INVALID_ARG, "decode needs page_table and seq_lens");
    if (q_begin != 0) return fail(DSA_ERR_INVALID_ARG, "decode requires q_begin = 0");
    if (page_size != 16 && page_size != 32 && page_size != 64 && page_size != 128)
        return fail(DSA_ERR_UNSUPPORTED, "page_size must be 16, 32, 64 or 128");
    if (max_pages <= 0) return fail(DSA_ERR_INVALID_ARG, "max_pages must be positive");
    if (S % page_size) return fail(DSA_ERR_INVALID_ARG, "S must be num_pages * page_size");
    const long long cap = (long long)max_pages * page_size;
    const int max_len = (int)(cap < ld_scores ? cap : ld_scores);
    e = launch_indexer_bf16_decode(static_cast<const __nv_bfloat16*>(q_idx),
                                   static_cast<const __nv_bfloat16*>(k_idx), w, rows, S,
                                   page_table, max_pages, page_size, seq_lens, max_len, scores,
                                   ld_scores, cs, ctx);
    return e == cudaSuccess ? DSA_OK : cuda_fail(e, "decode indexer launch");
}

dsa_status dsa_topk_select(const float* scores, long long ld_scores, int rows, int q_begin,
                           const int* row_len, int max_len, int k, int* idx, long long ld_idx,
                           dsa_stream_t stream) {
    g_last_error[0] = 0;
    if (!scores || !idx) return fail(DSA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(scores) || !aligned16(idx) || (row_len && !aligned16(row_len)))
        return fail(DSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (rows < 0 || q_begin < 0) return fail(DSA_ERR_INVALID_ARG, "negative rows / q_begin");
    if (k < 1 || k > 4096) return fail(DSA_ERR_UNSUPPORTED, "k must be in [1, 4096]");
    if (ld_idx < k) return fail(DSA_ERR_INVALID_ARG, "ld_idx < k");
    if (max_len < 1 || max_len > 262144)
        return fail(DSA_ERR_UNSUPPORTED, "max_len must be in [1, 262144]");
    if (max_len > ld_scores) return fail(DSA_ERR_INVALID_ARG, "max_len > ld_scores");
    if (ld_scores & 3)
        return fail(DSA_ERR_INVALID_ARG, "ld_scores must be a multiple of 4 (16-byte rows)");
    if (!row_len && (long long)q_begin + rows > max_len)
        return fail(DSA_ERR_INVALID_ARG, "causal rows need max_len >= q_begin + rows");
    if (rows == 0) return DSA_OK;
    DevCtx ctx;
    dsa_status st = check_stream_device(&ctx);
    if (st != DSA_OK) return st;
    cudaError_t e = launch_topk(scores, ld_scores, rows, q_begin, row_len, max_len, k, idx, ld_idx,
                                reinterpret_cast<cudaStream_t>(stream), ctx);
    return e == cudaSuccess ? DSA_OK : cuda_fail(e, "top-k launch");
}

size_t dsa_sparse_mla_workspace_size(int mode, int num_q, int H, int D_v, int k_sel) {
    if (mode != DSA_DECODE || num_q <= 0 || H <= 0 || D_v <= 0 || k_sel <= 0) return 0;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int splits = mla_decode_splits(num_q, k_sel, sms);
    return (size_t)num_q * splits * H * ((size_t)D_v + 1) * sizeof(float);
}

namespace {

// The absorbed-MLA path behind dsa_sparse_mla_fwd (bf16 cache) and dsa_sparse_mla_fp8_fwd.
dsa_status mla_absorbed(bool fp8, float kv_scale, int mode, int num_q, int H, int D_qk, int D_v,
                        float scale, const void* q, const void* kv, long long kv_rows,
                        const int* page_table, int max_pages, int page_size,
                        const int* seq_lens, const int* idx, int k_sel, long long ld_idx,
                        void* out, float* lse, void* workspace, size_t workspace_bytes,
                        cudaStream_t cs, const DevCtx& ctx) {
    if (H != 16 || D_qk != 576 || D_v != 512)
        return fail(DSA_ERR_UNSUPPORTED,
                    "MLA path is absorbed MLA: H=16, one shared 576-dim latent, D_v=512");
    if (k_sel > 2048 || (k_sel & 3) || (ld_idx & 3))
        return fail(DSA_ERR_UNSUPPORTED, "MLA path: k_sel <= 2048 and k_sel, ld_idx multiples of 4");
    cudaError_t e;
    if (mode == DSA_PREFILL) {
        if (page_table || seq_lens) return fail(DSA_ERR_INVALID_ARG, "prefill takes no pages");
        e = launch_sparse_mla_mma(static_cast<const __nv_bfloat16*>(q), kv, fp8, kv_scale, kv_rows,
                                  nullptr, 0, 0, nullptr, idx, k_sel, ld_idx, num_q, scale, 1,
                                  static_cast<__nv_bfloat16*>(out), lse, nullptr, nullptr, cs, ctx);
        return e == cudaSuccess ? DSA_OK : cuda_fail(e, "attention launch");
    }
    if (!page_table || !seq_lens) return fail(DSA_ERR_INVALID_ARG, "decode needs page_table and seq_lens");
    if (page_size <= 0 || max_pages <= 0 || kv_rows % page_size)
        return fail(DSA_ERR_INVALID_ARG, "kv_rows must be num_pages * page_size");
    const int splits = mla_decode_splits(num_q, k_sel, ctx.num_sms);
    const size_t need = (size_t)num_q * splits * H * ((size_t)D_v + 1) * sizeof(float);
    if (!workspace || workspace_bytes < need)
        return fail(DSA_ERR_WORKSPACE, "decode needs %zu workspace bytes, got %zu", need,
                    workspace_bytes);
    if (!aligned16(workspace)) return fail(DSA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    float* o_part = static_cast<float*>(workspace);
    float* lse_part = o_part + (size_t)num_q * splits * H * D_v;
    e = launch_sparse_mla_mma(static_cast<const __nv_bfloat16*>(q), kv, fp8, kv_scale, kv_rows,
                              page_table, max_pages, page_size, seq_lens, idx, k_sel, ld_idx,
                              num_q, scale, splits, nullptr, nullptr, o_part, lse_part, cs, ctx);
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    e = launch_mla_combine(o_part, lse_part, num_q, splits, static_cast<__nv_bfloat16*>(out), lse,
                           cs);
    return e == cudaSuccess ? DSA_OK : cuda_fail(e, "combine launch");
}

}  // namespace

dsa_status dsa_sparse_mla_fwd(int dtype, int mode, int num_q, int H, int num_kv_heads,
                              int D_qk, int D_v, float scale, const void* q, const void* kv,
                              const void* v, long long kv_rows, const int* page_table,
                              int max_pages, int page_size, const int* seq_lens,
                              const int* idx, int k_sel, long long ld_idx, void* out,
                              float* lse, void* workspace, size_t workspace_bytes,
                              dsa_stream_t stream) {
    g_last_error[0] = 0;
    if (!q || !kv || !idx || !out) return fail(DSA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(q) || !aligned16(kv) || !aligned16(idx) || !aligned16(out) ||
        (v && !aligned16(v)) || (lse && !aligned16(lse)))
        return fail(DSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (num_q < 0 || H <= 0 || num_kv_heads <= 0 || D_qk <= 0 || D_v <= 0 || kv_rows <= 0 ||
        k_sel <= 0 || ld_idx < k_sel)
        return fail(DSA_ERR_INVALID_ARG, "bad sizes");
    if (!(scale > 0.f) || scale != scale) return fail(DSA_ERR_INVALID_ARG, "scale must be > 0");
    if (mode != DSA_PREFILL && mode != DSA_DECODE) return fail(DSA_ERR_INVALID_ARG, "bad mode");
    if (dtype == DSA_FP8_E4M3)
        return fail(DSA_ERR_INVALID_ARG, "an fp8 cache needs its scale: use dsa_sparse_mla_fp8_fwd");
    if (dtype != DSA_BF16 && dtype != DSA_F32) return fail(DSA_ERR_INVALID_ARG, "bad dtype");
    if (num_q == 0) return DSA_OK;
    DevCtx ctx;
    dsa_status st = check_stream_device(&ctx);
    if (st != DSA_OK) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (dtype == DSA_F32) {
        if (mode != DSA_PREFILL) return fail(DSA_ERR_UNSUPPORTED, "fp32 attention is prefill only");
        if (!v || num_kv_heads != H || D_qk != D_v || D_qk > 64 || H > 16)
            return fail(DSA_ERR_UNSUPPORTED, "fp32 path: MHA with v, D <= 64, H <= 16");
        if (page_table || seq_lens) return fail(DSA_ERR_INVALID_ARG, "prefill takes no pages");
        cudaError_t e = launch_sparse_mha_f32(static_cast<const float*>(q), static_cast<const float*>(kv),
                                  static_cast<const float*>(v), num_q, H, D_qk, scale, kv_rows,
                                  idx, k_sel, ld_idx, static_cast<float*>(out), lse, cs, ctx);
        return e == cudaSuccess ? DSA_OK : cuda_fail(e, "attention launch");
    }
    if (num_kv_heads != 1 || v != nullptr)
        return fail(DSA_ERR_UNSUPPORTED, "bf16 path is absorbed MLA: one shared latent, v=NULL");
    return mla_absorbed(false, 1.f, mode, num_q, H, D_qk, D_v, scale, q, kv, kv_rows, page_table,
                        max_pages, page_size, seq_lens, idx, k_sel, ld_idx, out, lse, workspace,
                        workspace_bytes, cs, ctx);
}

dsa_status dsa_sparse_mla_fp8_fwd(int mode, int num_q, int H, int D_qk, int D_v, float scale,
                                  float kv_scale, const void* q, const void* kv,
                                  long long kv_rows, const int* page_table, int max_pages,
                                  int page_size, const int* seq_lens, const int* idx,
                                  int k_sel, long long ld_idx, void* out, float* lse,
                                  void* workspace, size_t workspace_bytes,
                                  dsa_stream_t stream) {
    g_last_error[0] = 0;
    if (!q || !kv || !idx || !out) return fail(DSA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(q) || !aligned16(kv) || !aligned16(idx) || !aligned16(out) ||
        (lse && !aligned16(lse)))
        return fail(DSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (num_q < 0 || H <= 0 || D_qk <= 0 || D_v <= 0 || kv_rows <= 0 || k_sel <= 0 ||
        ld_idx < k_sel)
        return fail(DSA_ERR_INVALID_ARG, "bad sizes");
    if (!(scale > 0.f) || scale != scale) return fail(DSA_ERR_INVALID_ARG, "scale must be > 0");
    if (!(kv_scale > 0.f) || !std::isfinite(kv_scale))
        return fail(DSA_ERR_INVALID_ARG, "kv_scale must be finite and > 0");
    if (mode != DSA_PREFILL && mode != DSA_DECODE) return fail(DSA_ERR_INVALID_ARG, "bad mode");
    if (num_q == 0) return DSA_OK;
    DevCtx ctx;
    dsa_status st = check_stream_device(&ctx);
    if (st != DSA_OK) return st;
    return mla_absorbed(true, kv_scale, mode, num_q, H, D_qk, D_v, scale, q, kv, kv_rows,
                        page_table, max_pages, page_size, seq_lens, idx, k_sel, ld_idx, out, lse,
                        workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream), ctx);
}

dsa_status dsa_latent_quantize_fp8(const void* src, long long n, float kv_scale, void* dst,
                                   dsa_stream_t stream) {
    g_last_error[0] = 0;
    if (n < 0) return fail(DSA_ERR_INVALID_ARG, "n must be >= 0");
    if (n == 0) return DSA_OK;
    if (!src || !dst) return fail(DSA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(src) || !aligned16(dst))
        return fail(DSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (!(kv_scale > 0.f) || !std::isfinite(kv_scale))
        return fail(DSA_ERR_INVALID_ARG, "kv_scale must be finite and > 0");
    DevCtx ctx;
    dsa_status st = check_stream_device(&ctx);
    if (st != DSA_OK) return st;
    cudaError_t e = launch_latent_quantize_fp8(static_cast<const __nv_bfloat16*>(src), n, kv_scale,
                                               static_cast<uint8_t*>(dst),
                                               reinterpret_cast<cudaStream_t>(stream), ctx);
    return e == cudaSuccess ? DSA_OK : cuda_fail(e, "quantize launch");
}

size_t dsa_index_varlen_workspace_size(int max_seq_len, int rows_window) {
    if (max_seq_len <= 0) return 0;
    const long long ld = ((long long)max_seq_len + 3) / 4 * 4;
    long long rw = rows_window > 0 ? rows_window : dsa_layer_stack_workspace_size(max_seq_len, 0) / (ld * 4);
    if (rw > max_seq_len) rw = max_seq_len;
    if (rw < 1) rw = 1;
    return (size_t)(rw * ld * 4);
}

dsa_status dsa_index_varlen(const void* q_idx, const void* k_idx, const float* w, int H_I, int D_I,
                            int num_tokens, int num_seqs, const int* seq_start, const int* seq_len,
                            int k, int* idx, long long ld_idx, void* workspace,
                            size_t workspace_bytes, dsa_stream_t stream) {
    g_last_error[0] = 0;
    if (num_seqs < 0 || num_tokens < 0) return fail(DSA_ERR_INVALID_ARG, "negative sizes");
    if (num_seqs == 0) return DSA_OK;
    if (!seq_start || !seq_len) return fail(DSA_ERR_INVALID_ARG, "seq_start / seq_len missing");
    if (!q_idx || !k_idx || !w || !idx) return fail(DSA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(idx))
        return fail(DSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (H_I != 16 || D_I != 64)
        return fail(DSA_ERR_UNSUPPORTED, "bf16 indexer supports H_I=16, D_I=64 only");
    if (k < 1 || k > 4096) return fail(DSA_ERR_UNSUPPORTED, "k must be in [1, 4096]");
    if (ld_idx < k) return fail(DSA_ERR_INVALID_ARG, "ld_idx < k");
    // the sequences: inside [0, num_tokens), in increasing order, not overlapping
    int max_len = 0;
    long long prev_end = 0;
    for (int b = 0; b < num_seqs; ++b) {
        const long long s0 = seq_start[b], L = seq_len[b];
        if (s0 < 0 || L < 0 || s0 + L > num_tokens)
            return fail(DSA_ERR_INVALID_ARG, "sequence %d [%lld, %lld) outside [0, %d)", b, s0,
                        s0 + L, num_tokens);
        if (s0 < prev_end)
            return fail(DSA_ERR_INVALID_ARG, "sequence %d starts before the end of the previous one", b);
        if (L > 262144) return fail(DSA_ERR_UNSUPPORTED, "sequences of at most 262144 tokens");
        prev_end = s0 + L;
        if (L > max_len) max_len = (int)L;
    }
    if (max_len == 0) return DSA_OK;
    const long long ld = ((long long)max_len + 3) / 4 * 4;
    if (!workspace || !aligned16(workspace) || workspace_bytes < (size_t)(ld * 4))
        return fail(DSA_ERR_WORKSPACE, "workspace must hold at least one row of %lld scores", ld);
    const long long rw = (long long)(workspace_bytes / (ld * 4));
    DevCtx ctx;
    dsa_status st = check_stream_device(&ctx);
    if (st != DSA_OK) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    float* scores = static_cast<float*>(workspace);
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q_idx);
    const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(k_idx);
    for (int b = 0; b < num_seqs; ++b) {
        const int s0 = seq_start[b], L = seq_len[b];
        // sequence b alone: its tokens are rows 0..L-1 of shifted tensors, and the top-k
        // adds s0 to the selected positions so that they name packed rows
        const __nv_bfloat16* qs = qb + (size_t)s0 * H_I * D_I;
        const __nv_bfloat16* ks = kb + (size_t)s0 * D_I;
        const float* ws = w + (size_t)s0 * H_I;
        for (long long q0 = 0; q0 < L; q0 += rw) {
            const int rows = (int)(L - q0 < rw ? L - q0 : rw);
            cudaError_t e;
            if (L > k) {  // otherwise every row selects all of its keys without reading scores
                e = launch_indexer_bf16_prefill(qs, ks, ws, (int)q0 + rows, L, (int)q0, rows,
                                                scores, ld, cs, ctx);
                if (e != cudaSuccess) return cuda_fail(e, "indexer launch");
            }
            e = launch_topk(scores, ld, rows, (int)q0, nullptr, L, k,
                            idx + ((long long)s0 + q0) * ld_idx, ld_idx, cs, ctx, nullptr, s0);
            if (e != cudaSuccess) return cuda_fail(e, "top-k launch");
        }
    }
    return DSA_OK;
}

dsa_status dsa_selftest_wait_timeout(int* gave_up, dsa_stream_t stream) {
    g_last_error[0] = 0;
    if (!gave_up || !aligned16(gave_up)) return fail(DSA_ERR_INVALID_ARG, "gave_up must be a 16-byte aligned device int");
    DevCtx ctx;
    dsa_status st = check_stream_device(&ctx);
    if (st != DSA_OK) return st;
    cudaError_t e = launch_wait_timeout_selftest(gave_up, reinterpret_cast<cudaStream_t>(stream), ctx);
    return e == cudaSuccess ? DSA_OK : cuda_fail(e, "self-test launch");
}

size_t dsa_layer_stack_workspace_size(int T, int rows_window) {
    if (T <= 0) return 0;
    const long long ld = ((long long)T + 3) / 4 * 4;
    long long rw = rows_window;
    if (rw <= 0) {
        // default: about 4 GB of scores per window.  Wider windows give the indexer and
        // top-k launches more rows per launch and fewer launch tails: at T = 65536 this is
        // 16384 rows, and the index phase measured 10.42 / 10.12 / 9.83 / 9.76 ms with
        // 4096 / 8192 / 16384 / 32768-row windows.
        rw = (4096ll << 20) / (ld * 4);
        if (rw < 128) rw = 128;
    }
    if (rw > T) rw = T;
    return (size_t)(rw * ld * 4);
}

// ---- filtered index selection (dsa_index_select) ----
namespace {

constexpr int kDenseRows = 8192;      // rows with at most this many keys take the dense path
constexpr int kListCap = 512;         // candidates per (row, 4096-key chunk, lane quadrant)

struct SelectLayout {
    int sample_stride;  // one 128-key tile in sample_stride is scored for the thresholds
    long long ld_sample, ld_dense, nchunk_max;
    size_t off_sample, off_tau, off_fb_row, off_fb_any, off_ccount, off_cand, off_dense;
    size_t total;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

SelectLayout select_layout(long long rows, long long S) {
    SelectLayout L{};
    // at most topk_sample_max() sampled keys per row: a stride of at least 16 tiles, more
    // for long rows
    const long long tiles = (S + 127) / 128;
    const long long max_tiles = topk_sample_max() / 128;
    L.sample_stride = (int)std::max(16LL, (tiles + max_tiles - 1) / max_tiles);
    L.ld_sample = topk_sample_max();
    L.ld_dense = (S + 3) / 4 * 4;
    L.nchunk_max = (S + 4095) / 4096;
    const long long lists = rows * L.nchunk_max * 4;
    size_t o = 0;
    L.off_sample = o; o = align256(o + (size_t)(rows * L.ld_sample) * 4);
    L.off_tau = o;    o = align256(o + (size_t)rows * 4);
    L.off_fb_row = o; o = align256(o + (size_t)rows * 4);
    L.off_fb_any = o; o = align256(o + 4);
    L.off_ccount = o; o = align256(o + (size_t)lists * 4);
    L.off_cand = o;   o = align256(o + (size_t)lists * kListCap * 8);
    L.off_dense = o;  o = align256(o + (size_t)(rows * L.ld_dense) * 4);
    L.total = o;
    return L;
}

}  // namespace

size_t dsa_index_select_workspace_size(int rows_window, int S) {
    if (rows_window <= 0 || S <= 0) return 0;
    return select_layout(rows_window, S).total;
}

dsa_status dsa_index_select(const void* q_idx, const void* k_idx, const float* w, int H_I, int D_I,
                            int q_begin, int rows, int S, int k, int* idx, long long ld_idx,
                            void* workspace, size_t ws_bytes, dsa_stream_t stream) {
    g_last_error[0] = 0;
    if (!q_idx || !k_idx || !w || !idx) return fail(DSA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(idx))
        return fail(DSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (rows < 0 || q_begin < 0 || S <= 0) return fail(DSA_ERR_INVALID_ARG, "bad rows / q_begin / S");
    if (H_I != 16 || D_I != 64)
        return fail(DSA_ERR_UNSUPPORTED, "bf16 indexer supports H_I=16, D_I=64 only");
    if (k < 1 || k > 4096) return fail(DSA_ERR_UNSUPPORTED, "k must be in [1, 4096]");
    if (ld_idx < k || (ld_idx & 3)) return fail(DSA_ERR_INVALID_ARG, "ld_idx must be >= k and a multiple of 4");
    if ((long long)q_begin + rows > S)
        return fail(DSA_ERR_INVALID_ARG, "causal keys 0..q_begin+rows-1 exceed S=%d", S);
    if ((long long)S > 262144) return fail(DSA_ERR_UNSUPPORTED, "S must be <= 262144");
    if (rows == 0) return DSA_OK;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return fail(DSA_ERR_INVALID_ARG, "workspace must be non-null and 256-byte aligned");
    // the largest window (a multiple of 16 rows, or all rows) whose scratch fits
    long long rw = rows;
    if (select_layout(rw, S).total > ws_bytes) {
        long long lo = 0, hi = rows;
        while (lo < hi) {
            const long long mid = (lo + hi + 1) / 2;
            if (select_layout(mid, S).total <= ws_bytes) lo = mid; else hi = mid - 1;
        }
        rw = lo / 16 * 16;
        if (rw < 16) return fail(DSA_ERR_WORKSPACE, "workspace holds fewer than 16 rows");
    }
    DevCtx ctx;
    dsa_status st = check_stream_device(&ctx);
    if (st != DSA_OK) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const SelectLayout L = select_layout(rw, S);
    char* base = static_cast<char*>(workspace);
    float* sample = reinterpret_cast<float*>(base + L.off_sample);
    uint32_t* tau = reinterpret_cast<uint32_t*>(base + L.off_tau);
    int* fb_row = reinterpret_cast<int*>(base + L.off_fb_row);
    int* fb_any = reinterpret_cast<int*>(base + L.off_fb_any);
    uint32_t* ccount = reinterpret_cast<uint32_t*>(base + L.off_ccount);
    uint2* cand = reinterpret_cast<uint2*>(base + L.off_cand);
    float* dense = reinterpret_cast<float*>(base + L.off_dense);
    const auto* qi = static_cast<const __nv_bfloat16*>(q_idx);
    const auto* ki = static_cast<const __nv_bfloat16*>(k_idx);
    const int T = q_begin + rows;  // query rows the tensor map of q_idx covers
    // windows of at most rw rows that do not straddle the dense / filtered boundary
    for (long long q0 = q_begin; q0 < T;) {
        long long q1 = q0 + rw < T ? q0 + rw : T;
        if (q0 < kDenseRows && q1 > kDenseRows) q1 = kDenseRows;
        const int nr = (int)(q1 - q0);
        int* out = idx + (q0 - q_begin) * ld_idx;
        cudaError_t e;
        if (q1 <= kDenseRows) {
            // short rows: dense scores and the dense top-k
            e = launch_indexer_bf16_prefill(qi, ki, w, T, S, (int)q0, nr, dense, L.ld_dense, cs,
                                            ctx);
            if (e == cudaSuccess)
                e = launch_topk(dense, L.ld_dense, nr, (int)q0, nullptr, (int)q1, k, out, ld_idx,
                                cs, ctx);
        } else {
            // 1. scores of one key tile in sample_stride; 2. per-row thresholds
            e = launch_indexer_bf16_sample(qi, ki, w, T, S, (int)q0, nr, L.sample_stride, sample,
                                           L.ld_sample, cs, ctx);
            if (e == cudaSuccess)
                e = launch_topk_threshold(sample, L.ld_sample, (int)q0, nr, L.sample_stride, k,
                                          tau, fb_any, cs);
            // 3. every score, keeping only the keys at or above the thresholds
            if (e == cudaSuccess)
                e = launch_indexer_bf16_filter(qi, ki, w, T, S, (int)q0, nr, tau, cand, ccount,
                                               kListCap, (int)L.nchunk_max, cs, ctx);
            // 4. exact top-k from the candidates
            if (e == cudaSuccess)
                e = launch_topk_candidates(cand, ccount, kListCap, (int)L.nchunk_max, (int)q0, nr,
                                           (int)q1, k, out, ld_idx, fb_row, fb_any, cs);
            // 5. rows the candidates could not settle: dense scores of the window and the
            //    dense top-k of those rows (both return at once when no row was flagged)
            if (e == cudaSuccess)
                e = launch_indexer_bf16_prefill(qi, ki, w, T, S, (int)q0, nr, dense, L.ld_dense,
                                                cs, ctx, fb_any);
            if (e == cudaSuccess)
                e = launch_topk(dense, L.ld_dense, nr, (int)q0, nullptr, (int)q1, k, out, ld_idx,
                                cs, ctx, fb_row);
        }
        if (e != cudaSuccess) return cuda_fail(e, "index selection launch");
        q0 = q1;
    }
    return DSA_OK;
}

dsa_status dsa_layer_stack(const char* pattern, int num_layers, int T, int topk, int H_I,
                           int D_I, int H, int D_qk, int D_v, float scale,
                           const void* const* q_idx, const void* const* k_idx,
                           const float* const* w, const void* const* q, const void* const* kv,
                           void* const* out, float* const* lse, int* idx_buf, void* workspace,
                           size_t workspace_bytes, dsa_stream_t stream) {
    g_last_error[0] = 0;
    if (!pattern || num_layers <= 0) return fail(DSA_ERR_INVALID_ARG, "empty pattern");
    if ((int)strnlen(pattern, (size_t)num_layers + 1) != num_layers)
        return fail(DSA_ERR_INVALID_ARG, "pattern length != num_layers");
    if (pattern[0] != 'F') return fail(DSA_ERR_INVALID_ARG, "pattern must start with 'F'");
    for (int l = 0; l < num_layers; ++l)
        if (pattern[l] != 'F' && pattern[l] != 'S')
            return fail(DSA_ERR_INVALID_ARG, "pattern character %d is not F or S", l);
    if (T <= 0 || topk < 1 || topk > 4096) return fail(DSA_ERR_INVALID_ARG, "bad T / topk");
    if (H_I != 16 || D_I != 64 || H != 16 || D_qk != 576 || D_v != 512)
        return fail(DSA_ERR_UNSUPPORTED, "layer stack supports the bf16 MLA shapes only");
    if (!q || !kv || !out || !idx_buf || !q_idx || !k_idx || !w)
        return fail(DSA_ERR_INVALID_ARG, "null array");
    for (int l = 0; l < num_layers; ++l) {
        if (!q[l] || !kv[l] || !out[l]) return fail(DSA_ERR_INVALID_ARG, "layer %d: null q/kv/out", l);
        if (pattern[l] == 'F' && (!q_idx[l] || !k_idx[l] || !w[l]))
            return fail(DSA_ERR_INVALID_ARG, "F layer %d: null indexer input", l);
    }
    const long long ld = ((long long)T + 3) / 4 * 4;
    long long rw = workspace ? (long long)(workspace_bytes / (size_t)(ld * 4)) : 0;
    if (rw < 1 || (rw < 16 && rw < T))
        return fail(DSA_ERR_WORKSPACE, "workspace holds fewer than 16 rows of scores");
    if (!aligned16(workspace)) return fail(DSA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    if (rw > T) rw = T;
    if (rw > 16) rw = rw / 16 * 16;  // whole 16-query blocks per window
    float* scores = static_cast<float*>(workspace);
    for (int l = 0; l < num_layers; ++l) {
        TraceRange layer_range("dsa layer %d (%c)", l, pattern[l]);
        if (pattern[l] == 'F') {
            for (long long q0 = 0; q0 < T; q0 += rw) {
                const int rows = (int)((T - q0) < rw ? (T - q0) : rw);
                TraceRange window_range("dsa index window %lld+%d", q0, rows);
                dsa_status st = dsa_indexer_scores(DSA_BF16, DSA_PREFILL, q_idx[l], k_idx[l], w[l],
                                                   H_I, D_I, (int)q0, rows, T, nullptr, 0, 0,
                                                   nullptr, scores, ld, stream);
                if (st != DSA_OK) return st;
                st = dsa_topk_select(scores, ld, rows, (int)q0, nullptr, (int)(q0 + rows), topk,
                                     idx_buf + q0 * topk, topk, stream);
                if (st != DSA_OK) return st;
            }
        }
        dsa_status st = dsa_sparse_mla_fwd(DSA_BF16, DSA_PREFILL, T, H, 1, D_qk, D_v, scale, q[l],
                                           kv[l], nullptr, T, nullptr, 0, 0, nullptr, idx_buf,
                                           topk, topk, out[l], lse ? lse[l] : nullptr, nullptr, 0,
                                           stream);
        if (st != DSA_OK) return st;
    }
    return DSA_OK;
}

dsa_status dsa_pattern_from_freq(int freq, int num_layers, char* out, int out_len) {
    g_last_error[0] = 0;
    if (freq < 1 || num_layers < 1) return fail(DSA_ERR_INVALID_ARG, "freq and num_layers must be >= 1");
    if (!out || out_len <= num_layers) return fail(DSA_ERR_INVALID_ARG, "output buffer too small");
    for (int i = 0; i < num_layers; ++i) out[i] = (i % freq == 0) ? 'F' : 'S';
    out[num_layers] = 0;
    return DSA_OK;
}

dsa_status dsa_check_device_errors(dsa_stream_t stream, unsigned* error_bits) {
    g_last_error[0] = 0;
    DevCtx ctx;
    dsa_status st = check_stream_device(&ctx);
    if (st != DSA_OK) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    unsigned bits = 0;
    cudaError_t e = cudaMemcpyAsync(&bits, ctx.err, sizeof(unsigned), cudaMemcpyDeviceToHost, cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e == cudaSuccess) e = cudaMemsetAsync(ctx.err, 0, sizeof(unsigned), cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    if (error_bits) *error_bits = bits;
    return bits ? fail(DSA_ERR_DEVICE_CHECK, "device error bits 0x%x", bits) : DSA_OK;
}

long long dsa_launch_count(int kind) {
    if (kind < 0 || kind >= DSA_KERNEL_KINDS) return -1;
    return g_launches[kind].load();
}

void dsa_reset_launch_counts(void) {
    for (int i = 0; i < DSA_KERNEL_KINDS; ++i) g_launches[i].store(0);
}

}  // extern "C"
