// noalloc.cu -- decode sparse MLA whose scratch memory is owned by the library.
//
// Some callers cannot allocate device memory at the point where they decode: code
// running under an allocator that must not grow (a memory pool sized at start-up, a
// serving loop that forbids allocation on its hot path) or a host that links this
// library without a device allocator of its own.  dsa_sparse_mla_fwd's decode path
// needs a workspace for the per-split partial outputs; this entry point keeps those
// partials in a fixed file-scope device array instead, so the caller passes only its
// inputs and outputs and nothing is allocated (no cudaMalloc / cudaFree, no allocating
// library routine).
//
// The array is kNoAllocScratchBytes (16 MiB) on every GPU that loads the library and
// stays there until the process exits.  In host code `g_decode_scratch` only names a
// host-side stand-in, so its device address is looked up with cudaGetSymbolAddress once
// per device, with that device current, on the first call made on that device.
#include <mutex>

#include "dsa_common.cuh"
#include "launch.h"

namespace dsa {
namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;
// One (sequence, split) unit needs 16 heads x (512 outputs + 1 log-sum-exp) fp32.
constexpr size_t kUnitBytes = 16u * (512u + 1u) * sizeof(float);
constexpr int kMaxUnits = (int)(kNoAllocScratchBytes / kUnitBytes);

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDev = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDev];

// Device address of this device's scratch array (looked up once per device).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" dsa_status dsa_sparse_mla_decode_noalloc(
    int num_q, int H, int D_qk, int D_v, float scale, const void* q, const void* kv,
    long long kv_rows, const int* page_table, int max_pages, int page_size,
    const int* seq_lens, const int* idx, int k_sel, long long ld_idx, void* out, float* lse,
    dsa_stream_t stream) {
    clear_last_error();
    auto aligned = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!q || !kv || !idx || !out || !page_table || !seq_lens)
        return fail_with(DSA_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned(q) || !aligned(kv) || !aligned(idx) || !aligned(out) || (lse && !aligned(lse)))
        return fail_with(DSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (num_q < 0 || kv_rows <= 0 || k_sel <= 0 || ld_idx < k_sel || page_size <= 0 ||
        max_pages <= 0 || kv_rows % page_size || !(scale > 0.f))
        return fail_with(DSA_ERR_INVALID_ARG, "bad sizes or scale");
    if (H != 16 || D_qk != 576 || D_v != 512 || k_sel > 2048 || (k_sel & 3) || (ld_idx & 3))
        return fail_with(DSA_ERR_UNSUPPORTED,
                         "absorbed MLA only: H=16, 576/512, k_sel <= 2048, multiples of 4");
    if (num_q == 0) return DSA_OK;
    if (num_q > kMaxUnits)  // even one split per sequence would not fit the array
        return fail_with(DSA_ERR_UNSUPPORTED, "at most %d sequences per call, got %d", kMaxUnits,
                         num_q);
    DevCtx ctx;
    cudaError_t e = get_dev_ctx(&ctx);
    if (e == cudaErrorNoKernelImageForDevice)
        return fail_with(DSA_ERR_UNSUPPORTED, "this library is built for sm_100a (B200) only");
    if (e != cudaSuccess) return fail_with(DSA_ERR_CUDA, "device query: %s", cudaGetErrorString(e));
    void* scratch = nullptr;
    e = scratch_address(&scratch);
    if (e != cudaSuccess)
        return fail_with(DSA_ERR_CUDA, "scratch array address: %s", cudaGetErrorString(e));
    // as many splits as the usual path would take, capped by what the array holds (a
    // trailing split left without keys writes a zero partial with log-sum-exp -inf, which
    // the merge ignores)
    int splits = mla_decode_splits(num_q, k_sel, ctx.num_sms);
    if (splits > kMaxUnits / num_q) splits = kMaxUnits / num_q;
    float* o_part = static_cast<float*>(scratch);
    float* lse_part = o_part + (size_t)num_q * splits * 16 * 512;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    // every (sequence, split) unit overwrites its partial output and log-sum-exp, so the
    // array needs no clearing between calls
    e = launch_sparse_mla_mma(static_cast<const __nv_bfloat16*>(q), kv, false, 1.f, kv_rows, page_table,
                               max_pages, page_size, seq_lens, idx, k_sel, ld_idx, num_q, scale,
                               splits, nullptr, nullptr, o_part, lse_part, cs, ctx);
    if (e != cudaSuccess) return fail_with(DSA_ERR_CUDA, "attention launch: %s", cudaGetErrorString(e));
    e = launch_mla_combine(o_part, lse_part, num_q, splits, static_cast<__nv_bfloat16*>(out), lse,
                           cs);
    if (e != cudaSuccess) return fail_with(DSA_ERR_CUDA, "combine launch: %s", cudaGetErrorString(e));
    return DSA_OK;
}
