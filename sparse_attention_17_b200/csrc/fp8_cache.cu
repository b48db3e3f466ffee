// fp8_cache.cu -- the write side of the fp8 latent cache: bf16 latent rows to E4M3 codes.
//
// DeepSeek-V2-Lite-Chat SIQ card (what is quantized, KV-cache bullet): the MLA KV cache
// can be kept in fp8, 576 bytes per token.  Encoding read here: E4M3 of the OCP 8-bit
// floating-point format with one fp32 scale per cache tensor, value = kv_scale * code.
//
//   code[i] = E4M3(src[i] / kv_scale)
//
// The quotient is the fp32 IEEE division (round to nearest); the conversion rounds to the
// nearest code, ties to even, and saturates finite magnitudes above 448 to 448.  The
// kernel streams 16 bytes in and 8 bytes out per thread and step: it is HBM-bound.
#include <cuda_fp8.h>

#include "dsa_common.cuh"
#include "launch.h"

namespace dsa {

namespace {

__device__ __forceinline__ uint32_t quantize_pair(uint32_t bf2, float kv_scale) {
    const float a = __fdiv_rn(__uint_as_float(bf2 << 16), kv_scale);
    const float b = __fdiv_rn(__uint_as_float(bf2 & 0xffff0000u), kv_scale);
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

__global__ void latent_quantize_fp8_kernel(const __nv_bfloat16* __restrict__ src, long long n,
                                           float kv_scale, uint8_t* __restrict__ dst) {
    const long long stride = (long long)gridDim.x * blockDim.x * 8;
    for (long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 8; i < n; i += stride) {
        if (i + 8 <= n) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + i));
            const uint32_t c0 = quantize_pair(v.x, kv_scale) | (quantize_pair(v.y, kv_scale) << 16);
            const uint32_t c1 = quantize_pair(v.z, kv_scale) | (quantize_pair(v.w, kv_scale) << 16);
            *reinterpret_cast<uint2*>(dst + i) = make_uint2(c0, c1);
        } else {
            const uint16_t* s16 = reinterpret_cast<const uint16_t*>(src);
            for (long long j = i; j < n; ++j)
                dst[j] = (uint8_t)(quantize_pair((uint32_t)s16[j], kv_scale) & 0xffu);
        }
    }
}

}  // namespace

cudaError_t launch_latent_quantize_fp8(const __nv_bfloat16* src, long long n, float kv_scale,
                                       uint8_t* dst, cudaStream_t stream, const DevCtx& ctx) {
    constexpr int kBlock = 256;
    const long long groups = (n + 7) / 8;
    long long blocks = (groups + kBlock - 1) / kBlock;
    const long long cap = 8ll * ctx.num_sms;  // a few resident CTAs per SM, grid-stride beyond
    if (blocks > cap) blocks = cap;
    latent_quantize_fp8_kernel<<<(int)blocks, kBlock, 0, stream>>>(src, n, kv_scale, dst);
    count_launch(DSA_KERNEL_QUANTIZE);
    return cudaGetLastError();
}

}  // namespace dsa
