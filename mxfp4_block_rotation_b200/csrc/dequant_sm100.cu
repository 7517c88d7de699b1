// dequant_sm100.cu -- MXFP4 dequantisation for B200 (sm_100a).
//
// The fake-quant "simulator" of the DuQuant++ write-up (jsqmd.com/news/928156,
// §5.1 item 5): v = E2M1(code) * 2^(byte - 127) for each element of a 32-element
// group.  Optionally the online transform of §3.3 is undone: the rotation
// (x = v * R^T, R^ orthogonal) and the smoothing (x *= Lambda).
//
// One thread per group.  Threads of a warp take consecutive groups, so the
// 16-byte code loads of a warp cover one contiguous 512-byte span.  Plain
// dequantisation is exact in fp32 and in bf16, so its output is bit-exact.  The
// rotation-undo variant keeps R^ in shared memory as fp32 [k][n] (every thread
// of a warp reads the same entry, a broadcast) and accumulates 32 FMAs per output
// in fp32.
#include <cuda_bf16.h>

#include "mxq_internal.h"

namespace mxq {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float e2m1_value(uint32_t code)
{
    // magnitudes of codes 0..7: {0, 0.5, 1, 1.5, 2, 3, 4, 6}; bit 3 is the sign
    const uint32_t m = code & 7u;
    const float mag = m < 4u ? 0.5f * static_cast<float>(m) : static_cast<float>(1u << ((m >> 1) - 1)) *
                                                                   (1.0f + 0.5f * static_cast<float>(m & 1u));
    return (code & 8u) ? -mag : mag;
}

__device__ __forceinline__ float e8m0_value(uint32_t byte)
{
    if (byte == 0xFFu) return __uint_as_float(0x7FC00000u);   // NaN
    if (byte == 0u) return __uint_as_float(0x00400000u);      // 2^-127 (fp32 subnormal)
    return __uint_as_float(byte << 23);                       // 2^(byte-127)
}

__device__ __forceinline__ uint32_t pack2(float a, float b)
{
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(a))) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(b))) << 16);
}

template <bool kRotate, bool kLambda>
__global__ void __launch_bounds__(kThreads)
    dequant_kernel(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scales, int64_t n_groups,
                   int64_t G, const uint16_t *__restrict__ rhat, const float *__restrict__ lambda,
                   uint16_t *__restrict__ out)
{
    __shared__ float r[32 * 32];   // R^[k][n] as fp32
    if constexpr (kRotate) {
        for (int i = threadIdx.x; i < 32 * 32; i += kThreads)
            r[i] = __bfloat162float(__ushort_as_bfloat16(rhat[i]));
        __syncthreads();
    }
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
    for (int64_t gi = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; gi < n_groups; gi += stride) {
        const uint4 c = __ldcs(reinterpret_cast<const uint4 *>(codes) + gi);
        const float s = e8m0_value(scales[gi]);
        const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(e2m1_value((cw[i >> 3] >> (4 * (i & 7))) & 15u), s);
        float x[32];
        if constexpr (kRotate) {
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                float acc = 0.0f;
#pragma unroll
                for (int n = 0; n < 32; ++n) acc = __fmaf_rn(v[n], r[k * 32 + n], acc);
                x[k] = acc;
            }
            if constexpr (kLambda) {
                const int64_t ch0 = (gi % G) * 32;
#pragma unroll
                for (int k = 0; k < 32; ++k) x[k] = __fmul_rn(x[k], lambda[ch0 + k]);
            }
        } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) x[k] = v[k];
        }
        uint4 *dst = reinterpret_cast<uint4 *>(out + gi * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            __stcs(dst + q, make_uint4(pack2(x[8 * q], x[8 * q + 1]), pack2(x[8 * q + 2], x[8 * q + 3]),
                                       pack2(x[8 * q + 4], x[8 * q + 5]), pack2(x[8 * q + 6], x[8 * q + 7])));
    }
}

template <bool kRotate, bool kLambda>
cudaError_t launch_one(const uint8_t *codes, const uint8_t *scales, int64_t n_groups, int64_t G,
                       const uint16_t *rhat, const float *lambda, uint16_t *out, int num_sms,
                       cudaStream_t stream)
{
    const int64_t want = (n_groups + kThreads - 1) / kThreads;
    const int64_t cap = static_cast<int64_t>(num_sms) * (kRotate ? 4 : 8);
    const int grid = static_cast<int>(want < cap ? want : cap);
    dequant_kernel<kRotate, kLambda><<<grid, kThreads, 0, stream>>>(codes, scales, n_groups, G, rhat, lambda, out);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dequant(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t cols,
                           const uint16_t *rhat, const float *lambda, uint16_t *out, int num_sms,
                           cudaStream_t stream)
{
    const int64_t G = cols / 32;
    const int64_t n_groups = rows * G;
    if (n_groups <= 0) return cudaSuccess;
    if (rhat == nullptr) return launch_one<false, false>(codes, scales, n_groups, G, rhat, lambda, out, num_sms, stream);
    if (lambda == nullptr) return launch_one<true, false>(codes, scales, n_groups, G, rhat, lambda, out, num_sms, stream);
    return launch_one<true, true>(codes, scales, n_groups, G, rhat, lambda, out, num_sms, stream);
}

}  // namespace mxq
