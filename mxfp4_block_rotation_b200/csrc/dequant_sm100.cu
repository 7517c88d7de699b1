// dequant_sm100.cu -- plain MXFP4 dequantisation for B200 (sm_100a).
//
// The fake-quant "simulator" of the DuQuant++ write-up (jsqmd.com/news/928156,
// §5.1 item 5): v = E2M1(code) * 2^(byte - 127) for each element of a 32-element
// group, written as bf16.  Every such value is exactly representable in bf16
// (two significant bits, fp32's exponent range), so the output is exact; a
// scale byte 0xFF gives NaN and values past bf16's range give +-Inf.
//
// One thread per 8 outputs: it loads 4 code bytes and its group's scale byte
// and looks each code byte up in a 256-entry shared-memory table.  The table
// holds the bf16 pair of the byte's two E2M1 values (low nibble = even column).
// One packed bf16x2 multiply by 2^e then gives two outputs at once.  The warp
// reads 128 contiguous code bytes and writes 512 contiguous output bytes.
//
// (Undoing the rotation is a 32x32 contraction and runs on the tensor cores in
// rotquant_sm100.cu.)
#include <cuda_bf16.h>

#include "mxq_internal.h"

namespace mxq {
namespace {

constexpr int kThreads = 256;

// bf16 bit pattern of the E2M1 value of a 4-bit code (bit 3 = sign).
__device__ __forceinline__ uint32_t e2m1_bf16_bits(uint32_t code)
{
    // magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}: code 1 is E2M1's subnormal 0.5; codes
    // 2..7 are 2^(e-1) * (1 + m/2) with e = code >> 1, m = code & 1
    const uint32_t m = code & 7u;
    const uint32_t mag = m == 0u ? 0u : (m == 1u ? 0x3F00u : (((125u + (m >> 1)) + 1u) << 7) | ((m & 1u) << 6));
    return mag | ((code & 8u) << 12);
}

// 2^(byte-127) as bf16 (byte 0 is the subnormal 2^-127; 0xFF is NaN), duplicated in both halves.
__device__ __forceinline__ __nv_bfloat162 e8m0_bf16x2(uint32_t byte)
{
    const uint32_t b = byte == 0xFFu ? 0x7FC0u : (byte == 0u ? 0x0040u : (byte << 7));
    return __halves2bfloat162(__ushort_as_bfloat16(static_cast<unsigned short>(b)),
                              __ushort_as_bfloat16(static_cast<unsigned short>(b)));
}

__device__ __forceinline__ uint32_t bf162_bits(__nv_bfloat162 v)
{
    return static_cast<uint32_t>(__bfloat16_as_ushort(__low2bfloat16(v))) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(__high2bfloat16(v))) << 16);
}

__global__ void __launch_bounds__(kThreads)
    dequant_plain_kernel(const uint32_t *__restrict__ codes4, const uint8_t *__restrict__ scales, int64_t n_chunks,
                         uint4 *__restrict__ out)
{
    __shared__ uint32_t lut[256];   // code byte -> bf16x2 (low nibble in the low half)
    for (int i = threadIdx.x; i < 256; i += kThreads)
        lut[i] = e2m1_bf16_bits(static_cast<uint32_t>(i) & 15u) | (e2m1_bf16_bits(static_cast<uint32_t>(i) >> 4) << 16);
    __syncthreads();
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; t < n_chunks; t += stride) {
        const uint32_t c = __ldcs(codes4 + t);                       // 8 codes
        const __nv_bfloat162 s2 = e8m0_bf16x2(__ldg(scales + (t >> 2)));   // 4 chunks per group
        uint32_t o[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const uint32_t pair = lut[(c >> (8 * b)) & 0xFFu];
            __nv_bfloat162 v = __halves2bfloat162(__ushort_as_bfloat16(static_cast<unsigned short>(pair & 0xFFFFu)),
                                                  __ushort_as_bfloat16(static_cast<unsigned short>(pair >> 16)));
            o[b] = bf162_bits(__hmul2(v, s2));   // exact: a power-of-two scaling of a 2-bit significand
        }
        __stcs(out + t, make_uint4(o[0], o[1], o[2], o[3]));
    }
}

}  // namespace

cudaError_t launch_dequant_plain(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t cols,
                                 uint16_t *out, int num_sms, cudaStream_t stream)
{
    const int64_t n_chunks = rows * cols / 8;
    if (n_chunks <= 0) return cudaSuccess;
    const int64_t want = (n_chunks + kThreads - 1) / kThreads;
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    const int grid = static_cast<int>(want < cap ? want : cap);
    dequant_plain_kernel<<<grid, kThreads, 0, stream>>>(reinterpret_cast<const uint32_t *>(codes), scales, n_chunks,
                                                        reinterpret_cast<uint4 *>(out));
    return cudaGetLastError();
}

}  // namespace mxq
