// dequant_sm100.cu -- MXFP4 dequantisation for B200 (sm_100a): plain, and undoing the transform.
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
// Undoing the rotation (and smoothing) is a 32x32 contraction and runs on the
// tensor cores in dequant_rot_kernel below.
#include <cuda_bf16.h>

#include "pipeline_sm100.cuh"

namespace mxq {
namespace {

constexpr int kPlainThreads = 256;

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

__global__ void __launch_bounds__(kPlainThreads)
    dequant_plain_kernel(const uint32_t *__restrict__ codes4, const uint8_t *__restrict__ scales, int64_t n_chunks,
                         uint4 *__restrict__ out)
{
    __shared__ uint32_t lut[256];   // code byte -> bf16x2 (low nibble in the low half)
    for (int i = threadIdx.x; i < 256; i += kPlainThreads)
        lut[i] = e2m1_bf16_bits(static_cast<uint32_t>(i) & 15u) | (e2m1_bf16_bits(static_cast<uint32_t>(i) >> 4) << 16);
    __syncthreads();
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kPlainThreads;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * kPlainThreads + threadIdx.x; t < n_chunks; t += stride) {
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

using namespace pipe;

// ---------------------------------------------------------------- undo the transform
//
// out = (v * R^T) * Lambda, v = E2M1(code) * 2^e.
// The same flat group-major pipeline as rotate_flat_kernel, run backwards.  Four
// decoder warps turn each stage's 512 groups of codes into bf16 values in
// shared memory: the MMA's A tile, 64-byte swizzle.  The values are exact in
// bf16: two significant bits times a power of two.  The MMA computes
// D[g][k] = sum_n v[g][n] * R^[k][n], so B is R^ as stored (row k, contiguous n
// = K-major).  The epilogue multiplies by Lambda_k and rounds to bf16.

constexpr int kDqDecWarp0 = 8;
constexpr int kDqDecWarps = 4;
constexpr int kDqMmaWarp = 12;
constexpr int kDqThreads = (kDqMmaWarp + 1) * 32;   // 416
constexpr int kDqStages = 3;
constexpr int kDqStageGroups = 512;                 // 4 MMAs of 128 groups
constexpr int kDqStageBytes = kDqStageGroups * 64;
constexpr int kDqAcc = 4;
constexpr int kDqAccCols = 128;
constexpr int kDqOutBuf = 32 * 64;                 // one epilogue warp's 32 output groups (2 KB)
constexpr int kDqOutBytes = kEpiWarps * 2 * kDqOutBuf;   // double-buffered per epilogue warp
constexpr int kDqLamBytes = kEpiWarps * 32 * 128;   // per epilogue warp: Lambda of its 32 groups
constexpr int kDqSmemBytes = kDqStages * kDqStageBytes + kBMatBytes + 1024 + kDqOutBytes + kDqLamBytes + 512 + 1024;

__device__ __forceinline__ uint32_t e2m1_bf16(uint32_t code)
{
    // magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}: code 1 is E2M1's subnormal 0.5; codes
    // 2..7 are 2^(e-1) * (1 + m/2) with e = code >> 1, m = code & 1
    const uint32_t m = code & 7u;
    const uint32_t mag = m == 0u ? 0u : (m == 1u ? 0x3F00u : ((126u + (m >> 1)) << 7) | ((m & 1u) << 6));
    return mag | ((code & 8u) << 12);
}

__device__ __forceinline__ uint32_t hmul2_bits(uint32_t a, __nv_bfloat162 s)
{
    const __nv_bfloat162 v = __halves2bfloat162(__ushort_as_bfloat16(static_cast<unsigned short>(a & 0xFFFFu)),
                                                __ushort_as_bfloat16(static_cast<unsigned short>(a >> 16)));
    const __nv_bfloat162 r = __hmul2(v, s);
    return static_cast<uint32_t>(__bfloat16_as_ushort(__low2bfloat16(r))) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(__high2bfloat16(r))) << 16);
}

template <bool kLambda>
__global__ void __launch_bounds__(kDqThreads, 1)
    dequant_rot_kernel(const __grid_constant__ CUtensorMap tmap_out, const uint4 *__restrict__ codes,
                       const uint8_t *__restrict__ scales, int64_t n_groups, int64_t G,
                       const uint16_t *__restrict__ rhat, const float *__restrict__ lambda, unsigned int *status)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *stages = align_1k(smem_raw);
    uint8_t *bmat = stages + kDqStages * kDqStageBytes;
    uint32_t *lut = reinterpret_cast<uint32_t *>(bmat + kBMatBytes);   // code byte -> bf16x2
    uint8_t *outbuf = bmat + kBMatBytes + 1024;                          // epilogue staging
    uint8_t *lambuf = outbuf + kDqOutBytes;                              // epilogue Lambda rows
    Bars *bars = reinterpret_cast<Bars *>(lambuf + kDqLamBytes);
    volatile int *abort = &bars->abort;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_chunks = static_cast<int>((n_groups + kDqStageGroups - 1) / kDqStageGroups);

    const uint32_t tmem_base = kernel_setup(
        bars, SetupCfg{kDqStages, kDqAcc, kDqDecWarps * 32, kDqDecWarps * 32, kDqMmaWarp}, &tmap_out, nullptr);

    if (warp >= kDqDecWarp0 && warp < kDqDecWarp0 + kDqDecWarps) {
        const int dt = threadIdx.x - kDqDecWarp0 * 32;   // 0..127
        for (int i = dt; i < 256; i += kDqDecWarps * 32)
            lut[i] = e2m1_bf16(static_cast<uint32_t>(i) & 15u) | (e2m1_bf16(static_cast<uint32_t>(i) >> 4) << 16);
        // B: row k holds R^[k][0..31] (bf16) in the first 64 B of a 128-byte-swizzled row
        if (dt < 32 * 4) {
            const int k = dt >> 2, c = dt & 3;
            const uint4 v = *reinterpret_cast<const uint4 *>(rhat + k * 32 + c * 8);
            *reinterpret_cast<uint4 *>(bmat + sw128(k, c)) = v;
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(ptx::smem_addr(&bars->b_full[0]));
        ptx::named_bar_sync(3, kDqDecWarps * 32);   // the table is complete
        int it = 0;
        for (int c = blockIdx.x; c < n_chunks; c += gridDim.x, ++it) {
            const int s = it % kDqStages;
            int ok = 0;
            if (lane == 0) ok = wait_bar(&bars->empty[s], ((it / kDqStages) & 1) ^ 1, abort, status);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            const uint32_t st = ptx::smem_addr(stages + s * kDqStageBytes);
#pragma unroll
            for (int i = 0; i < kDqStageGroups / (kDqDecWarps * 32); ++i) {
                const int r = dt + i * kDqDecWarps * 32;   // group row within the stage
                const int64_t g = static_cast<int64_t>(c) * kDqStageGroups + r;
                uint32_t w[16];
                if (g < n_groups) {
                    const uint4 cw = __ldcs(codes + g);
                    const uint32_t byte = __ldg(scales + g);
                    const uint32_t sb = byte == 0xFFu ? 0x7FC0u : (byte == 0u ? 0x0040u : (byte << 7));
                    const __nv_bfloat162 s2 = __halves2bfloat162(__ushort_as_bfloat16(static_cast<unsigned short>(sb)),
                                                                 __ushort_as_bfloat16(static_cast<unsigned short>(sb)));
                    const uint32_t cws[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
                    for (int b = 0; b < 16; ++b) w[b] = hmul2_bits(lut[(cws[b >> 2] >> (8 * (b & 3))) & 0xFFu], s2);
                } else {
#pragma unroll
                    for (int b = 0; b < 16; ++b) w[b] = 0u;
                }
                // 64-byte swizzle: 16-byte chunk q of row r sits at chunk q ^ ((r >> 1) & 3)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    ptx::st_shared_v4(st + r * 64 + ((q ^ ((r >> 1) & 3)) << 4), w[4 * q], w[4 * q + 1],
                                      w[4 * q + 2], w[4 * q + 3]);
            }
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(ptx::smem_addr(&bars->full[s]));
        }
    } else if (warp == kDqMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, 32);
            const uint32_t b_base = ptx::smem_addr(bmat);
            const bool b_ok = wait_bar(&bars->b_full[0], 0, abort, status);
            int it = 0;
            for (int c = blockIdx.x; b_ok && c < n_chunks; c += gridDim.x, ++it) {
                const int s = it % kDqStages;
                const int a = it % kDqAcc;
                if (!wait_bar(&bars->full[s], (it / kDqStages) & 1, abort, status)) break;
                if (!wait_bar(&bars->acc_empty[a], ((it / kDqAcc) & 1) ^ 1, abort, status)) break;
                ptx::tc_fence_after();
                const uint32_t a_base = ptx::smem_addr(stages + s * kDqStageBytes);
                const uint32_t d_base = tmem_base + static_cast<uint32_t>(a * kDqAccCols);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
#pragma unroll
                    for (int kh = 0; kh < 2; ++kh)
                        ptx::mma_bf16(d_base + j * 32, ptx::smem_desc_sw64(a_base + j * 128 * 64 + kh * 32),
                                      ptx::smem_desc_sw128(b_base + kh * 32), idesc, kh);
                }
                ptx::mma_commit(ptx::smem_addr(&bars->empty[s]));
                ptx::mma_commit(ptx::smem_addr(&bars->acc_full[a]));
            }
            drain_mmas(bars, status);
        }
    } else if (warp < kEpiWarps) {
        // Each warp stages its 32 groups' outputs (2 KB, 64-byte swizzle) and writes them
        // with one TMA bulk tensor store: 2 KB contiguous instead of 16-byte pieces.
        const int q = warp & 3;
        const int ewg = warp >> 2;
        const uint32_t obuf0 = ptx::smem_addr(outbuf + warp * 2 * kDqOutBuf);
        const bool lam_vec = kLambda && ((reinterpret_cast<uintptr_t>(lambda) & 15) == 0);
        float *lrows = reinterpret_cast<float *>(lambuf + warp * 32 * 128);   // 32 rows x 32 channels
        int it = 0, nstore = 0;
        for (int c = blockIdx.x; c < n_chunks; c += gridDim.x, ++it) {
            if ((it & 1) != ewg) continue;
            const int a = it % kDqAcc;
            int ok = 0;
            if (lane == 0) ok = wait_bar(&bars->acc_full[a], (it / kDqAcc) & 1, abort, status);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            ptx::tc_fence_after();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * kDqAccCols;
            const int64_t g_warp = static_cast<int64_t>(c) * kDqStageGroups + q * 32;
            // (one register buffer: with 13 warps an SMSP holds four, so 128 registers a thread)
#pragma unroll 1
            for (int j = 0; j < 4; ++j) {
                uint32_t cur[32];
                ptx::tmem_ld_32cols(t_row + j * 32, cur);
                ptx::tmem_wait_ld();
                const int64_t g0 = g_warp + j * 128;   // this warp's first group of MMA j
                // Lambda of the 32 groups' channels: fetched with coalesced loads (8 lanes per
                // 128-byte row) into this warp's rows, 16-byte chunks XOR-swizzled by row.
                if constexpr (kLambda) {
                    __syncwarp();
                    const int col0 = static_cast<int>(g0 % G);   // column group of this warp's first group
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = 4 * i + (lane >> 3), cc = lane & 7;
                        const float *src = lambda + static_cast<int64_t>((col0 + r) % static_cast<int>(G)) * 32 + cc * 4;
                        float4 l4;
                        if (lam_vec) {
                            l4 = __ldg(reinterpret_cast<const float4 *>(src));
                        } else {
                            l4.x = __ldg(src);
                            l4.y = __ldg(src + 1);
                            l4.z = __ldg(src + 2);
                            l4.w = __ldg(src + 3);
                        }
                        *reinterpret_cast<float4 *>(lrows + r * 32 + ((cc ^ (r & 7)) << 2)) = l4;
                    }
                    __syncwarp();
                }
                // times Lambda_k (channels of this group), then round to bf16 pairs
                uint32_t o[16];
#pragma unroll
                for (int k4 = 0; k4 < 8; ++k4) {
                    float4 l4 = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
                    if constexpr (kLambda)
                        l4 = *reinterpret_cast<const float4 *>(lrows + lane * 32 + ((k4 ^ (lane & 7)) << 2));
                    const __nv_bfloat162 p0 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(cur[4 * k4]), l4.x),
                                                                    __fmul_rn(__uint_as_float(cur[4 * k4 + 1]), l4.y));
                    const __nv_bfloat162 p1 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(cur[4 * k4 + 2]), l4.z),
                                                                    __fmul_rn(__uint_as_float(cur[4 * k4 + 3]), l4.w));
                    o[2 * k4] = static_cast<uint32_t>(__bfloat16_as_ushort(__low2bfloat16(p0))) |
                                (static_cast<uint32_t>(__bfloat16_as_ushort(__high2bfloat16(p0))) << 16);
                    o[2 * k4 + 1] = static_cast<uint32_t>(__bfloat16_as_ushort(__low2bfloat16(p1))) |
                                    (static_cast<uint32_t>(__bfloat16_as_ushort(__high2bfloat16(p1))) << 16);
                }
                const uint32_t buf = obuf0 + (nstore & 1) * kDqOutBuf;
                // the buffer's previous store (two stores ago) must have been read
                if (lane == 0) ptx::bulk_wait_group_read1();
                __syncwarp();
#pragma unroll
                for (int v = 0; v < 4; ++v)
                    ptx::st_shared_v4(buf + lane * 64 + ((v ^ ((lane >> 1) & 3)) << 4), o[4 * v], o[4 * v + 1],
                                      o[4 * v + 2], o[4 * v + 3]);
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && g0 < n_groups) {   // rows past n_groups are clipped by the tensor map
                    ptx::tma_store_2d(&tmap_out, 0, static_cast<int32_t>(g0), buf);
                    ptx::bulk_commit_group();
                }
                ++nstore;
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&bars->acc_empty[a]));
        }
        if (lane == 0) ptx::bulk_wait_group0();   // stores done before the CTA's shared memory goes
    }
    kernel_teardown(tmem_base, kDqMmaWarp);
}

static_assert(kDqSmemBytes <= 232448, "shared memory budget");

}  // namespace

cudaError_t launch_dequant_rot(const CUtensorMap &tmap_out, const uint8_t *codes, const uint8_t *scales, int64_t rows,
                               int64_t cols, const uint16_t *rhat, const float *lambda, int num_sms,
                               cudaStream_t stream)
{
    const int64_t G = cols / 32;
    const int64_t n_groups = rows * G;
    if (n_groups <= 0) return cudaSuccess;
    const int64_t n_chunks = (n_groups + kDqStageGroups - 1) / kDqStageGroups;
    const int grid = static_cast<int>(n_chunks < num_sms ? n_chunks : num_sms);
    unsigned int *status = status_word();
    if (!status) return cudaErrorInvalidSymbol;
    const uint4 *c4 = reinterpret_cast<const uint4 *>(codes);
    return lambda ? launch_pdl(dequant_rot_kernel<true>, grid, kDqThreads, kDqSmemBytes, stream, tmap_out, c4, scales,
                               n_groups, G, rhat, lambda, status)
                  : launch_pdl(dequant_rot_kernel<false>, grid, kDqThreads, kDqSmemBytes, stream, tmap_out, c4, scales,
                               n_groups, G, rhat, lambda, status);
}

cudaError_t launch_dequant_plain(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t cols,
                                 uint16_t *out, int num_sms, cudaStream_t stream)
{
    const int64_t n_chunks = rows * cols / 8;
    if (n_chunks <= 0) return cudaSuccess;
    const int64_t want = (n_chunks + kPlainThreads - 1) / kPlainThreads;
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    const int grid = static_cast<int>(want < cap ? want : cap);
    dequant_plain_kernel<<<grid, kPlainThreads, 0, stream>>>(reinterpret_cast<const uint32_t *>(codes), scales, n_chunks,
                                                        reinterpret_cast<uint4 *>(out));
    return cudaGetLastError();
}

}  // namespace mxq
