// pipeline_sm100.cuh -- pieces shared by the warp-specialised tcgen05 kernels
// (rotate_flat_sm100.cu, rotate_cols_sm100.cu, dequant_sm100.cu): warp roles,
// the shared-memory barrier block, the bounded mbarrier wait, the MXFP4 group
// quantiser, kernel set-up / tear-down and the programmatic-dependent launch.
#pragma once

#include <cuda_bf16.h>

#include "mxq_internal.h"
#include "sm100_bulk.cuh"
#include "sm100_ptx.cuh"

namespace mxq {
namespace pipe {

constexpr uint32_t kTmemCols = 512;      // all of TMEM: accumulator stages of 32 columns per MMA
constexpr int kMaxAcc = 8;
constexpr int kEpiWarps = 8;
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kBuildWarp0 = 10;
constexpr int kBuildWarps = 2;
constexpr int kThreads = (kEpiWarps + 2 + kBuildWarps) * 32;   // 384, the flat rotate kernel
constexpr int kBMatBytes = 32 * 128;     // one B atom: 32 rows (n) x 128 B, 128-byte swizzle
constexpr uint64_t kTimeoutNs = 2000000000ull;   // 2 s per wait
constexpr int kMaxStages = 8;

struct Bars {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t acc_full[kMaxAcc];
    uint64_t acc_empty[kMaxAcc];
    uint64_t b_full[2];
    uint64_t b_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int eg_ok[2][2];   // per epilogue warp group, per tile parity: the leader's wait result
    int bl_ok[2];      // per tile parity: the B builders' leader's wait result
};
static_assert(sizeof(Bars) <= 512, "barrier block");

// Bounded wait on an mbarrier phase.  False if the wait ran out or (when abort
// is non-null) another role has already aborted.  Drains at exit pass a null
// abort so they keep waiting, within the time bound, for work already in flight.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort, unsigned int *status,
                                         uint64_t timeout_ns = kTimeoutNs)
{
    const uint32_t b = ptx::smem_addr(bar);
    if (ptx::mbar_try_wait(b, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (ptx::mbar_try_wait(b, parity)) return true;
        if ((i & 63) == 0) {
            if (abort && *abort) return false;
            if (ptx::globaltimer_ns() - t0 > timeout_ns || i > (1u << 30)) {
                if (abort) *abort = 1;
                atomicOr(status, kStatusTimeout);
                return false;
            }
        }
    }
}

// Element [k][n] of the 32x32 rotation, as bf16 bits: the matrix itself, or for
// rotation blocks of 16 columns the block-diagonal diag(R16, R16) of a 16x16 input.
__device__ __forceinline__ uint16_t rhat_at(const RotArgs &a, int k, int n)
{
    if (a.rblk == 16) return ((k ^ n) & 16) ? static_cast<uint16_t>(0) : a.rhat[(k & 15) * 16 + (n & 15)];
    return a.rhat[k * 32 + n];
}

// Byte offset of 16-byte chunk c of row r inside a 128-byte-swizzled atom.
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t c)
{
    return r * 128u + ((c ^ (r & 7u)) << 4);
}

__device__ __forceinline__ uint32_t pack_bf16x2(__nv_bfloat16 lo, __nv_bfloat16 hi)
{
    return static_cast<uint32_t>(__bfloat16_as_ushort(lo)) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
}

__device__ __forceinline__ uint8_t *align_1k(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

// MXFP4 of one 32-value group (fp32 bit patterns): returns the E8M0 byte and
// writes the 32 E2M1 codes packed into four words (value 2i in the low nibble
// of byte i).  E8M0 = floor(log2 amax) - 2 + 127 comes straight from amax's
// exponent field (clamped at 0); 2^-e is built from bits, so the scaling is exact.
__device__ __forceinline__ uint32_t quantize_group(const uint32_t (&r)[32], uint32_t (&w)[4])
{
    float m[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        m[i] = ptx::fmax_nan(fabsf(__uint_as_float(r[2 * i])), fabsf(__uint_as_float(r[2 * i + 1])));
#pragma unroll
    for (int step = 8; step >= 1; step >>= 1)
#pragma unroll
        for (int i = 0; i < step; ++i) m[i] = ptx::fmax_nan(m[i], m[i + step]);
    const uint32_t E = (__float_as_uint(m[0]) >> 23) & 0xFFu;
    if (E == 0xFFu) {   // NaN/Inf group: scale byte 0xFF, codes 0
        w[0] = w[1] = w[2] = w[3] = 0u;
        return 0xFFu;
    }
    const uint32_t byte = E > 2u ? E - 2u : 0u;
    const float s = __uint_as_float((254u - byte) << 23);   // 2^-e
    float2 u[16];   // u = y * 2^-e, exact, on pairs (sm_100's packed fp32 multiply)
#pragma unroll
    for (int i = 0; i < 16; ++i)
        u[i] = __fmul2_rn(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), make_float2(s, s));
#pragma unroll
    for (int q = 0; q < 4; ++q)
        w[q] = ptx::cvt_e2m1x8(u[4 * q].x, u[4 * q].y, u[4 * q + 1].x, u[4 * q + 1].y, u[4 * q + 2].x, u[4 * q + 2].y,
                               u[4 * q + 3].x, u[4 * q + 3].y);
    return byte;
}

// Byte offset of the E8M0 scale of row r, group g in the block-scaled MMA's scale layout:
// 512-byte atoms of 128 rows x 4 groups, ordered by row block and then group block
// (kb4 = ceil(G / 4) atoms per row block); inside an atom, row r and group g sit at byte
// 16 (r % 32) + 4 ((r / 32) % 4) + g % 4.
__device__ __forceinline__ int64_t sf_mma_offset(int64_t r, int64_t g, int64_t kb4)
{
    return ((r >> 7) * kb4 + (g >> 2)) * 512 + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (g & 3);
}

// MXFP4 of one group as in quantize_group, plus its normalised quantisation error
// ||Q(y) - y||_2 / ||y||_2.  With u = y * 2^-e the power of two cancels:
// error = ||Q(u) - u|| / ||u||, where Q(u) is u's E2M1 value.  An all-zero group
// has error 0, a NaN/Inf group NaN.
__device__ __forceinline__ uint32_t quantize_group_err(const uint32_t (&r)[32], uint32_t (&w)[4], float &err)
{
    float m[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        m[i] = ptx::fmax_nan(fabsf(__uint_as_float(r[2 * i])), fabsf(__uint_as_float(r[2 * i + 1])));
#pragma unroll
    for (int step = 8; step >= 1; step >>= 1)
#pragma unroll
        for (int i = 0; i < step; ++i) m[i] = ptx::fmax_nan(m[i], m[i + step]);
    const uint32_t E = (__float_as_uint(m[0]) >> 23) & 0xFFu;
    if (E == 0xFFu) {
        w[0] = w[1] = w[2] = w[3] = 0u;
        err = __uint_as_float(0x7FC00000u);
        return 0xFFu;
    }
    const uint32_t byte = E > 2u ? E - 2u : 0u;
    const float s = __uint_as_float((254u - byte) << 23);   // 2^-e
    // the arithmetic on pairs of values (sm_100's packed fp32 instructions): u = y * 2^-e exactly
    float2 u[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        u[i] = __fmul2_rn(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), make_float2(s, s));
#pragma unroll
    for (int q = 0; q < 4; ++q)
        w[q] = ptx::cvt_e2m1x8(u[4 * q].x, u[4 * q].y, u[4 * q + 1].x, u[4 * q + 1].y, u[4 * q + 2].x, u[4 * q + 2].y,
                               u[4 * q + 3].x, u[4 * q + 3].y);
    // -|Q(u)| straight from the codes just produced: byte permutes pick the bf16 bits of each
    // code's magnitude {0, .5, 1, 1.5, 2, 3, 4, 6} (code 8q + k is nibble k of w[q]), with the
    // sign bit set; Q(u) has u's sign, so |Q(u) - u| = ||u| - |Q(u)||.
    float2 num[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
    float2 den[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t mg = w[q] & 0x77777777u;
        const uint32_t h0 = ptx::prmt(0xBFBFBF80u, 0xC0C0C0C0u, mg & 0xFFFFu);
        const uint32_t l0 = ptx::prmt(0xC0800000u, 0xC0804000u, mg & 0xFFFFu);
        const uint32_t h1 = ptx::prmt(0xBFBFBF80u, 0xC0C0C0C0u, mg >> 16);
        const uint32_t l1 = ptx::prmt(0xC0800000u, 0xC0804000u, mg >> 16);
        const uint32_t p[4] = {ptx::prmt(l0, h0, 0x5140u), ptx::prmt(l0, h0, 0x7362u), ptx::prmt(l1, h1, 0x5140u),
                               ptx::prmt(l1, h1, 0x7362u)};
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) {
            const int i = 4 * q + k2;   // the pair (2i, 2i + 1): nibbles 2 k2, 2 k2 + 1 of w[q]
            const float2 nq = make_float2(__uint_as_float(p[k2] << 16), __uint_as_float(p[k2] & 0xFFFF0000u));
            const float2 a = make_float2(fabsf(u[i].x), fabsf(u[i].y));
            const float2 d = __fadd2_rn(a, nq);
            num[i & 1] = __ffma2_rn(d, d, num[i & 1]);
            den[i & 1] = __ffma2_rn(u[i], u[i], den[i & 1]);
        }
    }
    const float n = (num[0].x + num[1].x) + (num[0].y + num[1].y);
    const float d = (den[0].x + den[1].x) + (den[0].y + den[1].y);
    err = d > 0.0f ? __fsqrt_rn(__fdiv_rn(n, d)) : 0.0f;
    return byte;
}

// NVFP4 of one 32-value group = two 16-value blocks (the public NVFP4 format; decided
// in fp32 as r_t = 1 / (6 s_t), v = amax * r_t, s_b = E4M3(v) round to nearest even
// saturating at 448, s = s_b * s_t, u = y * (1 / s), E2M1(u)).  Writes the 32 codes
// packed as quantize_group does and returns the two E4M3 scale bytes (block 0 in the
// low byte).  A block holding NaN or Inf gets 0x7F (E4M3 NaN) and codes 0; a zero
// scale gives codes 0.
__device__ __forceinline__ uint32_t quantize_group_nv(const uint32_t (&r)[32], uint32_t (&w)[4], float r_t, float s_t)
{
    float amax[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float m[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            m[i] = ptx::fmax_nan(fabsf(__uint_as_float(r[16 * h + 2 * i])),
                                 fabsf(__uint_as_float(r[16 * h + 2 * i + 1])));
#pragma unroll
        for (int step = 4; step >= 1; step >>= 1)
#pragma unroll
            for (int i = 0; i < step; ++i) m[i] = ptx::fmax_nan(m[i], m[i + step]);
        amax[h] = m[0];
    }
    uint32_t sb2;   // the two E4M3 bytes, block 0 low
    {
        const float v0 = __fmul_rn(amax[0], r_t), v1 = __fmul_rn(amax[1], r_t);
        uint16_t d;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(v1), "f"(v0));
        sb2 = d;
    }
    uint32_t out = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const bool bad = ((__float_as_uint(amax[h]) >> 23) & 0xFFu) == 0xFFu;
        const uint32_t b = bad ? 0x7Fu : ((sb2 >> (8 * h)) & 0xFFu);
        out |= b << (8 * h);
        // E4M3 -> fp32 (exact): exponent e (bias 7), 3 mantissa bits; e = 0 is subnormal m * 2^-9
        const uint32_t e = (b >> 3) & 15u, mm = b & 7u;
        const float sbv =
            e ? __uint_as_float(((e + 120u) << 23) | (mm << 20)) : __fmul_rn(static_cast<float>(mm), 0x1p-9f);
        const float s = __fmul_rn(sbv, s_t);
        const bool zero = b == 0x7Fu || s == 0.0f;   // NaN scale (bad block, or v = 0 * inf)
        const float rr = zero ? 0.0f : __frcp_rn(s);
        // u = y * (1/s), two elements per packed multiply; a zero block's codes are all 0
        float2 u[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            u[i] = __fmul2_rn(make_float2(__uint_as_float(r[16 * h + 2 * i]), __uint_as_float(r[16 * h + 2 * i + 1])),
                              make_float2(rr, rr));
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const uint32_t c = ptx::cvt_e2m1x8(u[4 * q].x, u[4 * q].y, u[4 * q + 1].x, u[4 * q + 1].y, u[4 * q + 2].x,
                                               u[4 * q + 2].y, u[4 * q + 3].x, u[4 * q + 3].y);
            w[2 * h + q] = zero ? 0u : c;
        }
    }
    return out;
}

// Sum over the warp in a fixed shuffle order (deterministic); the result is in lane 0.
__device__ __forceinline__ double warp_sum(double v)
{
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v += __shfl_down_sync(0xffffffffu, v, off);
    return v;
}

// Per-kernel numbers the shared set-up needs.
struct SetupCfg {
    int n_stages;     // shared-memory stages (full/empty barrier pairs)
    int n_acc;        // TMEM accumulator stages
    int full_count;   // arrivals that complete a stage's full barrier (1 for a TMA producer)
    int b_count;      // arrivals that complete b_full (the B builders' threads)
    int mma_warp;     // the warp that owns TMEM
};

// Barrier initialisation, TMEM allocation and the programmatic-dependent-launch
// handshake shared by the kernels.  Returns the TMEM base address.
__device__ __forceinline__ uint32_t kernel_setup(Bars *bars, const SetupCfg &cfg, const CUtensorMap *map0,
                                                 const CUtensorMap *map1)
{
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        for (int s = 0; s < cfg.n_stages; ++s) {
            ptx::mbar_init(ptx::smem_addr(&bars->full[s]), cfg.full_count);
            ptx::mbar_init(ptx::smem_addr(&bars->empty[s]), 1);
        }
        for (int a = 0; a < cfg.n_acc; ++a) {
            ptx::mbar_init(ptx::smem_addr(&bars->acc_full[a]), 1);
            ptx::mbar_init(ptx::smem_addr(&bars->acc_empty[a]), kEpiWarps / 2);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(ptx::smem_addr(&bars->b_full[s]), cfg.b_count);
            ptx::mbar_init(ptx::smem_addr(&bars->b_empty[s]), 1);
        }
        ptx::mbar_init(ptx::smem_addr(&bars->drain), 1);
        bars->abort = 0;
        ptx::fence_mbar_init();
        if (map0) ptx::prefetch_tmap(map0);
        if (map1) ptx::prefetch_tmap(map1);
    }
    if (warp == cfg.mma_warp) {
        ptx::tmem_alloc(ptx::smem_addr(&bars->tmem_base), kTmemCols);
        ptx::tmem_relinquish();
    }
    // Nothing above touches global memory, so the next kernel in the stream may start
    // its own set-up now; every global access below waits for the previous kernel.
    ptx::griddep_launch_dependents();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = bars->tmem_base;
    ptx::griddep_wait();
    return tmem_base;
}

// Producer epilogue: let the last copy into each stage land before the CTA can exit.
__device__ __forceinline__ void drain_loads(Bars *bars, int n_stages, int issued, unsigned int *status)
{
    for (int s = 0; s < n_stages && s < issued; ++s) {
        const int last = issued - 1 - ((issued - 1 - s) % n_stages);
        wait_bar(&bars->full[s], (last / n_stages) & 1, nullptr, status);
    }
}

// MMA epilogue: every MMA this thread issued must finish before TMEM is freed.
__device__ __forceinline__ void drain_mmas(Bars *bars, unsigned int *status)
{
    ptx::mma_commit(ptx::smem_addr(&bars->drain));
    wait_bar(&bars->drain, 0, nullptr, status);
}

__device__ __forceinline__ void kernel_teardown(uint32_t tmem_base, int mma_warp)
{
    ptx::tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == mma_warp) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, kTmemCols);
    }
}

// Launch with programmatic stream serialisation: the grid may start while the
// previous kernel in the stream drains (the kernels order their global accesses
// with griddepcontrol.wait).
// The dynamic shared-memory opt-in is set once per (kernel, device) (smem_optin); a
// launch the runtime refuses is retried once after setting it again, which covers a
// device reset having cleared it.
template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kern, int grid, int block, int smem, cudaStream_t stream, Args... args)
{
    const void *fn = reinterpret_cast<const void *>(kern);
    cudaError_t e = smem_optin(fn, smem, false);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, args...);
    if (e == cudaSuccess || smem <= 48 * 1024) return e;
    (void)cudaGetLastError();
    if ((e = smem_optin(fn, smem, true)) != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace pipe
}  // namespace mxq
