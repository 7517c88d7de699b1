// dequant_sm100.cu -- MXFP4 dequantisation for B200 (sm_100a): plain, and undoing the transform.
//
// The fake-quant "simulator" of the DuQuant++ write-up (jsqmd.com/news/928156,
// §5.1 item 5): v = E2M1(code) * 2^(byte - 127) for each element of a 32-element
// group, written as bf16.  Every such value is exactly representable in bf16
// (two significant bits, fp32's exponent range), so the output is exact; a
// scale byte 0xFF gives NaN and values past bf16's range give +-Inf.
//
// A thread takes 8 outputs at a time (four such chunks per pass, their loads
// issued together): it loads 4 code bytes and the group's scale byte and looks
// each code byte up in a 256-entry shared-memory table.  The table
// holds the bf16 pair of the byte's two E2M1 values (low nibble = even column).
// One packed bf16x2 multiply by 2^e then gives two outputs at once.  The warp
// reads 128 contiguous code bytes and writes 512 contiguous output bytes.
//
// Undoing the rotation (and smoothing) is a 32x32 contraction and runs on the
// tensor cores in dequant_rot_kernel below.
#include <cuda_bf16.h>

#include "pipeline_sm100.cuh"
#include "sm100_bulk.cuh"

namespace mxq {
namespace {

constexpr int kPlainThreads = 256;
constexpr int kPlainUnroll = 4;   // chunks per thread per pass

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
    // kPlainUnroll chunks per pass, all loads issued before any use: the code reads are
    // small (4 B a lane), so several must be in flight per thread to cover DRAM latency
    for (int64_t t0 = static_cast<int64_t>(blockIdx.x) * kPlainThreads + threadIdx.x; t0 < n_chunks;
         t0 += stride * kPlainUnroll) {
        uint32_t c[kPlainUnroll], sb[kPlainUnroll];
#pragma unroll
        for (int u = 0; u < kPlainUnroll; ++u) {
            const int64_t t = t0 + u * stride;
            c[u] = 0u;
            sb[u] = 0u;
            if (t < n_chunks) {
                c[u] = __ldcs(codes4 + t);                 // 8 codes
                sb[u] = __ldg(scales + (t >> 2));          // 4 chunks per group
            }
        }
#pragma unroll
        for (int u = 0; u < kPlainUnroll; ++u) {
            const int64_t t = t0 + u * stride;
            if (t >= n_chunks) break;
            const __nv_bfloat162 s2 = e8m0_bf16x2(sb[u]);
            uint32_t o[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint32_t pair = lut[(c[u] >> (8 * b)) & 0xFFu];
                __nv_bfloat162 v = __halves2bfloat162(__ushort_as_bfloat16(static_cast<unsigned short>(pair & 0xFFFFu)),
                                                      __ushort_as_bfloat16(static_cast<unsigned short>(pair >> 16)));
                o[b] = bf162_bits(__hmul2(v, s2));   // exact: a power-of-two scaling of a 2-bit significand
            }
            __stcs(out + t, make_uint4(o[0], o[1], o[2], o[3]));
        }
    }
}

using namespace pipe;

// ---------------------------------------------------------------- undo the transform
//
// out = (v * R^T) * Lambda, v = E2M1(code) * 2^e.
// The same flat group-major pipeline as rotate_flat_kernel, run backwards.
//   TMA warp    bulk-copies each stage's codes (512 groups x 16 B = 8 KB, contiguous) and,
//               when the copy can be 16-byte aligned, the stage's 512 scale bytes into a
//               3-deep shared-memory ring (a scale byte fetched from global memory just
//               before its use would expose a DRAM round trip every stage)
//   decoders    eight warps, two per scheduler: each lane takes one group per pass,
//               reads its 16 code bytes (and, with Lambda, its scale byte) from the ring,
//               decodes them with byte permutes (no table, so no bank conflicts), with Lambda
//               scales them by 2^e, and writes the MMA's A tile (bf16, 64-byte swizzle).  The
//               values are exact in bf16: two significant bits times a power of two.  Without
//               Lambda the epilogue applies 2^e to the fp32 sums instead (exact, the same
//               values), which moves work off the decoders, that form's critical path.
//   MMA warp    D[g][k] = sum_n v[g][n] * R^[k][n], so B is R^ as stored (row k,
//               contiguous n = K-major)
//   epilogue    eight warps in two groups of four (one warp per TMEM lane quarter), the
//               groups taking alternate stages: times Lambda_k, bf16, per-warp 2 KB TMA
//               stores.  Four warps, one per lane quarter, left the epilogue the critical
//               path.

// Lambda reaches the epilogue in one of two ways.  When all of it fits 64 KB (cols <=
// 16384) and is 16-byte aligned it is copied into shared memory once per CTA; each
// lane then reads its group's 32 channels from there (the group's row in Lambda
// viewed as [G][32] is its index mod G).  Otherwise each epilogue warp fetches the
// Lambda rows of its 32 groups per MMA into a double buffer (the rows of one
// 128-group MMA hold 128 consecutive column groups, so this is 128 B per group from
// L2).  The warp split: 8 epilogue warps and 8 decoders (18 warps with the MMA and TMA
// warps), except with per-warp fetches, whose registers allow 8 epilogue warps and 4
// decoders (14 warps).
template <int kLam>
struct DqSplit {
    static constexpr int kEpi = 8;
    static constexpr int kDec0 = kEpi;
    static constexpr int kDec = kLam == 1 ? 4 : 8;
    static constexpr int kMma = kDec0 + kDec;
    static constexpr int kTma = kMma + 1;
    static constexpr int kThreads = (kTma + 1) * 32;
};
constexpr int kDqStages = 3;
constexpr int kDqStageGroups = 512;                 // 4 MMAs of 128 groups
constexpr int kDqStageBytes = kDqStageGroups * 64;
constexpr int kDqCStages = 3;                       // codes ring
constexpr int kDqCodeBytes = kDqStageGroups * 16;   // 8 KB of codes per stage
constexpr int kDqCSlotBytes = kDqCodeBytes + kDqStageGroups;   // a ring slot: the codes, then the scale bytes
constexpr int kDqAcc = 4;
constexpr int kDqAccCols = 128;
constexpr int kDqOutBuf = 32 * 64;                 // one epilogue warp's 32 output groups (2 KB)
constexpr int kDqOutBufs = 2;                      // staging buffers per epilogue warp (4 measured no faster)
__host__ __device__ constexpr int dq_out_bytes(int epi) { return epi * kDqOutBufs * kDqOutBuf; }
// Lambda space: per warp, the rows of 32 groups double-buffered; or the whole resident table
__host__ __device__ constexpr int dq_lam_bytes(int epi, int lam)
{
    return lam == 2 ? 512 * 128 : (lam == 1 ? epi * 2 * 32 * 128 : 0);
}
__host__ __device__ constexpr int dq_smem_bytes(int epi, int lam)
{
    return kDqStages * kDqStageBytes + kBMatBytes + kDqCStages * kDqCSlotBytes + dq_out_bytes(epi) +
           dq_lam_bytes(epi, lam) + 512 + 128 + 1024;
}
static_assert(dq_smem_bytes(DqSplit<0>::kEpi, 0) <= 232448 && dq_smem_bytes(DqSplit<1>::kEpi, 1) <= 232448 &&
                  dq_smem_bytes(DqSplit<2>::kEpi, 2) <= 232448,
              "shared memory budget");
static_assert(kEpiWarps / 2 == 4, "acc_empty completes with four arrivals: one epilogue warp per lane quarter");

__device__ __forceinline__ uint32_t hmul2_bits(uint32_t a, __nv_bfloat162 s)
{
    const __nv_bfloat162 v = __halves2bfloat162(__ushort_as_bfloat16(static_cast<unsigned short>(a & 0xFFFFu)),
                                                __ushort_as_bfloat16(static_cast<unsigned short>(a >> 16)));
    const __nv_bfloat162 r = __hmul2(v, s);
    return static_cast<uint32_t>(__bfloat16_as_ushort(__low2bfloat16(r))) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(__high2bfloat16(r))) << 16);
}

// kLam: 0 no Lambda; 1 Lambda rows fetched per warp and MMA (any width); 2 all of Lambda
// resident in shared memory for the whole kernel (G <= kDqLamTableRows, 16-byte aligned).
constexpr int kDqLamTableRows = 512;   // 64 KB: cols <= 16384
template <int kLam>
__global__ void __launch_bounds__(DqSplit<kLam>::kThreads, 1)
    dequant_rot_kernel(const __grid_constant__ CUtensorMap tmap_out, const uint4 *__restrict__ codes,
                       const uint8_t *__restrict__ scales, int64_t n_groups, int64_t G,
                       const uint16_t *__restrict__ rhat, const float *__restrict__ lambda, unsigned int *status)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *stages = align_1k(smem_raw);
    uint8_t *bmat = stages + kDqStages * kDqStageBytes;
    uint8_t *cring = bmat + kBMatBytes;                                  // codes ring
    constexpr bool kLambda = kLam != 0;
    using W = DqSplit<kLam>;
    uint8_t *outbuf = cring + kDqCStages * kDqCSlotBytes;                 // epilogue staging
    uint8_t *lambuf = outbuf + dq_out_bytes(W::kEpi);                    // epilogue Lambda rows
    Bars *bars = reinterpret_cast<Bars *>(lambuf + dq_lam_bytes(W::kEpi, kLam));
    uint64_t *c_full = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(bars) + 512);
    uint64_t *c_empty = c_full + kDqCStages;
    volatile int *abort = &bars->abort;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_chunks = static_cast<int>((n_groups + kDqStageGroups - 1) / kDqStageGroups);

    if (threadIdx.x == 0) {   // the codes ring's barriers (kernel_setup fences every init)
        for (int s = 0; s < kDqCStages; ++s) {
            ptx::mbar_init(ptx::smem_addr(&c_full[s]), 1);
            ptx::mbar_init(ptx::smem_addr(&c_empty[s]), W::kDec);
        }
    }
    const uint32_t tmem_base = kernel_setup(
        bars, SetupCfg{kDqStages, kDqAcc, W::kDec, W::kDec * 32, W::kMma}, &tmap_out, nullptr);

    if (warp == W::kTma) {
        if (lane == 0) {
            const uint64_t pol = ptx::policy_evict_first();
            int it = 0;
            for (int c = blockIdx.x; c < n_chunks; c += gridDim.x, ++it) {
                const int cs = it % kDqCStages;
                if (!wait_bar(&c_empty[cs], ((it / kDqCStages) & 1) ^ 1, abort, status)) break;
                const int64_t g0 = static_cast<int64_t>(c) * kDqStageGroups;
                const int64_t n = n_groups - g0 < kDqStageGroups ? n_groups - g0 : kDqStageGroups;
                const uint32_t bar = ptx::smem_addr(&c_full[cs]);
                // the stage's scale bytes ride along when that copy can be 16-byte aligned (without
                // Lambda the epilogue applies the scales and fetches them itself)
                const bool sc_bulk =
                    kLambda && ((reinterpret_cast<uintptr_t>(scales + g0) & 15) == 0) && (n % 16) == 0;
                ptx::mbar_arrive_expect_tx(bar, static_cast<uint32_t>(n) * (sc_bulk ? 17u : 16u));
                ptx::bulk_load(ptx::smem_addr(cring + cs * kDqCSlotBytes), codes + g0, static_cast<uint32_t>(n) * 16u,
                               bar, pol);
                if (sc_bulk)
                    ptx::bulk_load(ptx::smem_addr(cring + cs * kDqCSlotBytes + kDqCodeBytes), scales + g0,
                                   static_cast<uint32_t>(n), bar, pol);
            }
            for (int cs = 0; cs < kDqCStages && cs < it; ++cs) {   // the last copies land before exit
                const int last = it - 1 - ((it - 1 - cs) % kDqCStages);
                wait_bar(&c_full[cs], (last / kDqCStages) & 1, nullptr, status);
            }
        }
    } else if (warp >= W::kDec0 && warp < W::kDec0 + W::kDec) {
        const int dt = threadIdx.x - W::kDec0 * 32;   // 0 .. 32 kDec - 1
        // B: row k holds R^[k][0..31] (bf16) in the first 64 B of a 128-byte-swizzled row
        if (dt < 32 * 4) {
            const int k = dt >> 2, c = dt & 3;
            const uint4 v = *reinterpret_cast<const uint4 *>(rhat + k * 32 + c * 8);
            *reinterpret_cast<uint4 *>(bmat + sw128(k, c)) = v;
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(ptx::smem_addr(&bars->b_full[0]));
        constexpr int kPer = kDqStageGroups / (W::kDec * 32);   // groups per lane per stage
        int it = 0;
        for (int c = blockIdx.x; c < n_chunks; c += gridDim.x, ++it) {
            const int s = it % kDqStages, cs = it % kDqCStages;
            const int64_t g0 = static_cast<int64_t>(c) * kDqStageGroups;
            // the scale bytes: from the ring when the TMA warp copied them (the same test it
            // made), otherwise fetched now, in flight while this warp waits
            const int64_t n_st = n_groups - g0 < kDqStageGroups ? n_groups - g0 : kDqStageGroups;
            const bool sc_bulk =
                kLambda && ((reinterpret_cast<uintptr_t>(scales + g0) & 15) == 0) && (n_st % 16) == 0;
            uint32_t sb[kPer] = {};
            if (kLambda && !sc_bulk) {
#pragma unroll
                for (int i = 0; i < kPer; ++i) {
                    const int64_t g = g0 + dt + i * W::kDec * 32;
                    sb[i] = g < n_groups ? static_cast<uint32_t>(__ldg(scales + g)) : 0u;
                }
            }
            int ok = 0;
            if (lane == 0)
                ok = wait_bar(&c_full[cs], (it / kDqCStages) & 1, abort, status) &&
                     wait_bar(&bars->empty[s], ((it / kDqStages) & 1) ^ 1, abort, status);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            const uint32_t st = ptx::smem_addr(stages + s * kDqStageBytes);
            const uint32_t cr = ptx::smem_addr(cring + cs * kDqCSlotBytes);
            if (sc_bulk) {
#pragma unroll
                for (int i = 0; i < kPer; ++i) sb[i] = ptx::ld_shared_u8(cr + kDqCodeBytes + dt + i * W::kDec * 32);
            }
#pragma unroll
            for (int i = 0; i < kPer; ++i) {
                const int r = dt + i * W::kDec * 32;   // group row within the stage
                uint32_t w[16];
                if (g0 + r < n_groups) {
                    const uint4 cw = ptx::ld_shared_v4(cr + r * 16);
                    const uint32_t byte = sb[i];
                    const uint32_t sbits = byte == 0xFFu ? 0x7FC0u : (byte == 0u ? 0x0040u : (byte << 7));
                    const __nv_bfloat162 s2 =
                        __halves2bfloat162(__ushort_as_bfloat16(static_cast<unsigned short>(sbits)),
                                           __ushort_as_bfloat16(static_cast<unsigned short>(sbits)));
                    const uint32_t cws[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t v[4];
                        ptx::e2m1x8_to_bf16(cws[q], v);
                        // without Lambda the E2M1 values go in as they are and the epilogue
                        // multiplies the fp32 result by 2^e (the decoders are that form's
                        // critical path, the epilogue has room); with Lambda the decoders scale
#pragma unroll
                        for (int e = 0; e < 4; ++e) w[4 * q + e] = kLambda ? hmul2_bits(v[e], s2) : v[e];
                    }
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
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&c_empty[cs]));   // this warp's reads of the ring are done
            ptx::fence_proxy_async_smem();   // each lane's A writes, then one arrival per warp
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&bars->full[s]));
        }
    } else if (warp == W::kMma) {
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
    } else if (warp < W::kEpi) {
        // Each warp stages its 32 groups' outputs (2 KB, 64-byte swizzle) and writes them
        // with one TMA bulk tensor store: 2 KB contiguous instead of 16-byte pieces.
        const int q = warp & 3;     // TMEM lane quarter
        const int ewg = warp >> 2;  // with 8 epilogue warps, the two groups take alternate stages
        const uint32_t obuf0 = ptx::smem_addr(outbuf + warp * kDqOutBufs * kDqOutBuf);
        const bool lam_vec = kLambda && ((reinterpret_cast<uintptr_t>(lambda) & 15) == 0);
        float *lrows2 = reinterpret_cast<float *>(lambuf + warp * 2 * 32 * 128);   // 2 x (32 rows x 32 channels)
        const int Gi = static_cast<int>(G);
        if constexpr (kLam == 2) {
            // Lambda as [G][32] once, 16-byte chunk c of row r at chunk c ^ (r & 7): the lanes of
            // a warp read consecutive rows (mod G), so a float4 read takes the minimum 4 wavefronts
            for (int i = threadIdx.x; i < Gi * 8; i += W::kEpi * 32) {
                const int r = i >> 3, cc = i & 7;
                ptx::cp_async16(ptx::smem_addr(lambuf + r * 128 + ((cc ^ (r & 7)) << 4)), lambda + r * 32 + cc * 4);
            }
            ptx::cp_async_commit();
            ptx::cp_async_wait<0>();
            ptx::named_bar_sync(1, W::kEpi * 32);
        }
        // Lambda rows by additions (no division per stage): the row of group g is g mod G, and
        // this lane's group (this warp's first, with per-warp fetches) advances by
        // kDqStageGroups x gridDim.x per CTA stage and by 128 per MMA.
        const int step_c = kLambda ? static_cast<int>((static_cast<int64_t>(kDqStageGroups) * gridDim.x) % G) : 0;
        const int step_j = kLambda ? static_cast<int>(128 % G) : 0;
        int row_c = kLambda ? static_cast<int>((static_cast<int64_t>(blockIdx.x) * kDqStageGroups + q * 32 +
                                                (kLam == 2 ? lane : 0)) % G)
                            : 0;
        int it = 0, nstore = 0;
        for (int c = blockIdx.x; c < n_chunks; c += gridDim.x, ++it) {
            const int row_stage = row_c;   // Lambda row of this stage's MMA 0 (lane's, or warp's first)
            if constexpr (kLambda) {
                row_c += step_c;
                if (row_c >= Gi) row_c -= Gi;
            }
            if (W::kEpi == 8 && (it & 1) != ewg) continue;
            const int a = it % kDqAcc;
            // without Lambda: this lane's group's scale byte for each of the stage's four MMAs,
            // in flight while the warp waits
            uint32_t esc[4] = {127u, 127u, 127u, 127u};
            if constexpr (!kLambda) {
                const int64_t gl = static_cast<int64_t>(c) * kDqStageGroups + q * 32 + lane;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (gl + j * 128 < n_groups) esc[j] = __ldg(scales + gl + j * 128);
            }
            int ok = 0;
            if (lane == 0) ok = wait_bar(&bars->acc_full[a], (it / kDqAcc) & 1, abort, status);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            ptx::tc_fence_after();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * kDqAccCols;
            const int64_t g_warp = static_cast<int64_t>(c) * kDqStageGroups + q * 32;
            // Lambda of the 32 groups of MMA j: rows (g % G) of Lambda viewed as [G][32],
            // copied into buffer (j & 1) with 16-byte chunks XOR-swizzled by row (8 lanes per
            // 128-byte row).  With a 16-byte-aligned Lambda the copies are asynchronous and the
            // next MMA's rows are in flight while this one is processed.
            // Column groups are taken mod G by subtraction (at most one step once G >= 128): a
            // division per stage instead of nine per fetch.
            const int col_warp = kLam == 1 ? row_stage : 0;
            int rj = kLam == 2 ? row_stage : 0;   // this lane's Lambda row for MMA j, advanced per MMA
            auto fetch_lambda = [&](int j) {
                int col0 = col_warp;
                for (int t = 0; t < j; ++t) {
                    col0 += step_j;
                    if (col0 >= Gi) col0 -= Gi;
                }
                float *dst_rows = lrows2 + (j & 1) * 32 * 32;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = 4 * i + (lane >> 3), cc = lane & 7;
                    int cg = col0 + r;
                    while (cg >= Gi) cg -= Gi;
                    const float *src = lambda + static_cast<int64_t>(cg) * 32 + cc * 4;
                    float *dst = dst_rows + r * 32 + ((cc ^ (r & 7)) << 2);
                    if (lam_vec) {
                        ptx::cp_async16(ptx::smem_addr(dst), src);
                    } else {
                        dst[0] = __ldg(src);
                        dst[1] = __ldg(src + 1);
                        dst[2] = __ldg(src + 2);
                        dst[3] = __ldg(src + 3);
                    }
                }
                ptx::cp_async_commit();
            };
            if constexpr (kLam == 1) {
                __syncwarp();   // the previous stage's reads of both buffers are done
                fetch_lambda(0);
            }
            // Two register buffers: MMA j + 1's TMEM rows are in flight while MMA j's are converted
            // and stored (with Lambda fetched per warp, one buffer: that form's registers are full).
            uint32_t rbuf[2][32];
            if constexpr (kLam != 1) {
                ptx::tmem_ld_32cols(t_row, rbuf[0]);
                ptx::tmem_wait_ld();
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t(&cur)[32] = rbuf[j & 1];
                if constexpr (kLam != 1) {
                    if (j + 1 < 4) ptx::tmem_ld_32cols(t_row + (j + 1) * 32, rbuf[(j + 1) & 1]);
                } else {
                    ptx::tmem_ld_32cols(t_row + j * 32, cur);
                }
                const int64_t g0 = g_warp + j * 128;   // this warp's first group of MMA j
                const float *lrows = lrows2 + (j & 1) * 32 * 32;
                if constexpr (kLam == 1) {
                    if (j + 1 < 4) {
                        __syncwarp();   // every lane is done reading buffer (j + 1) & 1 (MMA j - 1)
                        fetch_lambda(j + 1);
                        ptx::cp_async_wait<1>();   // MMA j's rows have landed
                    } else {
                        ptx::cp_async_wait<0>();
                    }
                    __syncwarp();
                }
                const float *ltab = reinterpret_cast<const float *>(lambuf) + rj * 32;
                if constexpr (kLam == 1) ptx::tmem_wait_ld();
                // times Lambda_k (channels of this group, two per packed multiply), then round to
                // bf16 pairs; without Lambda the fp32 values are rounded as they are
                uint32_t o[16];
                // 2^(byte - 127) as fp32 (byte 0 is the subnormal 2^-127, 0xFF is NaN): the sums
                // of exact products times a power of two, the same fp32 values as summing the
                // scaled products
                const uint32_t eb = esc[j];
                const float esf = __uint_as_float(eb == 0xFFu ? 0x7FC00000u : (eb == 0u ? 0x00400000u : (eb << 23)));
                const float2 es2 = make_float2(esf, esf);
#pragma unroll
                for (int k4 = 0; k4 < 8; ++k4) {
                    float2 v0 = make_float2(__uint_as_float(cur[4 * k4]), __uint_as_float(cur[4 * k4 + 1]));
                    float2 v1 = make_float2(__uint_as_float(cur[4 * k4 + 2]), __uint_as_float(cur[4 * k4 + 3]));
                    if constexpr (!kLambda) {
                        v0 = __fmul2_rn(v0, es2);
                        v1 = __fmul2_rn(v1, es2);
                    }
                    if constexpr (kLambda) {
                        const float4 l4 =
                            kLam == 1 ? *reinterpret_cast<const float4 *>(lrows + lane * 32 + ((k4 ^ (lane & 7)) << 2))
                                      : *reinterpret_cast<const float4 *>(ltab + ((k4 ^ (rj & 7)) << 2));
                        v0 = __fmul2_rn(v0, make_float2(l4.x, l4.y));
                        v1 = __fmul2_rn(v1, make_float2(l4.z, l4.w));
                    }
                    o[2 * k4] = bf162_bits(__floats2bfloat162_rn(v0.x, v0.y));
                    o[2 * k4 + 1] = bf162_bits(__floats2bfloat162_rn(v1.x, v1.y));
                }
                const uint32_t buf = obuf0 + (nstore % kDqOutBufs) * kDqOutBuf;
                // the buffer's previous store (kDqOutBufs stores ago) must have been read
                if (lane == 0) ptx::bulk_wait_group_read<kDqOutBufs - 1>();
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
                if constexpr (kLam != 1) {
                    if (j + 1 < 4) ptx::tmem_wait_ld();   // MMA j + 1's rows, for the next pass
                }
                if constexpr (kLam == 2) {
                    rj += step_j;
                    if (rj >= Gi) rj -= Gi;
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&bars->acc_empty[a]));
        }
        if (lane == 0) ptx::bulk_wait_group0();   // stores done before the CTA's shared memory goes
    }
    kernel_teardown(tmem_base, W::kMma);
}


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
    if (!lambda)
        return launch_pdl(dequant_rot_kernel<0>, grid, DqSplit<0>::kThreads, dq_smem_bytes(DqSplit<0>::kEpi, 0), stream,
                          tmap_out, c4, scales, n_groups, G, rhat, lambda, status);
    // all of Lambda fits the per-warp buffers' space (and can be copied in 16-byte pieces): keep it resident
    if (G <= kDqLamTableRows && (reinterpret_cast<uintptr_t>(lambda) & 15) == 0)
        return launch_pdl(dequant_rot_kernel<2>, grid, DqSplit<2>::kThreads, dq_smem_bytes(DqSplit<2>::kEpi, 2), stream,
                          tmap_out, c4, scales, n_groups, G, rhat, lambda, status);
    return launch_pdl(dequant_rot_kernel<1>, grid, DqSplit<1>::kThreads, dq_smem_bytes(DqSplit<1>::kEpi, 1), stream,
                      tmap_out, c4, scales, n_groups, G, rhat, lambda, status);
}

cudaError_t launch_dequant_plain(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t cols,
                                 uint16_t *out, int num_sms, cudaStream_t stream)
{
    const int64_t n_chunks = rows * cols / 8;
    if (n_chunks <= 0) return cudaSuccess;
    const int64_t want = (n_chunks + kPlainThreads - 1) / kPlainThreads;
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    const int grid = static_cast<int>(want < cap ? want : cap);
    dequant_plain_kernel<<<grid, kPlainThreads, 0, stream>>>(reinterpret_cast<const uint32_t *>(codes), scales,
                                                             n_chunks, reinterpret_cast<uint4 *>(out));
    return cudaGetLastError();
}

}  // namespace mxq
