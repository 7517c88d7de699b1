// rotquant_sm100.cu -- fused smooth -> rotate -> MXFP4-quantise kernel for B200 (sm_100a).
//
// Computes the online step of the DuQuant++ write-up (jsqmd.com/news/928156),
// X_hat = X * Lambda^-1 * R^ (§3.3), one 32x32 R^ shared by every 32-element group
// (§2.3, §3.2 step 4).  It then quantises each group to MXFP4 as in §2.1: absmax ->
// E8M0 scale -> divide -> nearest E2M1, under the OCP MX rule.  §5.2 item 1 asks for
// smoothing and rotation in one kernel; the quantiser is fused in too, so X is read
// once and only the packed codes and scales are written.
//
// Design (one persistent CTA per SM, warp-specialised):
//   * Tile = 128 rows x 128 columns (4 groups).  One TMA producer thread streams
//     tiles into a ring of shared-memory stages (two 64-column boxes per stage,
//     128-byte swizzle).
//   * One MMA thread issues tcgen05.mma (M=128, N=32, K=16, bf16 in, fp32 out).  Per
//     group: A = the group's 128x32 slice of the tile, B = R^ (K-major, i.e. R^T
//     row-major), D = 128 lanes x 32 fp32 columns of tensor memory.  Four
//     accumulator stages of 128 columns fill the 512 TMEM columns.
//   * With Lambda, the B operand of group g is diag(1/Lambda_g)·R^.  It is built
//     per tile in fp32 and split into three bf16 parts, high + middle + low
//     (three MMAs into the same accumulator, ~24 bits of B).  X stays the exact
//     bf16 A operand, and the smoothing adds only ~2^-25 relative error on top
//     of fp32 accumulation.  Two builder warps make these matrices into a
//     double-buffered slot.
//   * Eight epilogue warps (two groups of four; each group takes every other
//     tile).  tcgen05.ld 32x32b.x32 gives each thread one row's whole 32-value
//     group, so absmax, E8M0, scaling and the E2M1 conversion are thread-local.
//     The thread puts the 16 code bytes of each group into a shared-memory
//     staging tile (128 rows x 64 B, 64-byte swizzle).  One thread then writes
//     the tile with a single TMA bulk tensor store: 64 contiguous bytes per
//     row, instead of 32 scattered 16-byte pieces per warp instruction.  The
//     scattered form flooded the L2 with partial-sector writes.  The four
//     scale bytes of a row go out with one 32-bit store.
//   * Every mbarrier wait is bounded in time.  If one runs out, the kernel sets
//     the device status word, lets every role leave its loop, drains its own
//     copies and MMAs (again bounded), frees TMEM and returns.
#include <cuda_bf16.h>

#include "mxq_internal.h"
#include "sm100_ptx.cuh"

namespace mxq {

__device__ unsigned int g_status;

namespace {

constexpr int kTileG = 4;                              // groups per tile
constexpr int kStageBytes = kTileM * kTileCols * 2;    // 32 KB of bf16 per stage
constexpr int kBoxBytes = kStageBytes / 2;             // one TMA box: 128 rows x 128 B
constexpr int kAccStages = 4;
constexpr uint32_t kTmemCols = kAccStages * kTileCols; // 512
constexpr int kEpiWarps = 8;
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kBuildWarp0 = 10;
constexpr int kBuildWarps = 2;
constexpr int kThreads = (kEpiWarps + 2 + kBuildWarps) * 32;   // 384
constexpr int kBMatBytes = 32 * 128;                   // one B atom: 32 rows (n) x 128 B
// With Lambda a tile's B slot holds, per group j, an atom [hi | mid] at j*4 KB and
// the low parts of groups 2p and 2p+1 side by side in the atom at 16 KB + p*4 KB.
constexpr int kBLoOffset = kTileG * kBMatBytes;
constexpr int kBSlotBytes = kBLoOffset + (kTileG / 2) * kBMatBytes;   // 24 KB
constexpr uint64_t kTimeoutNs = 2000000000ull;         // 2 s per wait

constexpr int kCodeTileBytes = kTileM * kTileG * 16;    // 128 rows x 64 B of packed codes

template <bool kLambda>
struct Cfg {
    static constexpr int kStages = kLambda ? 4 : 6;
    static constexpr int kBBytes = kLambda ? 2 * kBSlotBytes : kBMatBytes;
    static constexpr int kStageOffset = 2 * kCodeTileBytes;   // code staging tiles first (1 KB aligned)
    static constexpr int kBOffset = kStageOffset + kStages * kStageBytes;
    static constexpr int kRtOffset = kBOffset + kBBytes;
    static constexpr int kBarOffset = kRtOffset + 32 * 32 * 4;
    static constexpr int kSmemBytes = kBarOffset + 256 + 1024;   // + barrier block + alignment slack
};

struct Bars {
    uint64_t full[8];
    uint64_t empty[8];
    uint64_t acc_full[kAccStages];
    uint64_t acc_empty[kAccStages];
    uint64_t b_full[2];
    uint64_t b_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int eg_ok[2][2];   // per epilogue warp group, per tile parity: the leader's wait result
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// Bounded wait on an mbarrier phase.  False if the wait ran out or (when abort
// is non-null) another role has already aborted.  Drains at exit pass a null
// abort so they keep waiting, within the time bound, for work already in flight.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort,
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
                atomicOr(&g_status, kStatusTimeout);
                return false;
            }
        }
    }
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
    float u[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) u[i] = __fmul_rn(__uint_as_float(r[i]), s);
#pragma unroll
    for (int q = 0; q < 4; ++q)
        w[q] = ptx::cvt_e2m1x8(u[8 * q], u[8 * q + 1], u[8 * q + 2], u[8 * q + 3], u[8 * q + 4], u[8 * q + 5],
                               u[8 * q + 6], u[8 * q + 7]);
    return byte;
}

template <bool kLambda, RotOut kMode>
__global__ void __launch_bounds__(kThreads, 1)
    rotate_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_codes,
                  const RotArgs args)
{
    using C = Cfg<kLambda>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *code_tiles = smem;                       // one staging tile per epilogue warp group
    uint8_t *stages = smem + C::kStageOffset;
    uint8_t *bmat = smem + C::kBOffset;
    float *rt = reinterpret_cast<float *>(smem + C::kRtOffset);   // R^ as fp32, [n][k]
    Bars *bars = reinterpret_cast<Bars *>(smem + C::kBarOffset);
    volatile int *abort = &bars->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t rows = args.rows;
    const int64_t cols = args.cols;
    const int64_t G = cols / 32;
    const int n_ct = static_cast<int>((cols + kTileCols - 1) / kTileCols);
    const int n_rt = static_cast<int>((rows + kTileM - 1) / kTileM);
    const int num_tiles = n_ct * n_rt;

    // ---------------------------------------------------------------- set-up
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            ptx::mbar_init(ptx::smem_addr(&bars->full[s]), 1);
            ptx::mbar_init(ptx::smem_addr(&bars->empty[s]), 1);
        }
        for (int a = 0; a < kAccStages; ++a) {
            ptx::mbar_init(ptx::smem_addr(&bars->acc_full[a]), 1);
            ptx::mbar_init(ptx::smem_addr(&bars->acc_empty[a]), kEpiWarps / 2);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(ptx::smem_addr(&bars->b_full[s]), kBuildWarps * 32);
            ptx::mbar_init(ptx::smem_addr(&bars->b_empty[s]), 1);
        }
        ptx::mbar_init(ptx::smem_addr(&bars->drain), 1);
        bars->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kTmaWarp && lane == 0) {
        ptx::prefetch_tmap(&tmap_x);
        if constexpr (kMode == RotOut::Quant) ptx::prefetch_tmap(&tmap_codes);
    }
    if (warp == kMmaWarp) {
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

    // ---------------------------------------------------------------- roles
    if (warp == kTmaWarp) {
        if (lane == 0) {
            const uint64_t pol = ptx::policy_evict_first();
            int it = 0;
            for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
                const int s = it % C::kStages;
                const uint32_t ph = (it / C::kStages) & 1;
                if (!wait_bar(&bars->empty[s], ph ^ 1, abort)) break;
                const int rtile = tile / n_ct, ctile = tile % n_ct;
                const uint32_t full = ptx::smem_addr(&bars->full[s]);
                const uint32_t dst = ptx::smem_addr(stages + s * kStageBytes);
                ptx::mbar_arrive_expect_tx(full, kStageBytes);
                ptx::tma_load_2d(dst, &tmap_x, ctile * kTileCols, rtile * kTileM, full, pol);
                ptx::tma_load_2d(dst + kBoxBytes, &tmap_x, ctile * kTileCols + 64, rtile * kTileM, full,
                                 pol);
            }
            // Let the last copy into each stage land before the CTA can exit.
            for (int s = 0; s < C::kStages && s < it; ++s) {
                const int last = it - 1 - ((it - 1 - s) % C::kStages);
                wait_bar(&bars->full[s], (last / C::kStages) & 1, nullptr);
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, 32);
            const uint32_t b_base0 = ptx::smem_addr(bmat);
            // without smoothing, B is built once by the builder warps
            const bool b_ok = kLambda || wait_bar(&bars->b_full[0], 0, abort);
            int it = 0;
            for (int tile = blockIdx.x; b_ok && tile < num_tiles; tile += gridDim.x, ++it) {
                const int s = it % C::kStages;
                const int a = it % kAccStages;
                const int slot = it & 1;
                if (!wait_bar(&bars->full[s], (it / C::kStages) & 1, abort)) break;
                if (!wait_bar(&bars->acc_empty[a], ((it / kAccStages) & 1) ^ 1, abort)) break;
                if constexpr (kLambda) {
                    if (!wait_bar(&bars->b_full[slot], (it >> 1) & 1, abort)) break;
                }
                ptx::tc_fence_after();
                const uint32_t a_base = ptx::smem_addr(stages + s * kStageBytes);
                const uint32_t b_base = b_base0 + (kLambda ? slot * kBSlotBytes : 0);
                const uint32_t d_base = tmem_base + static_cast<uint32_t>(a * kTileCols);
#pragma unroll
                for (int j = 0; j < kTileG; ++j) {
                    const uint32_t a_j = a_base + (j >> 1) * kBoxBytes + (j & 1) * 64;
                    const uint32_t d_j = d_base + j * 32;
#pragma unroll
                    for (int kh = 0; kh < 2; ++kh) {
                        const uint64_t ad = ptx::smem_desc_sw128(a_j + kh * 32);
                        if constexpr (kLambda) {
                            // smallest part first; the first MMA of the group overwrites D
                            const uint32_t b_hi = b_base + j * kBMatBytes + kh * 32;
                            const uint32_t b_lo =
                                b_base + kBLoOffset + (j >> 1) * kBMatBytes + (j & 1) * 64 + kh * 32;
                            ptx::mma_bf16(d_j, ad, ptx::smem_desc_sw128(b_lo), idesc, kh);
                            ptx::mma_bf16(d_j, ad, ptx::smem_desc_sw128(b_hi + 64), idesc, 1);
                            ptx::mma_bf16(d_j, ad, ptx::smem_desc_sw128(b_hi), idesc, 1);
                        } else {
                            ptx::mma_bf16(d_j, ad, ptx::smem_desc_sw128(b_base + kh * 32), idesc, kh);
                        }
                    }
                }
                ptx::mma_commit(ptx::smem_addr(&bars->empty[s]));
                ptx::mma_commit(ptx::smem_addr(&bars->acc_full[a]));
                if constexpr (kLambda) ptx::mma_commit(ptx::smem_addr(&bars->b_empty[slot]));
            }
            // Every MMA this thread issued must finish before TMEM is freed.
            ptx::mma_commit(ptx::smem_addr(&bars->drain));
            wait_bar(&bars->drain, 0, nullptr);
        }
    } else if (warp >= kBuildWarp0) {
        // Builders: R^ in fp32, transposed to [n][k], then the B operand(s) of the MMA.
        const int bt = threadIdx.x - kBuildWarp0 * 32;
        for (int i = bt; i < 32 * 32; i += kBuildWarps * 32) {
            const int k = i >> 5, n = i & 31;
            rt[n * 32 + k] = __bfloat162float(__ushort_as_bfloat16(args.rhat[i]));
        }
        ptx::named_bar_sync(3, kBuildWarps * 32);
        if constexpr (!kLambda) {
            // B = R^ in K-major form (row n holds R^[0..31][n]), bf16, built once; signalled
            // through phase 0 of b_full[0].
            for (int t = bt; t < 32 * 4; t += kBuildWarps * 32) {
                const int n = t >> 2, c = t & 3;
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int k = c * 8 + 2 * e;
                    w[e] = static_cast<uint32_t>(args.rhat[k * 32 + n]) |
                           (static_cast<uint32_t>(args.rhat[(k + 1) * 32 + n]) << 16);
                }
                *reinterpret_cast<uint4 *>(bmat + sw128(n, c)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(ptx::smem_addr(&bars->b_full[0]));
        } else {
            int it = 0;
            for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
                const int slot = it & 1;
                if (!wait_bar(&bars->b_empty[slot], ((it >> 1) & 1) ^ 1, abort)) break;
                const int64_t ch_tile = static_cast<int64_t>(tile % n_ct) * kTileCols;
                uint8_t *bs = bmat + slot * kBSlotBytes;
                // 4 groups x 32 rows (n) x 4 chunks of 8 k = 512 chunk tasks.
                for (int task = bt; task < kTileG * 32 * 4; task += kBuildWarps * 32) {
                    const int j = task >> 7, n = (task >> 2) & 31, c = task & 3;
                    const int64_t ch0 = ch_tile + j * 32 + c * 8;
                    uint32_t hw[4], mw[4], lw[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        __nv_bfloat16 h[2], m[2], l[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int k = c * 8 + 2 * e + u;
                            const int64_t ch = ch0 + 2 * e + u;
                            const float val =
                                ch < cols ? __fdiv_rn(rt[n * 32 + k], args.lambda[ch]) : 0.0f;
                            // val = hi + mid + lo to ~24 bits; each residual is exact in fp32
                            h[u] = __float2bfloat16_rn(val);
                            const float r1 = val - __bfloat162float(h[u]);
                            m[u] = __float2bfloat16_rn(r1);
                            l[u] = __float2bfloat16_rn(r1 - __bfloat162float(m[u]));
                        }
                        hw[e] = pack_bf16x2(h[0], h[1]);
                        mw[e] = pack_bf16x2(m[0], m[1]);
                        lw[e] = pack_bf16x2(l[0], l[1]);
                    }
                    uint8_t *bm = bs + j * kBMatBytes;
                    uint8_t *bl = bs + kBLoOffset + (j >> 1) * kBMatBytes;
                    *reinterpret_cast<uint4 *>(bm + sw128(n, c)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    *reinterpret_cast<uint4 *>(bm + sw128(n, c + 4)) =
                        make_uint4(mw[0], mw[1], mw[2], mw[3]);
                    *reinterpret_cast<uint4 *>(bl + sw128(n, c + 4 * (j & 1))) =
                        make_uint4(lw[0], lw[1], lw[2], lw[3]);
                }
                ptx::fence_proxy_async_smem();
                ptx::mbar_arrive(ptx::smem_addr(&bars->b_full[slot]));
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;       // TMEM lane quarter this warp may access
        const int ewg = warp >> 2;    // which half of the tiles this warp group takes
        const bool scale_vec = (G % 4 == 0) && ((reinterpret_cast<uintptr_t>(args.scales) & 3) == 0);
        const uint32_t ctile_smem = ptx::smem_addr(code_tiles + ewg * kCodeTileBytes);
        const bool leader = (warp & 3) == 0 && lane == 0;   // issues this warp group's code stores
        int it = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
            if ((it & 1) != ewg) continue;
            const int a = it % kAccStages;
            // The leader alone waits (bounded) and hands the verdict to its warp group through a
            // named barrier, so the four warps leave the loop together or not at all.
            volatile int *ok_slot = &bars->eg_ok[ewg][(it >> 1) & 1];
            if (leader) {
                int ok = wait_bar(&bars->acc_full[a], (it / kAccStages) & 1, abort);
                // the staging tile must have been read by this group's previous store
                if constexpr (kMode == RotOut::Quant) ptx::bulk_wait_group_read0();
                *ok_slot = ok;
            }
            __syncwarp();
            ptx::named_bar_sync(1 + ewg, 128);
            if (!*ok_slot) break;
            ptx::tc_fence_after();
            const int rtile = tile / n_ct, ctile = tile % n_ct;
            const int r_local = q * 32 + lane;
            const int64_t row = static_cast<int64_t>(rtile) * kTileM + r_local;
            const bool row_ok = row < rows;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(a * kTileCols);
            uint32_t sc_word = 0;
            // Two register buffers: the TMEM load of group j+1 is in flight while group j
            // is quantised.  Fully unrolled so both buffers stay in fixed registers.
            uint32_t ra[32], rb[32];
            ptx::tmem_ld_32cols(t_row, ra);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < kTileG; ++j) {
                uint32_t(&cur)[32] = (j & 1) ? rb : ra;
                uint32_t(&nxt)[32] = (j & 1) ? ra : rb;
                if (j + 1 < kTileG) ptx::tmem_ld_32cols(t_row + (j + 1) * 32, nxt);
                const int64_t g = static_cast<int64_t>(ctile) * kTileG + j;
                if constexpr (kMode == RotOut::F32) {
                    if (g < G && row_ok) {
                        float *dst = args.y + row * cols + g * 32;
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            ptx::st_global_v4(dst + 4 * i, cur[4 * i], cur[4 * i + 1], cur[4 * i + 2],
                                              cur[4 * i + 3]);
                    }
                } else {
                    uint32_t w[4];
                    const uint32_t byte = quantize_group(cur, w);
                    // 64-byte swizzle: 16-byte chunk j of row r sits at chunk j ^ ((r >> 1) & 3)
                    const uint32_t chunk = static_cast<uint32_t>(j) ^ ((static_cast<uint32_t>(r_local) >> 1) & 3u);
                    ptx::st_shared_v4(ctile_smem + r_local * 64 + chunk * 16, w[0], w[1], w[2], w[3]);
                    if (scale_vec)
                        sc_word |= byte << (8 * j);
                    else if (g < G && row_ok)
                        args.scales[row * G + g] = static_cast<uint8_t>(byte);
                }
                if (j + 1 < kTileG) ptx::tmem_wait_ld();
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&bars->acc_empty[a]));
            if constexpr (kMode == RotOut::Quant) {
                if (scale_vec && row_ok)
                    *reinterpret_cast<uint32_t *>(args.scales + row * G +
                                                  static_cast<int64_t>(ctile) * kTileG) = sc_word;
                // staging tile complete -> one bulk store (rows/columns past the tensor are clipped)
                ptx::fence_proxy_async_smem();
                __syncwarp();
                ptx::named_bar_sync(1 + ewg, 128);
                if (leader) {
                    ptx::tma_store_2d(&tmap_codes, ctile * (kTileCols / 2), rtile * kTileM, ctile_smem);
                    ptx::bulk_commit_group();
                }
            }
        }
        if constexpr (kMode == RotOut::Quant) {
            if (leader) ptx::bulk_wait_group0();   // stores done before the CTA's shared memory goes
        }
    }

    // ---------------------------------------------------------------- teardown
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, kTmemCols);
    }
}

// Diagnostic: one thread waits on an mbarrier phase that nothing completes, so the
// bounded wait must run out, set the status word and return.  It exercises the
// same wait routine as the pipeline, without any TMA, MMA or TMEM in play.
__global__ void bounded_wait_selftest(uint64_t timeout_ns, int *result)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    abort_flag = 0;
    ptx::mbar_init(ptx::smem_addr(&bar), 1);
    ptx::fence_mbar_init();
    const bool ok = wait_bar(&bar, 0, &abort_flag, timeout_ns);
    *result = ok ? 1 : (abort_flag ? 2 : 3);
    // complete the phase so the barrier is not left mid-phase
    ptx::mbar_arrive(ptx::smem_addr(&bar));
}

template <bool kLambda, RotOut kMode>
cudaError_t launch_one(const CUtensorMap &tmap, const CUtensorMap &tmap_codes, const RotArgs &args, int grid,
                       cudaStream_t stream)
{
    auto kern = rotate_kernel<kLambda, kMode>;
    constexpr int smem = Cfg<kLambda>::kSmemBytes;
    static_assert(smem <= 232448, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    // Programmatic dependent launch: this grid may start while the previous kernel in the
    // stream drains; the kernel orders its global accesses with griddepcontrol.wait.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmap, tmap_codes, args);
}

}  // namespace

cudaError_t launch_rotate(const CUtensorMap &tmap_x, const CUtensorMap &tmap_codes, const RotArgs &args,
                          RotOut mode, int num_sms, cudaStream_t stream)
{
    const int64_t n_tiles = ((args.rows + kTileM - 1) / kTileM) * ((args.cols + kTileCols - 1) / kTileCols);
    if (n_tiles <= 0) return cudaSuccess;
    const int grid = static_cast<int>(n_tiles < num_sms ? n_tiles : num_sms);
    const bool lam = args.lambda != nullptr;
    if (mode == RotOut::Quant)
        return lam ? launch_one<true, RotOut::Quant>(tmap_x, tmap_codes, args, grid, stream)
                   : launch_one<false, RotOut::Quant>(tmap_x, tmap_codes, args, grid, stream);
    return lam ? launch_one<true, RotOut::F32>(tmap_x, tmap_codes, args, grid, stream)
               : launch_one<false, RotOut::F32>(tmap_x, tmap_codes, args, grid, stream);
}

cudaError_t launch_wait_selftest(uint64_t timeout_ns, int *result, cudaStream_t stream)
{
    bounded_wait_selftest<<<1, 32, 0, stream>>>(timeout_ns, result);
    return cudaGetLastError();
}

cudaError_t read_and_clear_status(unsigned int *host_status, cudaStream_t stream)
{
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(host_status, g_status, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_status, &zero, sizeof(unsigned int));
}

}  // namespace mxq
