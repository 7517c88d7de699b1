// rotquant_sm100.cu -- fused smooth -> rotate -> MXFP4-quantise kernels for B200 (sm_100a).
//
// They compute the online step of the DuQuant++ write-up (jsqmd.com/news/928156),
// X_hat = X * Lambda^-1 * R^ (§3.3), with one 32x32 R^ shared by every 32-element
// group (§2.3, §3.2 step 4).  Each group is then quantised to MXFP4 as in §2.1:
// absmax -> E8M0 scale -> divide -> nearest E2M1, under the OCP MX rule.  §5.2
// item 1 asks for the smoothing and the rotation in one kernel.  The quantiser is
// fused in too, so X is read once and only the packed codes and scales are written.
//
// Both kernels run one persistent CTA per SM and are warp-specialised:
//   warps 0-7   epilogue, two groups of four, each group taking every other stage
//   warp 8      TMA producer (one thread)
//   warp 9      TMEM allocator + MMA issuer (one thread)
//   warps 10-11 builders of the MMA's B operand (10-13 in the smoothing kernel)
// The rotation is a dense bf16 contraction on the tensor cores: tcgen05.mma
// M=128, N=32, K=16, fp32 accumulate.  A is 128 groups of X staged by TMA in
// shared memory, B = R^ in K-major form (R^T row-major), and D is 128 TMEM
// lanes x 32 columns.  Accumulator stages (32 columns per MMA) fill TMEM's 512
// columns.  The epilogue reads TMEM with tcgen05.ld 32x32b.x32, so each thread
// holds one group's 32 rotated values.  Absmax, E8M0, scaling and the E2M1
// conversion are therefore thread-local.
//
// Without Lambda (rotate_flat_kernel): X is a dense [rows*cols/32, 32] matrix,
// the reshape-and-bmm form of §3.3's implementation tips.  An MMA takes 128
// consecutive groups; a stage is kFlatMmas MMAs' worth, loaded as TMA boxes of
// 16 contiguous KB.  A warp's 32 lanes quantise 32 consecutive groups, so its code store
// covers 512 contiguous bytes and its scale store 32.  Loads and stores all
// stream through HBM in address order.
//
// With Lambda (rotate_cols_kernel): the B operand depends on the channel
// group, B_g = diag(1/Lambda_g)·R^, so an MMA must hold one column group over
// 128 token rows.  A tile is 128 rows x 128 columns (4 groups); tiles go round
// robin over the row-major tile list, so the CTAs together read whole rows.
// The builder warps make each tile's four B_g in fp32 and split them three
// ways into bf16, high + middle + low (three MMAs into one accumulator, ~24
// bits of B).  X stays
// the exact bf16 A operand, so the smoothing adds only ~2^-25 relative error on
// top of fp32 accumulation.  Codes go through a shared-memory staging tile and
// one TMA bulk tensor store per tile (64 contiguous bytes per row).
//
// Every mbarrier wait is bounded in time.  If one runs out, the kernel sets the
// device status word and every role leaves its loop.  The kernel then drains its
// own copies and MMAs (again bounded), frees TMEM and returns.  The kernels
// signal programmatic dependent launch at once and make no global access before
// griddepcontrol.wait, so the next launch's set-up overlaps this one's tail.
#include <cuda_bf16.h>

#include "mxq_internal.h"
#include "sm100_ptx.cuh"

namespace mxq {

__device__ unsigned int g_status;

namespace {

constexpr uint32_t kTmemCols = 512;      // all of TMEM: accumulator stages of 32 columns per MMA
constexpr int kMaxAcc = 8;
constexpr int kEpiWarps = 8;
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kBuildWarp0 = 10;
constexpr int kBuildWarps = 2;
constexpr int kThreads = (kEpiWarps + 2 + kBuildWarps) * 32;   // 384
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
    float u[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) u[i] = __fmul_rn(__uint_as_float(r[i]), s);
#pragma unroll
    for (int q = 0; q < 4; ++q)
        w[q] = ptx::cvt_e2m1x8(u[8 * q], u[8 * q + 1], u[8 * q + 2], u[8 * q + 3], u[8 * q + 4], u[8 * q + 5],
                               u[8 * q + 6], u[8 * q + 7]);
    return byte;
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
__device__ __forceinline__ void drain_loads(Bars *bars, int n_stages, int issued)
{
    for (int s = 0; s < n_stages && s < issued; ++s) {
        const int last = issued - 1 - ((issued - 1 - s) % n_stages);
        wait_bar(&bars->full[s], (last / n_stages) & 1, nullptr);
    }
}

// MMA epilogue: every MMA this thread issued must finish before TMEM is freed.
__device__ __forceinline__ void drain_mmas(Bars *bars)
{
    ptx::mma_commit(ptx::smem_addr(&bars->drain));
    wait_bar(&bars->drain, 0, nullptr);
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

// =====================================================================================
// Without smoothing: X as a dense [n_groups, 32] matrix.
// =====================================================================================

constexpr int kFlatBoxGroups = 256;                        // one TMA box: 256 groups x 64 B = 16 KB
constexpr int kFlatMmas = 4;                               // MMAs (of 128 groups) per stage
constexpr int kFlatStageGroups = 128 * kFlatMmas;
constexpr int kFlatBoxes = kFlatStageGroups / kFlatBoxGroups;
constexpr int kFlatStageBytes = kFlatStageGroups * 64;
constexpr int kFlatStages = 3;                             // ~96 KB in flight per SM measured best
constexpr int kFlatAccCols = 32 * kFlatMmas;               // TMEM columns per accumulator stage
constexpr int kFlatAcc = (512 / kFlatAccCols) < kMaxAcc ? (512 / kFlatAccCols) : kMaxAcc;
constexpr int kFlatSmemBytes = kFlatStages * kFlatStageBytes + kBMatBytes + 512 + 1024;
static_assert(kFlatBoxes >= 1 && kFlatStageGroups % kFlatBoxGroups == 0 && kFlatStages <= kMaxStages, "flat tiling");

template <RotOut kMode>
__global__ void __launch_bounds__(kThreads, 1)
    rotate_flat_kernel(const __grid_constant__ CUtensorMap tmap_g, const RotArgs args)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *stages = align_1k(smem_raw);
    uint8_t *bmat = stages + kFlatStages * kFlatStageBytes;
    Bars *bars = reinterpret_cast<Bars *>(bmat + kBMatBytes);
    volatile int *abort = &bars->abort;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t n_groups = args.rows * (args.cols / 32);
    const int n_chunks = static_cast<int>((n_groups + kFlatStageGroups - 1) / kFlatStageGroups);

    const uint32_t tmem_base =
        kernel_setup(bars, SetupCfg{kFlatStages, kFlatAcc, 1, kBuildWarps * 32, kMmaWarp}, &tmap_g, nullptr);

    if (warp == kTmaWarp) {
        if (lane == 0) {
            const uint64_t pol = ptx::policy_evict_first();
            int it = 0;
            for (int c = blockIdx.x; c < n_chunks; c += gridDim.x, ++it) {
                const int s = it % kFlatStages;
                if (!wait_bar(&bars->empty[s], ((it / kFlatStages) & 1) ^ 1, abort)) break;
                const uint32_t full = ptx::smem_addr(&bars->full[s]);
                const uint32_t dst = ptx::smem_addr(stages + s * kFlatStageBytes);
                const int g0 = c * kFlatStageGroups;
                ptx::mbar_arrive_expect_tx(full, kFlatStageBytes);
#pragma unroll
                for (int b = 0; b < kFlatBoxes; ++b)
                    ptx::tma_load_2d(dst + b * kFlatBoxGroups * 64, &tmap_g, 0, g0 + b * kFlatBoxGroups, full, pol);
            }
            drain_loads(bars, kFlatStages, it);
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, 32);
            const uint32_t b_base = ptx::smem_addr(bmat);
            const bool b_ok = wait_bar(&bars->b_full[0], 0, abort);   // B is built once
            int it = 0;
            for (int c = blockIdx.x; b_ok && c < n_chunks; c += gridDim.x, ++it) {
                const int s = it % kFlatStages;
                const int a = it % kFlatAcc;
                if (!wait_bar(&bars->full[s], (it / kFlatStages) & 1, abort)) break;
                if (!wait_bar(&bars->acc_empty[a], ((it / kFlatAcc) & 1) ^ 1, abort)) break;
                ptx::tc_fence_after();
                const uint32_t a_base = ptx::smem_addr(stages + s * kFlatStageBytes);
                const uint32_t d_base = tmem_base + static_cast<uint32_t>(a * kFlatAccCols);
#pragma unroll
                for (int j = 0; j < kFlatMmas; ++j) {
#pragma unroll
                    for (int kh = 0; kh < 2; ++kh)
                        ptx::mma_bf16(d_base + j * 32, ptx::smem_desc_sw64(a_base + j * 128 * 64 + kh * 32),
                                      ptx::smem_desc_sw128(b_base + kh * 32), idesc, kh);
                }
                ptx::mma_commit(ptx::smem_addr(&bars->empty[s]));
                ptx::mma_commit(ptx::smem_addr(&bars->acc_full[a]));
            }
            drain_mmas(bars);
        }
    } else if (warp >= kBuildWarp0) {
        // B = R^ in K-major form: row n holds R^[0..31][n] (bf16, first 64 B of a 128-B row).
        const int bt = threadIdx.x - kBuildWarp0 * 32;
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
        const int q = warp & 3;       // TMEM lane quarter this warp may access
        const int ewg = warp >> 2;    // which half of the stages this warp group takes
        int it = 0;
        for (int c = blockIdx.x; c < n_chunks; c += gridDim.x, ++it) {
            if ((it & 1) != ewg) continue;
            const int a = it % kFlatAcc;
            int ok = 0;
            if (lane == 0) ok = wait_bar(&bars->acc_full[a], (it / kFlatAcc) & 1, abort);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            ptx::tc_fence_after();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * kFlatAccCols;
            const int64_t g_lane = static_cast<int64_t>(c) * kFlatStageGroups + q * 32 + lane;
            // The TMEM load of MMA j+1 is in flight while group j is quantised; fully
            // unrolled so both register buffers stay put.
            uint32_t ra[32], rb[32];
            ptx::tmem_ld_32cols(t_row, ra);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < kFlatMmas; ++j) {
                uint32_t(&cur)[32] = (j & 1) ? rb : ra;
                uint32_t(&nxt)[32] = (j & 1) ? ra : rb;
                if (j + 1 < kFlatMmas) ptx::tmem_ld_32cols(t_row + (j + 1) * 32, nxt);
                const int64_t g = g_lane + j * 128;
                if (g < n_groups) {
                    if constexpr (kMode == RotOut::F32) {
                        float *dst = args.y + g * 32;
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            ptx::st_global_v4(dst + 4 * i, cur[4 * i], cur[4 * i + 1], cur[4 * i + 2],
                                              cur[4 * i + 3]);
                    } else {
                        uint32_t w[4];
                        const uint32_t byte = quantize_group(cur, w);
                        ptx::st_global_v4(args.codes + g * 16, w[0], w[1], w[2], w[3]);
                        args.scales[g] = static_cast<uint8_t>(byte);
                    }
                }
                if (j + 1 < kFlatMmas) ptx::tmem_wait_ld();
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&bars->acc_empty[a]));
        }
    }
    kernel_teardown(tmem_base, kMmaWarp);
}

// =====================================================================================
// With smoothing: 128-row x 128-column tiles, per-tile B_g = diag(1/Lambda_g) R^.
// =====================================================================================

constexpr int kColTileG = 4;                                  // groups per tile
constexpr int kColAcc = 4;                                    // accumulator stages of 128 columns
constexpr int kColAccCols = 128;
constexpr int kColStageBytes = kTileM * kTileCols * 2;        // 32 KB of bf16 per stage
constexpr int kColBoxBytes = kColStageBytes / 2;              // one TMA box: 128 rows x 128 B
constexpr int kCodeTileBytes = kTileM * kColTileG * 16;       // 128 rows x 64 B of packed codes
// A tile's B slot holds, per group j, an atom [hi | mid] at j*4 KB and the low
// parts of groups 2p and 2p+1 side by side in the atom at 16 KB + p*4 KB.
constexpr int kBLoOffset = kColTileG * kBMatBytes;
constexpr int kBSlotBytes = kBLoOffset + (kColTileG / 2) * kBMatBytes;   // 24 KB
constexpr int kColStages = 4;
constexpr int kColStageOffset = 2 * kCodeTileBytes;           // code staging tiles first
constexpr int kColBOffset = kColStageOffset + kColStages * kColStageBytes;
constexpr int kColRtOffset = kColBOffset + 2 * kBSlotBytes;
constexpr int kColInvOffset = kColRtOffset + 32 * 32 * 4;     // per slot: 1/Lambda of the tile's 128 channels
constexpr int kColBarOffset = kColInvOffset + 2 * kTileCols * 8;
constexpr int kColSmemBytes = kColBarOffset + 512 + 1024;
constexpr int kColBuildWarps = 4;                             // warps 10-13
constexpr int kColThreads = (kEpiWarps + 2 + kColBuildWarps) * 32;   // 448

// Tile order of the smoothing kernel.  A unit is kUnitRows consecutive row
// blocks of one column tile, so one B_g build serves kUnitRows tiles.  Units are
// numbered band-major (u = band * n_ct + ct) and dealt round robin to the CTAs.
// At any moment the CTAs' units therefore cover whole rows of a couple of row
// bands, which DRAM reads well.  Only the last band can be shorter than
// kUnitRows, and a CTA meets it only in its last units, so a CTA's it-th tile
// has a closed form.
constexpr int kUnitRows = 4;

struct UnitSched {
    int n_ct, cta, grid, r_last, k_full, n_units_cta, n_tiles;
    __device__ UnitSched(int n_ct_, int n_rt, int cta_, int grid_) : n_ct(n_ct_), cta(cta_), grid(grid_)
    {
        const int n_bands = (n_rt + kUnitRows - 1) / kUnitRows;
        r_last = n_rt - (n_bands - 1) * kUnitRows;
        const int n_units = n_ct * n_bands;
        n_units_cta = cta < n_units ? (n_units - cta + grid - 1) / grid : 0;
        const int before_last = (n_bands - 1) * n_ct;   // units in full bands
        const int k = cta < before_last ? (before_last - cta + grid - 1) / grid : 0;
        k_full = k < n_units_cta ? k : n_units_cta;
        n_tiles = k_full * kUnitRows + (n_units_cta - k_full) * r_last;
    }
    // The it-th tile of this CTA: its unit's ordinal ui, the position in the unit and the unit's length.
    __device__ void at(int it, int &ui, int &sub, int &len) const
    {
        if (it < k_full * kUnitRows) {
            ui = it / kUnitRows;
            sub = it % kUnitRows;
            len = kUnitRows;
        } else {
            const int t = it - k_full * kUnitRows;
            ui = k_full + t / r_last;
            sub = t % r_last;
            len = r_last;
        }
    }
    __device__ int ct_of_unit(int ui) const { return (cta + ui * grid) % n_ct; }
    __device__ int rt0_of_unit(int ui) const { return ((cta + ui * grid) / n_ct) * kUnitRows; }
};

template <RotOut kMode>
__global__ void __launch_bounds__(kColThreads, 1)
    rotate_cols_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_codes,
                       const RotArgs args)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1k(smem_raw);
    uint8_t *code_tiles = smem;                       // one staging tile per epilogue warp group
    uint8_t *stages = smem + kColStageOffset;
    uint8_t *bmat = smem + kColBOffset;
    float *rt = reinterpret_cast<float *>(smem + kColRtOffset);   // R^ as fp32, [n][k]
    float2 *inv_tab = reinterpret_cast<float2 *>(smem + kColInvOffset);   // [slot][channel] (1/L, residual)
    Bars *bars = reinterpret_cast<Bars *>(smem + kColBarOffset);
    volatile int *abort = &bars->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t rows = args.rows;
    const int64_t cols = args.cols;
    const int64_t G = cols / 32;
    const int n_ct = static_cast<int>((cols + kTileCols - 1) / kTileCols);
    const int n_rt = static_cast<int>((rows + kTileM - 1) / kTileM);
    const UnitSched sched(n_ct, n_rt, blockIdx.x, gridDim.x);

    const uint32_t tmem_base =
        kernel_setup(bars, SetupCfg{kColStages, kColAcc, 1, kColBuildWarps * 32, kMmaWarp}, &tmap_x,
                     kMode == RotOut::Quant ? &tmap_codes : nullptr);

    if (warp == kTmaWarp) {
        if (lane == 0) {
            const uint64_t pol = ptx::policy_evict_first();
            int it = 0;
            for (; it < sched.n_tiles; ++it) {
                const int s = it % kColStages;
                if (!wait_bar(&bars->empty[s], ((it / kColStages) & 1) ^ 1, abort)) break;
                int ui, sub, len;
                sched.at(it, ui, sub, len);
                const int ctile = sched.ct_of_unit(ui), rtile = sched.rt0_of_unit(ui) + sub;
                const uint32_t full = ptx::smem_addr(&bars->full[s]);
                const uint32_t dst = ptx::smem_addr(stages + s * kColStageBytes);
                ptx::mbar_arrive_expect_tx(full, kColStageBytes);
                ptx::tma_load_2d(dst, &tmap_x, ctile * kTileCols, rtile * kTileM, full, pol);
                ptx::tma_load_2d(dst + kColBoxBytes, &tmap_x, ctile * kTileCols + 64, rtile * kTileM, full, pol);
            }
            drain_loads(bars, kColStages, it);
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, 32);
            const uint32_t b_base0 = ptx::smem_addr(bmat);
            for (int it = 0; it < sched.n_tiles; ++it) {
                const int s = it % kColStages;
                const int a = it % kColAcc;
                int ui, sub, len;
                sched.at(it, ui, sub, len);
                const int slot = ui & 1;
                if (!wait_bar(&bars->full[s], (it / kColStages) & 1, abort)) break;
                if (!wait_bar(&bars->acc_empty[a], ((it / kColAcc) & 1) ^ 1, abort)) break;
                if (sub == 0 && !wait_bar(&bars->b_full[slot], (ui >> 1) & 1, abort)) break;
                ptx::tc_fence_after();
                const uint32_t a_base = ptx::smem_addr(stages + s * kColStageBytes);
                const uint32_t b_base = b_base0 + slot * kBSlotBytes;
                const uint32_t d_base = tmem_base + static_cast<uint32_t>(a * kColAccCols);
#pragma unroll
                for (int j = 0; j < kColTileG; ++j) {
                    const uint32_t a_j = a_base + (j >> 1) * kColBoxBytes + (j & 1) * 64;
                    const uint32_t d_j = d_base + j * 32;
#pragma unroll
                    for (int kh = 0; kh < 2; ++kh) {
                        const uint64_t ad = ptx::smem_desc_sw128(a_j + kh * 32);
                        // smallest part first; the first MMA of the group overwrites D
                        const uint32_t b_hi = b_base + j * kBMatBytes + kh * 32;
                        const uint32_t b_lo = b_base + kBLoOffset + (j >> 1) * kBMatBytes + (j & 1) * 64 + kh * 32;
                        ptx::mma_bf16(d_j, ad, ptx::smem_desc_sw128(b_lo), idesc, kh);
                        ptx::mma_bf16(d_j, ad, ptx::smem_desc_sw128(b_hi + 64), idesc, 1);
                        ptx::mma_bf16(d_j, ad, ptx::smem_desc_sw128(b_hi), idesc, 1);
                    }
                }
                ptx::mma_commit(ptx::smem_addr(&bars->empty[s]));
                ptx::mma_commit(ptx::smem_addr(&bars->acc_full[a]));
                if (sub == len - 1) ptx::mma_commit(ptx::smem_addr(&bars->b_empty[slot]));
            }
            drain_mmas(bars);
        }
    } else if (warp >= kBuildWarp0) {
        // Builders: R^ in fp32, transposed to [n][k]; then per tile 1/Lambda of its 128
        // channels (a reciprocal plus its FMA residual, so R*(1/Lambda) is good to about
        // an ulp), then the four B_g = diag(1/Lambda_g) R^ split three ways into bf16.
        const int bt = threadIdx.x - kBuildWarp0 * 32;   // 0..127
        constexpr int kB = kColBuildWarps * 32;
        for (int i = bt; i < 32 * 32; i += kB) {
            const int k = i >> 5, n = i & 31;
            rt[n * 32 + k] = __bfloat162float(__ushort_as_bfloat16(args.rhat[i]));
        }
        ptx::named_bar_sync(3, kB);
        int built0 = -1, built1 = -1;   // column tile whose B_g each slot holds
        for (int ui = 0; ui < sched.n_units_cta; ++ui) {
            const int slot = ui & 1;
            // one thread waits (bounded) for the slot; the verdict goes to all builders
            // (the flag alternates per unit, so a slow reader never sees the next unit's value)
            if (bt == 0) bars->bl_ok[ui & 1] = wait_bar(&bars->b_empty[slot], ((ui >> 1) & 1) ^ 1, abort);
            __syncwarp();
            ptx::named_bar_sync(3, kB);
            if (!*reinterpret_cast<volatile int *>(&bars->bl_ok[ui & 1])) break;
            const int ct = sched.ct_of_unit(ui);
            if ((slot ? built1 : built0) != ct) {
                if (slot)
                    built1 = ct;
                else
                    built0 = ct;
                const int64_t ch_tile = static_cast<int64_t>(ct) * kTileCols;
                float2 *inv = inv_tab + slot * kTileCols;
                {
                    const int64_t ch = ch_tile + bt;
                    float ih = 0.0f, il = 0.0f;
                    if (ch < cols) {
                        const float lam = args.lambda[ch];
                        ih = __frcp_rn(lam);
                        il = __fmul_rn(__fmaf_rn(-lam, ih, 1.0f), ih);   // 1/lam - ih, to working precision
                    }
                    inv[bt] = make_float2(ih, il);
                }
                ptx::named_bar_sync(3, kB);
                uint8_t *bs = bmat + slot * kBSlotBytes;
                // 4 groups x 32 rows (n) x 4 chunks of 8 k = 512 chunk tasks.
                for (int task = bt; task < kColTileG * 32 * 4; task += kB) {
                    const int j = task >> 7, n = (task >> 2) & 31, c = task & 3;
                    uint32_t hw[4], mw[4], lw[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        __nv_bfloat16 h[2], m[2], l[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int k = c * 8 + 2 * e + u;
                            const float2 iv = inv[j * 32 + k];
                            const float r = rt[n * 32 + k];
                            const float val = __fmaf_rn(r, iv.x, __fmul_rn(r, iv.y));   // R / Lambda
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
                    *reinterpret_cast<uint4 *>(bm + sw128(n, c + 4)) = make_uint4(mw[0], mw[1], mw[2], mw[3]);
                    *reinterpret_cast<uint4 *>(bl + sw128(n, c + 4 * (j & 1))) =
                        make_uint4(lw[0], lw[1], lw[2], lw[3]);
                }
                ptx::fence_proxy_async_smem();
            }
            ptx::mbar_arrive(ptx::smem_addr(&bars->b_full[slot]));
        }
    } else {
        const int q = warp & 3;
        const int ewg = warp >> 2;
        const bool scale_vec = (G % 4 == 0) && ((reinterpret_cast<uintptr_t>(args.scales) & 3) == 0);
        const uint32_t ctile_smem = ptx::smem_addr(code_tiles + ewg * kCodeTileBytes);
        const bool leader = q == 0 && lane == 0;   // issues this warp group's code stores
        for (int it = ewg; it < sched.n_tiles; it += 2) {
            const int a = it % kColAcc;
            // The leader alone waits (bounded) and hands the verdict to its warp group through a
            // named barrier, so the four warps leave the loop together or not at all.
            volatile int *ok_slot = &bars->eg_ok[ewg][(it >> 1) & 1];
            if (leader) {
                int ok = wait_bar(&bars->acc_full[a], (it / kColAcc) & 1, abort);
                // the staging tile must have been read by this group's previous store
                if constexpr (kMode == RotOut::Quant) ptx::bulk_wait_group_read0();
                *ok_slot = ok;
            }
            __syncwarp();
            ptx::named_bar_sync(1 + ewg, 128);
            if (!*ok_slot) break;
            ptx::tc_fence_after();
            int ui, sub, len;
            sched.at(it, ui, sub, len);
            const int ctile = sched.ct_of_unit(ui), rtile = sched.rt0_of_unit(ui) + sub;
            const int r_local = q * 32 + lane;
            const int64_t row = static_cast<int64_t>(rtile) * kTileM + r_local;
            const bool row_ok = row < rows;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * kColAccCols;
            uint32_t sc_word = 0;
            uint32_t ra[32], rb[32];
            ptx::tmem_ld_32cols(t_row, ra);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < kColTileG; ++j) {
                uint32_t(&cur)[32] = (j & 1) ? rb : ra;
                uint32_t(&nxt)[32] = (j & 1) ? ra : rb;
                if (j + 1 < kColTileG) ptx::tmem_ld_32cols(t_row + (j + 1) * 32, nxt);
                const int64_t g = static_cast<int64_t>(ctile) * kColTileG + j;
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
                if (j + 1 < kColTileG) ptx::tmem_wait_ld();
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&bars->acc_empty[a]));
            if constexpr (kMode == RotOut::Quant) {
                if (scale_vec && row_ok)
                    *reinterpret_cast<uint32_t *>(args.scales + row * G + static_cast<int64_t>(ctile) * kColTileG) =
                        sc_word;
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
    kernel_teardown(tmem_base, kMmaWarp);
}

// =====================================================================================
// Dequantise and undo the transform: out = (v * R^T) * Lambda, v = E2M1(code) * 2^e.
// =====================================================================================
//
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
                       const uint16_t *__restrict__ rhat, const float *__restrict__ lambda)
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
            if (lane == 0) ok = wait_bar(&bars->empty[s], ((it / kDqStages) & 1) ^ 1, abort);
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
            const bool b_ok = wait_bar(&bars->b_full[0], 0, abort);
            int it = 0;
            for (int c = blockIdx.x; b_ok && c < n_chunks; c += gridDim.x, ++it) {
                const int s = it % kDqStages;
                const int a = it % kDqAcc;
                if (!wait_bar(&bars->full[s], (it / kDqStages) & 1, abort)) break;
                if (!wait_bar(&bars->acc_empty[a], ((it / kDqAcc) & 1) ^ 1, abort)) break;
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
            drain_mmas(bars);
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
            if (lane == 0) ok = wait_bar(&bars->acc_full[a], (it / kDqAcc) & 1, abort);
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

static_assert(kFlatSmemBytes <= 232448 && kColSmemBytes <= 232448 && kDqSmemBytes <= 232448, "shared memory budget");

// Launch with programmatic stream serialisation: the grid may start while the
// previous kernel in the stream drains (the kernels order their global accesses
// with griddepcontrol.wait).
template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kern, int grid, int block, int smem, cudaStream_t stream, Args... args)
{
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
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
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Diagnostic: one thread waits on an mbarrier phase that nothing completes, so the
// bounded wait must run out, set the status word and return.  It exercises the
// same wait routine as the pipelines, without any TMA, MMA or TMEM in play.
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
    ptx::mbar_arrive(ptx::smem_addr(&bar));   // complete the phase before exit
}

}  // namespace

cudaError_t launch_rotate(const RotMaps &maps, const RotArgs &args, RotOut mode, int num_sms, cudaStream_t stream)
{
    if (args.rows <= 0 || args.cols <= 0) return cudaSuccess;
    if (args.lambda == nullptr) {
        const int64_t n_groups = args.rows * (args.cols / 32);
        const int64_t n_chunks = (n_groups + kFlatStageGroups - 1) / kFlatStageGroups;
        const int grid = static_cast<int>(n_chunks < num_sms ? n_chunks : num_sms);
        return mode == RotOut::Quant
                   ? launch_pdl(rotate_flat_kernel<RotOut::Quant>, grid, kThreads, kFlatSmemBytes, stream, maps.groups,
                                args)
                   : launch_pdl(rotate_flat_kernel<RotOut::F32>, grid, kThreads, kFlatSmemBytes, stream, maps.groups,
                                args);
    }
    const int64_t n_tiles = ((args.rows + kTileM - 1) / kTileM) * ((args.cols + kTileCols - 1) / kTileCols);
    const int grid = static_cast<int>(n_tiles < num_sms ? n_tiles : num_sms);
    return mode == RotOut::Quant
               ? launch_pdl(rotate_cols_kernel<RotOut::Quant>, grid, kColThreads, kColSmemBytes, stream, maps.x,
                            maps.codes, args)
               : launch_pdl(rotate_cols_kernel<RotOut::F32>, grid, kColThreads, kColSmemBytes, stream, maps.x,
                            maps.codes, args);
}

cudaError_t launch_dequant_rot(const CUtensorMap &tmap_out, const uint8_t *codes, const uint8_t *scales, int64_t rows,
                               int64_t cols, const uint16_t *rhat, const float *lambda, int num_sms,
                               cudaStream_t stream)
{
    const int64_t G = cols / 32;
    const int64_t n_groups = rows * G;
    if (n_groups <= 0) return cudaSuccess;
    const int64_t n_chunks = (n_groups + kDqStageGroups - 1) / kDqStageGroups;
    const int grid = static_cast<int>(n_chunks < num_sms ? n_chunks : num_sms);
    const uint4 *c4 = reinterpret_cast<const uint4 *>(codes);
    return lambda ? launch_pdl(dequant_rot_kernel<true>, grid, kDqThreads, kDqSmemBytes, stream, tmap_out, c4, scales,
                               n_groups, G, rhat, lambda)
                  : launch_pdl(dequant_rot_kernel<false>, grid, kDqThreads, kDqSmemBytes, stream, tmap_out, c4, scales,
                               n_groups, G, rhat, lambda);
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
