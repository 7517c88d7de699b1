// rotate_flat_sm100.cu -- fused rotate -> MXFP4-quantise kernel without smoothing (B200, sm_100a).
//
// The online step of the DuQuant++ write-up (jsqmd.com/news/928156), X_hat = X * R^
// (§2.3, §3.3), one 32x32 R^ shared by every 32-element group (§3.2 step 4).  Each
// group is then quantised to MXFP4 as in §2.1: absmax -> E8M0 scale -> divide ->
// nearest E2M1, under the OCP MX rule.  Fusing the quantiser in (§5.2 item 1 asks
// for the smoothing and rotation in one kernel) means X is read once and only
// the packed codes and scales are written.
//
// X is a dense [rows*cols/32, 32] bf16 matrix, the reshape-and-bmm form of
// §3.3's implementation tips.  One persistent CTA per SM, warp-specialised:
//   warps 0-7   epilogue, two groups of four, each group taking every other stage
//   warp 8      TMA producer (one thread)
//   warp 9      TMEM allocator + MMA issuer (one thread)
//   warps 10-11 build the B operand (R^ in K-major form) once
// The MMA (tcgen05, M=128, N=32, K=16, bf16 in, fp32 accumulate) takes 128
// consecutive groups: A from shared memory (64-byte swizzle, staged by TMA in
// boxes of 256 groups = 16 contiguous KB), B = R^T row-major, D = 128 TMEM lanes
// x 32 columns.  A stage is 4 MMAs (512 groups); 3 stages (~96 KB in flight per
// SM) measured best.  The epilogue reads TMEM with tcgen05.ld 32x32b.x32.  Each
// thread then holds one group's 32 rotated values, so absmax, E8M0, scaling and
// the E2M1 conversion are thread-local.  A warp's 32 lanes hold 32 consecutive
// groups, so its code store covers 512 contiguous bytes and its scale store 32.
#include "pipeline_sm100.cuh"

namespace mxq {
namespace {

using namespace pipe;

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

// Warp roles per output mode.  The error mode's epilogue (quantise, decode, two sums per
// group) is the longest, so it runs four groups of four epilogue warps, each taking every
// fourth stage (one accumulator stage each); the others run two groups.
template <RotOut kMode>
struct FlatRoles {
    static constexpr int kGroups = (kMode == RotOut::Err || rot_nvfp4(kMode)) ? 4 : 2;
    static constexpr int kEpi = 4 * kGroups;
    static constexpr int kTma = kEpi;
    static constexpr int kMma = kEpi + 1;
    static constexpr int kBuild0 = kEpi + 2;
    static constexpr int kThreadsF = (kEpi + 2 + kBuildWarps) * 32;
};
static_assert(kFlatAcc % FlatRoles<RotOut::Err>::kGroups == 0, "one accumulator stage per epilogue group");

template <RotOut kMode>
__global__ void __launch_bounds__(FlatRoles<kMode>::kThreadsF, 1)
    rotate_flat_kernel(const __grid_constant__ CUtensorMap tmap_g, const RotArgs args, unsigned int *status)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *stages = align_1k(smem_raw);
    uint8_t *bmat = stages + kFlatStages * kFlatStageBytes;
    Bars *bars = reinterpret_cast<Bars *>(bmat + kBMatBytes);
    volatile int *abort = &bars->abort;
    using Ro = FlatRoles<kMode>;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t n_groups = args.rows * (args.cols / 32);
    const int n_chunks = static_cast<int>((n_groups + kFlatStageGroups - 1) / kFlatStageGroups);

    const uint32_t tmem_base =
        kernel_setup(bars, SetupCfg{kFlatStages, kFlatAcc, 1, kBuildWarps * 32, Ro::kMma}, &tmap_g, nullptr);

    if (warp == Ro::kTma) {
        if (lane == 0) {
            const uint64_t pol = ptx::policy_evict_first();
            int it = 0;
            for (int c = blockIdx.x; c < n_chunks; c += gridDim.x, ++it) {
                const int s = it % kFlatStages;
                if (!wait_bar(&bars->empty[s], ((it / kFlatStages) & 1) ^ 1, abort, status)) break;
                const uint32_t full = ptx::smem_addr(&bars->full[s]);
                const uint32_t dst = ptx::smem_addr(stages + s * kFlatStageBytes);
                const int g0 = c * kFlatStageGroups;
                ptx::mbar_arrive_expect_tx(full, kFlatStageBytes);
#pragma unroll
                for (int b = 0; b < kFlatBoxes; ++b)
                    ptx::tma_load_2d(dst + b * kFlatBoxGroups * 64, &tmap_g, 0, g0 + b * kFlatBoxGroups, full, pol);
            }
            drain_loads(bars, kFlatStages, it, status);
        }
    } else if (warp == Ro::kMma) {
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, 32);
            const uint32_t b_base = ptx::smem_addr(bmat);
            const bool b_ok = wait_bar(&bars->b_full[0], 0, abort, status);   // B is built once
            int it = 0;
            for (int c = blockIdx.x; b_ok && c < n_chunks; c += gridDim.x, ++it) {
                const int s = it % kFlatStages;
                const int a = it % kFlatAcc;
                if (!wait_bar(&bars->full[s], (it / kFlatStages) & 1, abort, status)) break;
                if (!wait_bar(&bars->acc_empty[a], ((it / kFlatAcc) & 1) ^ 1, abort, status)) break;
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
            drain_mmas(bars, status);
        }
    } else if (warp >= Ro::kBuild0) {
        // B = R^ in K-major form: row n holds R^[0..31][n] (bf16, first 64 B of a 128-B row).
        const int bt = threadIdx.x - Ro::kBuild0 * 32;
        for (int t = bt; t < 32 * 4; t += kBuildWarps * 32) {
            const int n = t >> 2, c = t & 3;
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int k = c * 8 + 2 * e;
                w[e] = static_cast<uint32_t>(rhat_at(args, k, n)) |
                       (static_cast<uint32_t>(rhat_at(args, k + 1, n)) << 16);
            }
            *reinterpret_cast<uint4 *>(bmat + sw128(n, c)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(ptx::smem_addr(&bars->b_full[0]));
    } else {
        const int q = warp & 3;       // TMEM lane quarter this warp may access
        const int ewg = warp >> 2;    // which of the stages (every kGroups-th) this warp group takes
        // NVFP4: the tensor scale s_t and r_t = 1 / (6 s_t), once per thread
        float nv_st = 0.0f, nv_rt = 0.0f;
        if constexpr (rot_nvfp4(kMode)) {
            nv_st = *args.nv_scale;
            nv_rt = __frcp_rn(__fmul_rn(6.0f, nv_st));
        }
        int it = 0;
        for (int c = blockIdx.x; c < n_chunks; c += gridDim.x, ++it) {
            if ((it % Ro::kGroups) != ewg) continue;
            const int a = it % kFlatAcc;
            int ok = 0;
            if (lane == 0) ok = wait_bar(&bars->acc_full[a], (it / kFlatAcc) & 1, abort, status);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            ptx::tc_fence_after();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * kFlatAccCols;
            const int64_t g_lane = static_cast<int64_t>(c) * kFlatStageGroups + q * 32 + lane;
            double err_acc = 0.0;   // Err mode: this lane's groups, in order
            // scales in the MMA layout: the lane's row and group from one division per stage,
            // then advanced by 128 groups per MMA with additions (at most one wrap when G >= 128)
            [[maybe_unused]] const int64_t G = args.cols / 32;
            [[maybe_unused]] int64_t sf_r = 0, sf_g = 0;
            if constexpr (rot_sf_mma(kMode)) {
                sf_r = g_lane / G;
                sf_g = g_lane - sf_r * G;
            }
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
                    } else if constexpr (kMode == RotOut::Err) {
                        uint32_t w[4];
                        float e;
                        quantize_group_err(cur, w, e);
                        if (args.err) args.err[g] = e;
                        err_acc += static_cast<double>(e);
                    } else if constexpr (rot_nvfp4(kMode)) {
                        uint32_t w[4];
                        const uint32_t bytes = quantize_group_nv(cur, w, nv_rt, nv_st);
                        ptx::st_global_v4(args.codes + g * 16, w[0], w[1], w[2], w[3]);
                        if constexpr (kMode == RotOut::QuantNvMma)   // blocks 2g, 2g + 1: one aligned 16-bit word
                            *reinterpret_cast<uint16_t *>(args.sf_mma + sf_mma_offset(sf_r, 2 * sf_g, (2 * G + 3) >> 2)) =
                                static_cast<uint16_t>(bytes);
                        else
                            reinterpret_cast<uint16_t *>(args.scales)[g] = static_cast<uint16_t>(bytes);
                    } else {
                        uint32_t w[4];
                        const uint32_t byte = quantize_group(cur, w);
                        ptx::st_global_v4(args.codes + g * 16, w[0], w[1], w[2], w[3]);
                        if constexpr (kMode == RotOut::QuantMma)
                            args.sf_mma[sf_mma_offset(sf_r, sf_g, (G + 3) >> 2)] = static_cast<uint8_t>(byte);
                        else
                            args.scales[g] = static_cast<uint8_t>(byte);
                    }
                }
                if constexpr (rot_sf_mma(kMode)) {
                    sf_g += 128;
                    while (sf_g >= G) {
                        sf_g -= G;
                        ++sf_r;
                    }
                }
                if (j + 1 < kFlatMmas) ptx::tmem_wait_ld();
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&bars->acc_empty[a]));
            if constexpr (kMode == RotOut::Err) {
                const double sum = warp_sum(err_acc);
                if (lane == 0) args.partials[static_cast<int64_t>(c) * 4 + q] = sum;   // one slot per warp and stage
            }
        }
    }
    kernel_teardown(tmem_base, Ro::kMma);
}

static_assert(kFlatSmemBytes <= 232448, "shared memory budget");

}  // namespace

cudaError_t launch_rotate_flat(const CUtensorMap &tmap_groups, const RotArgs &args, RotOut mode, int num_sms,
                               cudaStream_t stream)
{
    const int64_t n_groups = args.rows * (args.cols / 32);
    const int64_t n_chunks = (n_groups + kFlatStageGroups - 1) / kFlatStageGroups;
    if (n_chunks <= 0) return cudaSuccess;
    const int grid = static_cast<int>(n_chunks < num_sms ? n_chunks : num_sms);
    unsigned int *status = status_word();
    if (!status) return cudaErrorInvalidSymbol;
    if (mode == RotOut::Quant)
        return launch_pdl(rotate_flat_kernel<RotOut::Quant>, grid, FlatRoles<RotOut::Quant>::kThreadsF, kFlatSmemBytes,
                          stream, tmap_groups, args, status);
    if (mode == RotOut::QuantMma)
        return launch_pdl(rotate_flat_kernel<RotOut::QuantMma>, grid, FlatRoles<RotOut::QuantMma>::kThreadsF,
                          kFlatSmemBytes, stream, tmap_groups, args, status);
    if (mode == RotOut::QuantNvMma)
        return launch_pdl(rotate_flat_kernel<RotOut::QuantNvMma>, grid, FlatRoles<RotOut::QuantNvMma>::kThreadsF,
                          kFlatSmemBytes, stream, tmap_groups, args, status);
    if (mode == RotOut::Err)
        return launch_pdl(rotate_flat_kernel<RotOut::Err>, grid, FlatRoles<RotOut::Err>::kThreadsF, kFlatSmemBytes,
                          stream, tmap_groups, args, status);
    if (mode == RotOut::QuantNv)
        return launch_pdl(rotate_flat_kernel<RotOut::QuantNv>, grid, FlatRoles<RotOut::QuantNv>::kThreadsF,
                          kFlatSmemBytes, stream, tmap_groups, args, status);
    return launch_pdl(rotate_flat_kernel<RotOut::F32>, grid, FlatRoles<RotOut::F32>::kThreadsF, kFlatSmemBytes, stream,
                      tmap_groups, args, status);
}

int64_t rotate_flat_partials(int64_t rows, int64_t cols)
{
    return ((rows * (cols / 32) + kFlatStageGroups - 1) / kFlatStageGroups) * 4;
}

}  // namespace mxq
