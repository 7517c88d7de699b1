// rotate_block_sm100.cu -- rotate -> MXFP4 with rotation blocks wider than a group (B200, sm_100a).
//
// The DuQuant++ write-up's §4.3 ablation rotates blocks of B = 16, 32, 64 or
// 128 channels with one shared B x B matrix, while the MXFP4 groups stay at 32
// elements.  B = 32 is the main path, and B = 16 is a block-diagonal 32 x 32
// matrix on the main path's kernels.  This file covers B = 64 and 128 without
// smoothing.
//
// X is viewed as a dense [rows*cols/B, B] bf16 matrix (one row per rotation
// block) and the product is one tcgen05 GEMM per 128 blocks: M = 128, N = B,
// K = B (B/16 MMAs of K = 16), bf16 in, fp32 accumulate in TMEM.  A stage holds
// 32 KB of X: 256 blocks of 64, or 128 blocks of 128.  It is staged by TMA in
// 128-byte-swizzled K-atoms of 64 columns (one atom for B = 64, two for 128).
// Each TMEM row then holds B/32 MXFP4 groups of one block.  The epilogue takes
// them 32 columns at a time, so, as in the flat kernel, each thread quantises
// one whole group from registers.  Warp roles, the barriers and the bounded
// waits are those of the flat kernel.
#include "pipeline_sm100.cuh"

namespace mxq {
namespace {

using namespace pipe;

constexpr int kBlkStageBytes = 32 * 1024;
constexpr int kBlkAccCols = 128;                           // TMEM columns per accumulator stage
constexpr int kBlkAcc = 512 / kBlkAccCols;

template <int kBlk>
struct BlockCfg {
    static constexpr int kAtoms = kBlk / 64;                       // 128-byte K-atoms per row
    static constexpr int kStageRows = kBlkStageBytes / (2 * kBlk);  // blocks per stage
    static constexpr int kSub = kStageRows / 128;                  // MMAs (of 128 blocks) per stage
    static constexpr int kAtomBytes = kStageRows * 128;            // one K-atom of a stage
    static constexpr int kBBytes = kBlk * 2 * kBlk;                // B operand: N = kBlk rows, K-major
    static constexpr int kBAtomBytes = kBlk * 128;
    static constexpr int kGroupsPerRow = kBlk / 32;
    // 3 stages (96 KB in flight) measured best for both widths, as for the flat
    // kernel: 2 or 4-5 stages were 4-7 % slower.
    static constexpr int kStages = 3;
    static constexpr int kSmem = kStages * kBlkStageBytes + kBBytes + 512 + 1024;
    static_assert(kBlk == 64 || kBlk == 128, "block width");
    static_assert(kSub * kBlk == kBlkAccCols, "one accumulator stage holds a whole stage");
    static_assert(kSub * kGroupsPerRow == 4, "four 32-column TMEM loads per stage");
    static_assert(kSmem <= 232448, "shared memory budget");
};

template <int kBlk, RotOut kMode>
__global__ void __launch_bounds__(kThreads, 1)
    rotate_block_kernel(const __grid_constant__ CUtensorMap tmap_b, const RotArgs args, unsigned int *status)
{
    using C = BlockCfg<kBlk>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *stages = align_1k(smem_raw);
    uint8_t *bmat = stages + C::kStages * kBlkStageBytes;
    Bars *bars = reinterpret_cast<Bars *>(bmat + C::kBBytes);
    volatile int *abort = &bars->abort;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t n_blocks = args.rows * (args.cols / kBlk);
    const int n_chunks = static_cast<int>((n_blocks + C::kStageRows - 1) / C::kStageRows);

    const uint32_t tmem_base =
        kernel_setup(bars, SetupCfg{C::kStages, kBlkAcc, 1, kBuildWarps * 32, kMmaWarp}, &tmap_b, nullptr);

    if (warp == kTmaWarp) {
        if (lane == 0) {
            const uint64_t pol = ptx::policy_evict_first();
            int it = 0;
            for (int c = blockIdx.x; c < n_chunks; c += gridDim.x, ++it) {
                const int s = it % C::kStages;
                if (!wait_bar(&bars->empty[s], ((it / C::kStages) & 1) ^ 1, abort, status)) break;
                const uint32_t full = ptx::smem_addr(&bars->full[s]);
                const uint32_t dst = ptx::smem_addr(stages + s * kBlkStageBytes);
                ptx::mbar_arrive_expect_tx(full, kBlkStageBytes);
#pragma unroll
                for (int ka = 0; ka < C::kAtoms; ++ka)
                    ptx::tma_load_2d(dst + ka * C::kAtomBytes, &tmap_b, ka * 64, c * C::kStageRows, full, pol);
            }
            drain_loads(bars, C::kStages, it, status);
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, kBlk);
            const uint32_t b_base = ptx::smem_addr(bmat);
            const bool b_ok = wait_bar(&bars->b_full[0], 0, abort, status);   // B is built once
            int it = 0;
            for (int c = blockIdx.x; b_ok && c < n_chunks; c += gridDim.x, ++it) {
                const int s = it % C::kStages;
                const int a = it % kBlkAcc;
                if (!wait_bar(&bars->full[s], (it / C::kStages) & 1, abort, status)) break;
                if (!wait_bar(&bars->acc_empty[a], ((it / kBlkAcc) & 1) ^ 1, abort, status)) break;
                ptx::tc_fence_after();
                const uint32_t a_base = ptx::smem_addr(stages + s * kBlkStageBytes);
                const uint32_t d_base = tmem_base + static_cast<uint32_t>(a * kBlkAccCols);
#pragma unroll
                for (int m = 0; m < C::kSub; ++m) {
#pragma unroll
                    for (int kk = 0; kk < kBlk / 16; ++kk) {
                        const uint32_t ao = (kk >> 2) * C::kAtomBytes + m * 128 * 128 + (kk & 3) * 32;
                        const uint32_t bo = (kk >> 2) * C::kBAtomBytes + (kk & 3) * 32;
                        ptx::mma_bf16(d_base + m * kBlk, ptx::smem_desc_sw128(a_base + ao),
                                      ptx::smem_desc_sw128(b_base + bo), idesc, kk);
                    }
                }
                ptx::mma_commit(ptx::smem_addr(&bars->empty[s]));
                ptx::mma_commit(ptx::smem_addr(&bars->acc_full[a]));
            }
            drain_mmas(bars, status);
        }
    } else if (warp >= kBuildWarp0) {
        // B = R_B in K-major form: row n holds R_B[0..kBlk-1][n], split into 128-byte
        // K-atoms of 64 values, each atom [kBlk rows x 128 B] with the 128-byte swizzle.
        const int bt = threadIdx.x - kBuildWarp0 * 32;
        constexpr int kChunks = kBlk * (kBlk / 8);   // 16-byte chunks of B
        for (int t = bt; t < kChunks; t += kBuildWarps * 32) {
            const int n = t / (kBlk / 8), kc = t % (kBlk / 8);   // kc: chunk of 8 k values
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int k = kc * 8 + 2 * e;
                w[e] = static_cast<uint32_t>(args.rhat[k * kBlk + n]) |
                       (static_cast<uint32_t>(args.rhat[(k + 1) * kBlk + n]) << 16);
            }
            *reinterpret_cast<uint4 *>(bmat + (kc >> 3) * C::kBAtomBytes + sw128(n, kc & 7)) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(ptx::smem_addr(&bars->b_full[0]));
    } else {
        const int q = warp & 3;       // TMEM lane quarter this warp may access
        const int ewg = warp >> 2;    // which half of the stages this warp group takes
        int it = 0;
        for (int c = blockIdx.x; c < n_chunks; c += gridDim.x, ++it) {
            if ((it & 1) != ewg) continue;
            const int a = it % kBlkAcc;
            int ok = 0;
            if (lane == 0) ok = wait_bar(&bars->acc_full[a], (it / kBlkAcc) & 1, abort, status);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            ptx::tc_fence_after();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * kBlkAccCols;
            const int64_t blk_lane = static_cast<int64_t>(c) * C::kStageRows + q * 32 + lane;
            // Column 32*j of the stage's accumulator is group h = j % (B/32) of the block
            // in sub-tile m = j / (B/32).  The load of j+1 is in flight while j is quantised.
            uint32_t ra[32], rb[32];
            ptx::tmem_ld_32cols(t_row, ra);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t(&cur)[32] = (j & 1) ? rb : ra;
                uint32_t(&nxt)[32] = (j & 1) ? ra : rb;
                if (j + 1 < 4) ptx::tmem_ld_32cols(t_row + (j + 1) * 32, nxt);
                const int m = j / C::kGroupsPerRow, h = j % C::kGroupsPerRow;
                const int64_t blk = blk_lane + m * 128;
                if (blk < n_blocks) {
                    const int64_t g = blk * C::kGroupsPerRow + h;
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
                if (j + 1 < 4) ptx::tmem_wait_ld();
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&bars->acc_empty[a]));
        }
    }
    kernel_teardown(tmem_base, kMmaWarp);
}

template <int kBlk>
cudaError_t launch_block(const CUtensorMap &tmap, const RotArgs &args, RotOut mode, int num_sms, cudaStream_t stream)
{
    using C = BlockCfg<kBlk>;
    const int64_t n_blocks = args.rows * (args.cols / kBlk);
    const int64_t n_chunks = (n_blocks + C::kStageRows - 1) / C::kStageRows;
    if (n_chunks <= 0) return cudaSuccess;
    const int grid = static_cast<int>(n_chunks < num_sms ? n_chunks : num_sms);
    unsigned int *status = status_word();
    if (!status) return cudaErrorInvalidSymbol;
    if (mode == RotOut::Quant)
        return launch_pdl(rotate_block_kernel<kBlk, RotOut::Quant>, grid, kThreads, C::kSmem, stream, tmap, args,
                          status);
    if (mode == RotOut::F32)
        return launch_pdl(rotate_block_kernel<kBlk, RotOut::F32>, grid, kThreads, C::kSmem, stream, tmap, args,
                          status);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_rotate_block(const CUtensorMap &tmap_blocks, const RotArgs &args, int blk, RotOut mode,
                                int num_sms, cudaStream_t stream)
{
    if (blk == 64) return launch_block<64>(tmap_blocks, args, mode, num_sms, stream);
    if (blk == 128) return launch_block<128>(tmap_blocks, args, mode, num_sms, stream);
    return cudaErrorInvalidValue;
}

}  // namespace mxq
