// mxq_internal.h -- declarations shared by the library's translation units
// (kernel launchers and the C ABI layer).  Not part of the public ABI.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace mxq {

// Device status word bits (written by kernels, read by mxq_sync_check).
enum : unsigned int {
    kStatusTimeout = 1u,   // a bounded pipeline wait ran out
};

// Output mode of the fused rotate kernels: packed codes + scales, the rotated
// fp32 values, the per-group MXFP4 quantisation error (plus per-warp partial
// sums for its mean), or NVFP4 (codes + one E4M3 scale per 16 values).
// Quant: MXFP4 codes and row-major scales; QuantMma: the same codes with the scales in
// the block-scaled MMA's atom layout (args.sf_mma); F32: the rotated values; Err: the
// per-group quantisation error; QuantNv: NVFP4; QuantNvMma: NVFP4 with its E4M3 scales in
// the same atom layout (one atom column per 16-value block).
enum class RotOut { Quant, F32, Err, QuantNv, QuantMma, QuantNvMma };
__host__ __device__ constexpr bool rot_nvfp4(RotOut m) { return m == RotOut::QuantNv || m == RotOut::QuantNvMma; }
__host__ __device__ constexpr bool rot_sf_mma(RotOut m) { return m == RotOut::QuantMma || m == RotOut::QuantNvMma; }

struct RotArgs {
    const uint16_t *rhat;      // bf16 [32][32], row-major [k][n]; [16][16] when rblk == 16
    int rblk;                  // 16: R^ is diag(R16, R16) built from a 16x16 input; otherwise 32
    int lam_mul;               // 1: multiply by lambda (the weights' side); 0: divide (activations)
    const float *nv_scale;     // QuantNv: the fp32 tensor scale s_t (device, one float)
    const float *lambda;       // fp32 [cols] or nullptr
    uint8_t *codes;            // [rows, cols/2]   (Quant)
    uint8_t *scales;           // [rows, cols/32]  (Quant)
    uint8_t *sf_mma;           // QuantMma, QuantNvMma: the scales in the block-scaled MMA's atom
                               // layout (mxq_scales_to_mma_layout's or mxq_nvfp4_scales_to_mma_layout's output)
    float *y;                  // [rows, cols]     (F32)
    float *err;                // [rows, cols/32]  (Err; may be null)
    double *partials;          // per-warp error sums (Err): see rotate_*_partials()
    int64_t rows;
    int64_t cols;
};

// Fused rotate -> MXFP4 without smoothing.  `tmap_groups` views X as a dense
// [rows*cols/32, 32] bf16 matrix (box {32, 256}, 64-byte swizzle).
cudaError_t launch_rotate_flat(const CUtensorMap &tmap_groups, const RotArgs &args, RotOut mode, int num_sms,
                               cudaStream_t stream);

// Fused smooth -> rotate -> MXFP4 (args.lambda non-null).  `tmap_x` views X as
// [rows, cols] bf16 (box {64, 128}, 128-byte swizzle); `tmap_codes` the packed
// codes as [rows, cols/2] uint8 (box {32, 32}: one epilogue warp's rows of a 64-column
// tile, 32-byte swizzle; Quant mode only).
cudaError_t launch_rotate_cols(const CUtensorMap &tmap_x, const CUtensorMap &tmap_codes, const RotArgs &args,
                               RotOut mode, int num_sms, cudaStream_t stream);

// Rotate -> MXFP4 with rotation blocks of blk = 64 or 128 columns (no smoothing).
// `tmap_blocks` views X as [rows*cols/blk, blk] bf16 (box {64, 16384/blk}, 128-byte
// swizzle); args.rhat is bf16 [blk][blk].
cudaError_t launch_rotate_block(const CUtensorMap &tmap_blocks, const RotArgs &args, int blk, RotOut mode,
                                int num_sms, cudaStream_t stream);

// The MXFP4 x MXFP4 consumer GEMM: Y[M, N] = deq(A)[M, K] * deq(B)[N, K]^T.  `tmap_a` /
// `tmap_b` view the codes as uint8 [M, K/2] / [N, K/2] (boxes {128, 128} / {128, 256},
// 128-byte swizzle).
struct GemmArgs {
    void *y;                   // [M, N] fp32 or bf16, row-major, 16-byte aligned
    int64_t M, N, K;
    int out_bf16;
    int nvfp4;                 // 0: MXFP4 (E8M0 per 32 k); 1: NVFP4 (E4M3 per 16 k, times the tensor scales)
    const float *a_tscale;     // NVFP4: the operands' fp32 tensor scales (device, one float each)
    const float *b_tscale;
};
// The GEMM runs on CTA pairs (cta_group::2, 256 x 256 tiles): tmap_a / tmap_b in boxes of
// 128 rows x 128 B; tmap_sfa / tmap_sfb: the scale atoms as uint32 [row blocks][cb_n * 128],
// boxes of 256 (two atoms) x 1 row block (A) or 2 (B).
cudaError_t launch_mxfp4_gemm(const CUtensorMap &tmap_a, const CUtensorMap &tmap_b, const CUtensorMap &tmap_sfa,
                              const CUtensorMap &tmap_sfb, const GemmArgs &args, int num_sms, cudaStream_t stream);

// Row-major E8M0 scales [rows, G] -> the block-scaled MMA's 512-byte atoms (128 rows x 4
// k-blocks; row r, k-block j at byte 16 (r % 32) + 4 (r / 32) + j; padding 0).
cudaError_t launch_scales_to_mma(const uint8_t *scales, int64_t rows, int64_t G, uint8_t *out, cudaStream_t stream);

// Number of per-warp partial sums the Err mode writes (one double each).
int64_t rotate_flat_partials(int64_t rows, int64_t cols);
int64_t rotate_cols_partials(int64_t rows, int64_t cols);

// Mean of the per-group errors from the partial sums, in a fixed order: out = sum / n_groups.
cudaError_t launch_error_mean(const double *partials, int64_t n_partials, int64_t n_groups, double *out,
                              cudaStream_t stream);

// Dequantise to bf16 in the rotated domain (codes 16-byte aligned, out 16-byte aligned).
cudaError_t launch_dequant_plain(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t cols,
                                 uint16_t *out, int num_sms, cudaStream_t stream);

// Dequantise and undo the rotation (rhat non-null) and the smoothing (lambda, may be
// null).  `tmap_out` views the bf16 output as [rows*cols/32, 32] (box {32, 32},
// 64-byte swizzle).
cudaError_t launch_dequant_rot(const CUtensorMap &tmap_out, const uint8_t *codes, const uint8_t *scales, int64_t rows,
                               int64_t cols, const uint16_t *rhat, const float *lambda, int num_sms,
                               cudaStream_t stream);

// The outlier-aware rotation search (all pointers device memory; see mxq.h).
struct SearchArgs {
    const void *X;             // bf16 [rows, cols], 16-byte aligned
    const float *lambda;       // fp32 [cols] or nullptr
    int64_t rows;
    int64_t cols;
    int max_steps;             // K
    int n_angle;               // the Givens grid has 2 * n_angle angles
    double *R;                 // [32][32] result, row-major [k][n]
    uint16_t *rhat;            // bf16 [32][32] or nullptr
    int32_t *trace;            // [max_steps][3] (d, j, angle) or nullptr
    double *linf;              // [max_steps + 1] or nullptr
    int32_t *steps;            // steps taken, or nullptr
    int64_t *group;            // the worst group, or nullptr
    void *workspace;           // rotation_search_workspace() bytes, 256-byte aligned
};
size_t rotation_search_workspace(int64_t rows, int64_t cols, int n_angle);
cudaError_t launch_rotation_search(const SearchArgs &args, int num_sms, cudaStream_t stream);
int rotation_search_launches(int max_steps);

// Diagnostic kernel: a bounded wait on a barrier nothing completes (writes 2 to
// *result once the wait ran out and the abort flag was raised).
cudaError_t launch_wait_selftest(uint64_t timeout_ns, int *result, cudaStream_t stream);

// Set the text mxq_last_cuda_error() returns on this thread.
void set_last_error(const char *msg);

// Device address of the status word on the current device (nullptr on failure).  It is
// looked up on every call, so it stays right after a device reset moves the module.
unsigned int *status_word();

// Opt `func` in to `smem` bytes of dynamic shared memory on the current device.  The
// runtime call is made once per (kernel, device, size); force makes it again.
cudaError_t smem_optin(const void *func, int smem, bool force);

// Read-and-clear of the device status word, stream ordered.
cudaError_t read_and_clear_status(unsigned int *host_status, cudaStream_t stream);

// Rows per tile and columns per tile of the fused kernel (for host-side sizing).
constexpr int kTileM = 128;
constexpr int kTileCols = 128;

}  // namespace mxq
