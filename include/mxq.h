/*
 * mxq.h -- C ABI of the B200 (sm_100a) fused smooth-rotate-MXFP4 library, libmxq.so.
 *
 * The operation is the online step of DuQuant++ as the write-up "DuQuant++:
 * block-aligned rotation quantisation for MXFP4 activation outliers"
 * (jsqmd.com/news/928156) describes it.
 *   - Each activation row is cut into 32-element MXFP4 groups (§2.1, §2.3).
 *   - Every group is divided per channel by the SmoothQuant scale Lambda
 *     (§3.1; online it is X * Lambda^-1, §3.3).
 *   - It is then multiplied by one shared, outlier-aware 32x32 orthogonal
 *     matrix R^, i.e. X -> X * R^ (§2.3, §3.2 step 4, §3.3).  No permutation
 *     and no second rotation.
 *   - Last, the group is quantised to MXFP4 (§2.1, §5.1 item 5).  One shared
 *     power-of-two scale per group comes from its absmax, and each element is
 *     rounded to the nearest 4-bit float.
 * §5.2 item 1 and §5.4 item 3 ask for the smoothing and the rotation to be
 * fused into one kernel ahead of the MXFP4 linear layer.  Here the
 * quantisation is fused in as well.
 *
 * MXFP4 rule (the OCP Microscaling v1.0 reading of §2.1; the page gives none):
 *   amax  = max_n |y_n| over the group's 32 rotated fp32 values
 *   e     = clamp(floor(log2 amax) - 2, -127, 127); amax == 0 gives e = -127
 *   scale byte (E8M0) = e + 127; a NaN/Inf amax gives byte 0xFF and all codes 0
 *   code_n = E2M1(y_n * 2^-e): round to nearest, ties to the even code,
 *            |.| > 6 saturates to 6, sign kept (-0 and tiny negatives -> 0x8)
 *   E2M1 codes 0..7 = magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}; bit 3 = sign.
 *
 * Layouts (all row-major, no padding between rows):
 *   X       bf16  [rows, cols]           cols % 32 == 0
 *   R^      bf16  [32, 32]               R^[k][n]: y_n = sum_k x_k * R^[k][n]
 *   Lambda  fp32  [cols] or NULL         strictly positive and finite; NULL = no smoothing
 *   codes   uint8 [rows, cols/2]         byte i of a row holds column 2i in its low
 *                                        nibble and column 2i+1 in its high nibble
 *   scales  uint8 [rows, cols/32]        one E8M0 byte per group
 *
 * Common rules for every entry point below.
 *   Memory.  All pointers are device memory owned by the caller (for example
 *     from PyTorch).  The library allocates nothing and may be called from
 *     several host threads.  Between calls it keeps only host-side caches that
 *     cannot change a result: per host thread, the TMA descriptors of the last
 *     few calls (keyed by everything a descriptor is encoded from), and per
 *     device, the SM count and the kernels whose shared-memory opt-in is set.
 *   Streams.  `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is queued on it asynchronously; the call returns right
 *     after the launch.
 *   Errors.  Bad arguments return MXQ_ERR_INVALID_ARG before anything is
 *     launched.  That covers NULL pointers where one is required, negative
 *     sizes, cols % 32 != 0, misaligned pointers, pointers that are not device
 *     memory of the current device, and outputs that overlap inputs.
 *     rows == 0 or cols == 0 is a valid no-op (pointers are then not looked at).
 *     Launch failures return MXQ_ERR_CUDA.
 *     Faults during execution surface at the caller's next synchronisation.
 *   Bounded waits.  The kernels' internal pipeline waits are bounded.  If one
 *     runs out, the kernel records MXQ_ERR_TIMEOUT in a device status word and
 *     returns early; its outputs are then undefined.  mxq_sync_check() reads
 *     and clears that word.
 *   Contract on values.  Results are defined for finite inputs whose rotated
 *     values are finite in fp32.  Inf/NaN inputs give scale byte 0xFF for the
 *     groups they reach.
 */
#ifndef MXQ_H
#define MXQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MXQ_OK = 0,
    MXQ_ERR_INVALID_ARG = 1,   /* rejected before launch; nothing was queued */
    MXQ_ERR_UNSUPPORTED = 2,   /* device is not sm_100 or lacks the needed shared memory */
    MXQ_ERR_CUDA = 3,          /* a CUDA runtime/driver call or the launch failed */
    MXQ_ERR_TIMEOUT = 4        /* a kernel's bounded pipeline wait ran out (see mxq_sync_check) */
} mxq_status;

/*
 * Fused smooth -> rotate -> MXFP4 quantise (DuQuant++ write-up §3.3 online
 * step X * Lambda^-1 * R^, followed by §2.1's MXFP4 quantiser).
 *
 *   X_bf16              in   bf16 [rows, cols], 16-byte aligned
 *   rows, cols          in   rows >= 0; cols >= 0 and cols % 32 == 0
 *   Rhat_bf16           in   bf16 [32, 32] row-major [k][n], 2-byte aligned
 *   Lambda_or_null      in   fp32 [cols], 4-byte aligned, or NULL for no smoothing
 *   out_codes_u8_packed out  uint8 [rows, cols/2], 16-byte aligned
 *   out_scales_e8m0     out  uint8 [rows, cols/32], any alignment
 *   stream              in   cudaStream_t
 *
 * The rotation runs on the tensor cores.  X is the exact bf16 A operand and
 * R^ (or, with Lambda, diag(1/Lambda)·R^ split into three bf16 parts: high,
 * middle and low) is the B operand, with fp32 accumulation.  The scale and the
 * codes are then decided on those fp32 values.
 */
mxq_status mxq_smooth_rotate_quantize(const void *X_bf16, int64_t rows, int64_t cols,
                                      const void *Rhat_bf16, const float *Lambda_or_null,
                                      uint8_t *out_codes_u8_packed, uint8_t *out_scales_e8m0,
                                      void *stream);

/*
 * mxq_smooth_rotate_quantize with the scales written straight into the layout
 * the block-scaled MMA reads them in (DuQuant++ write-up §3.3: the rotated
 * activations feed the MXFP4 linear; §1 and §5.4: Blackwell's native MXFP4
 * tensor cores), so mxq_mxfp4_gemm takes them with no layout pass between.
 * The codes and the scale bytes are the same as mxq_smooth_rotate_quantize's;
 * out_scales_mma holds exactly what mxq_scales_to_mma_layout makes of its
 * scales, padding included (rows past the matrix in the last 128-row block and
 * k-blocks past cols/32 read 0: the call zeroes the buffer first when the
 * shape has such padding, so the kernel itself writes only the scales).
 *
 *   X_bf16, rows, cols, Rhat_bf16, Lambda_or_null, out_codes_u8_packed, stream
 *                       as mxq_smooth_rotate_quantize
 *   out_scales_mma      out  mxq_scales_mma_bytes(rows, cols) bytes, 16-byte aligned
 * Errors as mxq_smooth_rotate_quantize.
 */
mxq_status mxq_smooth_rotate_quantize_mma(const void *X_bf16, int64_t rows, int64_t cols,
                                          const void *Rhat_bf16, const float *Lambda_or_null,
                                          uint8_t *out_codes_u8_packed, uint8_t *out_scales_mma,
                                          void *stream);

/*
 * Same inputs as mxq_smooth_rotate_quantize.  Writes the rotated fp32 values
 * Y = X * Lambda^-1 * R^ (§3.3) instead of quantising them.  It checks the
 * intermediate precision; the quantiser decides on these same values.
 *
 *   out_f32             out  fp32 [rows, cols], 16-byte aligned
 */
mxq_status mxq_smooth_rotate_f32(const void *X_bf16, int64_t rows, int64_t cols,
                                 const void *Rhat_bf16, const float *Lambda_or_null,
                                 float *out_f32, void *stream);

/*
 * The weights' side of the absorption (DuQuant++ write-up, §3.3: Ŵ = R̂ᵀ·Λ·W,
 * done offline so that X̂·Ŵ = X·W).  With W stored transposed, Wt = Wᵀ
 * [rows = n_out, cols = k_in] bf16, each row becomes (row · Λ) · R̂ per
 * 32-column group: the same computation as mxq_smooth_rotate_quantize with Λ
 * multiplying instead of dividing.  The result is quantised to MXFP4 along
 * k_in, in the layout mxq_mxfp4_gemm takes as its B operand.
 *   arguments, layouts and errors as mxq_smooth_rotate_quantize (Λ may be NULL:
 *   then it is identical to mxq_smooth_rotate_quantize without Λ).
 */
mxq_status mxq_weight_rotate_quantize(const void *Wt_bf16, int64_t rows, int64_t cols,
                                      const void *Rhat_bf16, const float *Lambda_or_null,
                                      uint8_t *out_codes_u8_packed, uint8_t *out_scales_e8m0,
                                      void *stream);

/*
 * The same rotation quantised to NVFP4 instead of MXFP4 (DuQuant++ write-up,
 * §5.3, names NVFP4 as another block-scaled format the method suits; it gives
 * no rule for it, so the public NVFP4 format is the one taken).  Each 32-value
 * group of Y = X * Lambda^-1 * R^ is quantised as two blocks of 16 values.
 * There is one E4M3 scale per block and one fp32 tensor scale s_t, which the
 * caller supplies in device memory.  Every decision is made in fp32:
 *   r_t = 1 / (6 s_t);  v = amax(block) * r_t;  s_b = E4M3(v), round to nearest
 *   even, saturating at 448;  s = s_b * s_t;  code_n = E2M1(y_n * (1 / s)) as for MXFP4.
 * A block holding NaN or Inf gets scale 0x7F (E4M3 NaN) and codes 0, and so
 * does a block whose scale is NaN or 0.  With s_t = amax(Y) / (6 * 448), every
 * block scale covers its block.
 *
 *   X_bf16, rows, cols, Rhat_bf16, Lambda_or_null   as mxq_smooth_rotate_quantize
 *   tensor_scale_f32    in   fp32 [1] in device memory, 4-byte aligned; read by the kernel
 *   out_codes_u8_packed out  uint8 [rows, cols/2], 16-byte aligned (even column in the low nibble)
 *   out_scales_e4m3     out  uint8 [rows, cols/16], 2-byte aligned
 *   stream              in   cudaStream_t
 * Errors as mxq_smooth_rotate_quantize; a NULL tensor scale is MXQ_ERR_INVALID_ARG.
 */
mxq_status mxq_smooth_rotate_quantize_nvfp4(const void *X_bf16, int64_t rows, int64_t cols,
                                            const void *Rhat_bf16, const float *Lambda_or_null,
                                            const float *tensor_scale_f32, uint8_t *out_codes_u8_packed,
                                            uint8_t *out_scales_e4m3, void *stream);

/*
 * Row-major E8M0 scales [rows, K/32] (the quantisers' layout) -> the layout
 * Blackwell's block-scaled MMA reads scale factors in.  The output is 512-byte
 * atoms, one per 128 rows × 4 k-blocks, ordered by row block and then k-block.
 * Inside an atom, the scale of row r (0..127) and k-block j (0..3) is byte
 * 16·(r % 32) + 4·(r / 32) + j.  Rows and k-blocks past the matrix are 0.  A
 * lane of the MMA's scale loader thus finds its four 32-bit scale words in one
 * contiguous 16-byte line.  This is layout work only: the same bytes, moved.
 *   scales  in   [rows, K/32] bytes;  K a multiple of 32
 *   out     out  mxq_scales_mma_bytes(rows, K) bytes, 16-byte aligned
 */
size_t mxq_scales_mma_bytes(int64_t rows, int64_t K);
mxq_status mxq_scales_to_mma_layout(const uint8_t *scales, int64_t rows, int64_t K, uint8_t *out, void *stream);

/*
 * The MXFP4 × MXFP4 consumer GEMM on the block-scaled tensor cores (the
 * write-up's §3.3 inference step; §1 and §5.4 name Blackwell's native MXFP4):
 *   Y[m][n] = Σ_k deq(A)[m][k] · deq(B)[n][k],  deq = E2M1 code · 2^(E8M0 byte − 127)
 * A is the activations (mxq_smooth_rotate_quantize's output), B the absorbed
 * weights (mxq_weight_rotate_quantize's output), both K-major: codes two per
 * byte (even k in the low nibble), one scale per 32 k, the scales converted by
 * mxq_scales_to_mma_layout.  The tensor cores accumulate in fp32.
 *   a_codes       in   [M, K/2] bytes, 16-byte aligned
 *   a_scales_mma  in   mxq_scales_mma_bytes(M, K) bytes, 16-byte aligned
 *   b_codes       in   [N, K/2] bytes, 16-byte aligned
 *   b_scales_mma  in   mxq_scales_mma_bytes(N, K) bytes, 16-byte aligned
 *   K                  a multiple of 32; M, N, K < 2^31
 *   out           out  [M, N] row-major, fp32 (out_bf16 = 0) or bf16 rounded to
 *                      nearest even (out_bf16 = 1), 16-byte aligned; K = 0 writes zeros
 *   A 0xFF scale byte (NaN) makes the products it scales NaN.
 * Errors: MXQ_ERR_INVALID_ARG for a bad size or alignment, a host pointer or an
 * output that overlaps an input.
 */
mxq_status mxq_mxfp4_gemm(const uint8_t *a_codes, const uint8_t *a_scales_mma, const uint8_t *b_codes,
                          const uint8_t *b_scales_mma, int64_t M, int64_t N, int64_t K, void *out,
                          int out_bf16, void *stream);

/*
 * The NVFP4 × NVFP4 consumer GEMM (the NVFP4 reading of the write-up's §5.3 on
 * the same block-scaled tensor cores): operands as mxq_smooth_rotate_quantize_nvfp4
 * writes them, one E4M3 scale per 16 k and one fp32 tensor scale per operand:
 *   Y[m][n] = Σ_k deq(A)[m][k] · deq(B)[n][k],
 *   deq = E2M1 code · E4M3 block scale · tensor scale
 * The tensor cores accumulate Σ code·scale·code·scale in fp32; the product of
 * the two tensor scales (fp32) then multiplies every output.
 *   a_codes, b_codes     in   [M, K/2], [N, K/2] bytes, 16-byte aligned
 *   a_scales_mma, ...    in   mxq_nvfp4_scales_mma_bytes(rows, K) bytes, 16-byte aligned:
 *                             the [rows, K/16] E4M3 scales through mxq_nvfp4_scales_to_mma_layout
 *                             (the same 512-byte atoms, each holding 64 k of 128 rows)
 *   a_tensor_scale, ...  in   one fp32 each, device memory, 4-byte aligned; read by the kernel
 *   K, out, out_bf16, errors as mxq_mxfp4_gemm.  A NaN scale (0x7F or 0xFF) makes the
 *   products it scales NaN.
 */
size_t mxq_nvfp4_scales_mma_bytes(int64_t rows, int64_t K);

/*
 * mxq_smooth_rotate_quantize_nvfp4 with the E4M3 scales written straight into
 * the layout mxq_nvfp4_gemm reads (what mxq_nvfp4_scales_to_mma_layout makes of
 * the row-major scales, padding included; zeroed first only when the shape has
 * padding), so the NVFP4 GEMM takes them with no layout pass between.
 *   X_bf16, rows, cols, Rhat_bf16, Lambda_or_null, tensor_scale_f32,
 *   out_codes_u8_packed, stream   as mxq_smooth_rotate_quantize_nvfp4
 *   out_scales_mma      out  mxq_nvfp4_scales_mma_bytes(rows, cols) bytes, 16-byte aligned
 * Errors as mxq_smooth_rotate_quantize_nvfp4.
 */
mxq_status mxq_smooth_rotate_quantize_nvfp4_mma(const void *X_bf16, int64_t rows, int64_t cols,
                                                const void *Rhat_bf16, const float *Lambda_or_null,
                                                const float *tensor_scale_f32, uint8_t *out_codes_u8_packed,
                                                uint8_t *out_scales_mma, void *stream);
mxq_status mxq_nvfp4_scales_to_mma_layout(const uint8_t *scales, int64_t rows, int64_t K, uint8_t *out,
                                          void *stream);
mxq_status mxq_nvfp4_gemm(const uint8_t *a_codes, const uint8_t *a_scales_mma, const float *a_tensor_scale,
                          const uint8_t *b_codes, const uint8_t *b_scales_mma, const float *b_tensor_scale,
                          int64_t M, int64_t N, int64_t K, void *out, int out_bf16, void *stream);

/*
 * Rotation-block-size variants (DuQuant++ write-up, §4.3: rotation blocks of
 * B = 16, 32, 64 or 128 channels, B = 32 found best).  The MXFP4 groups stay
 * at 32 columns.  Each row is cut into cols/B blocks; block x becomes
 * y = (x / Λ) · R_B, with one shared B×B matrix R_B.  Every 32 consecutive
 * columns of y are then quantised exactly as mxq_smooth_rotate_quantize does.
 * B = 32 is mxq_smooth_rotate_quantize itself.  B = 16 runs on the same kernels
 * with the block-diagonal diag(R_16, R_16).  B = 64 and 128 run on a kernel
 * whose MMA is B wide and B deep.
 *
 *   block           16, 32, 64 or 128; cols must be a multiple of max(block, 32)
 *   R_bf16          in   [block][block] bf16 row-major [k][n], 2-byte aligned
 *   Lambda_or_null  in   [cols] fp32, for block 16 or 32 only (NULL for 64, 128)
 *   other arguments, layouts and errors as mxq_smooth_rotate_quantize /
 *   mxq_smooth_rotate_f32; a block width outside the list, cols not a multiple
 *   of it, or Λ with block 64/128 return MXQ_ERR_INVALID_ARG.
 */
mxq_status mxq_rotate_quantize_block(const void *X_bf16, int64_t rows, int64_t cols, int block,
                                     const void *R_bf16, const float *Lambda_or_null,
                                     uint8_t *out_codes_u8_packed, uint8_t *out_scales_e8m0,
                                     void *stream);
mxq_status mxq_rotate_block_f32(const void *X_bf16, int64_t rows, int64_t cols, int block,
                                const void *R_bf16, const float *Lambda_or_null, float *out_f32,
                                void *stream);

/*
 * MXFP4 dequantise: the fake-quant "simulator" of the write-up's §5.1 item 5.
 * Each value is v = E2M1(code) * 2^(byte - 127), with byte 0xFF giving NaN.
 *
 *   codes, scales       in   as produced above; codes 16-byte aligned
 *   rows, cols          in   as above
 *   Rhat_bf16_or_null   in   16-byte aligned.  NULL: write v itself.  It is exactly representable
 *                            in bf16, so the output is bit-exact (overflow
 *                            gives +-Inf).
 *                            non-NULL: undo the rotation, x_k = sum_n v_n R^[k][n]
 *                            (v * R^T), on the tensor cores: v is the exact bf16
 *                            A operand, fp32 accumulation.
 *   Lambda_or_null      in   non-NULL: undo the smoothing too, x_k *= Lambda[k]
 *                            (allowed only together with R^)
 *   out_bf16            out  bf16 [rows, cols], 16-byte aligned; the fp32 result
 *                            rounded to nearest even
 */
mxq_status mxq_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t rows,
                          int64_t cols, const void *Rhat_bf16_or_null,
                          const float *Lambda_or_null, void *out_bf16, void *stream);

/*
 * The per-group MXFP4 quantisation error: the write-up's §4.1, Figure 1, which
 * compares the original activations, a random Hadamard block rotation and the
 * outlier-aware rotation by this error inside each group.  Each group's 32
 * values y = X * Lambda^-1 * R^ (fp32, as the quantiser sees them) are quantised
 * exactly as mxq_smooth_rotate_quantize does, then dequantised to Q(y).  The
 * error is
 *     e_g = ||Q(y) - y||_2 / ||y||_2      (0 for an all-zero group, NaN for a NaN/Inf one)
 * and the call also returns the mean of e_g over all rows * cols/32 groups.  The
 * mean is summed in a fixed order, so it is the same on every run.
 *
 *   X_bf16, rows, cols, Rhat_bf16, Lambda_or_null   as for mxq_smooth_rotate_quantize
 *                                                    (rows, cols > 0)
 *   out_group_err_or_null   out  fp32 [rows, cols/32], 4-byte aligned, or NULL
 *   out_mean                out  one double (device), 8-byte aligned
 *   workspace               in/out  device scratch for per-warp partial sums, 8-byte
 *                                aligned, at least mxq_quant_error_workspace_bytes()
 *                                bytes; caller-owned, overwritten, no state kept
 *
 * If a bounded wait runs out (the device status word then holds MXQ_ERR_TIMEOUT,
 * which mxq_sync_check reports), some partial sums are never written, so the mean
 * is written as NaN rather than summed from stale scratch.
 */
size_t mxq_quant_error_workspace_bytes(int64_t rows, int64_t cols, int with_lambda);
mxq_status mxq_quant_error(const void *X_bf16, int64_t rows, int64_t cols, const void *Rhat_bf16,
                           const float *Lambda_or_null, float *out_group_err_or_null, double *out_mean,
                           void *workspace, size_t workspace_bytes, void *stream);

/*
 * mxq_quant_error without a workspace, for callers that cannot allocate device
 * memory (no counterpart in the write-up; it only changes where scratch lives).
 * Such callers include a plug-in handed only input and output pointers, a
 * process whose framework already holds the GPU's free memory (cudaMalloc
 * would fail), and a latency-critical path that cannot take cudaMalloc's
 * implicit synchronisation.  The partial sums mxq_quant_error keeps in its
 * workspace live instead in a fixed 1 MiB array of device memory inside the
 * library.  Every GPU that loads the library holds it until the process exits.
 * The function itself allocates nothing.
 *
 *   arguments        as mxq_quant_error, without workspace/workspace_bytes
 *   limit            131072 partial sums.  Without Lambda: at most 16,777,216
 *                    groups of 32 (rows * cols <= 536,870,912).  With Lambda:
 *                    one sum per 32 rows x 64 columns, so rows * cols <=
 *                    268,435,456 with rows rounded up to a multiple of 128 and
 *                    cols to a multiple of 64.  Larger inputs return
 *                    MXQ_ERR_INVALID_ARG and mxq_last_cuda_error() says why
 *   set-up           every call looks up the array's device address
 *                    (cudaGetSymbolAddress) with the current device, so the
 *                    address stays right after a device reset; the first call on
 *                    a device also loads the library's device code there, so make
 *                    that first call before any stream capture
 *   sharing          all calls use the same array; each call writes every slot
 *                    it reads, so nothing carries over.  Calls whose GPU work
 *                    overlaps (different streams, no ordering) race on it.
 *   timeout          if a kernel's bounded wait runs out (mxq_sync_check then
 *                    returns MXQ_ERR_TIMEOUT), some slots of that call are never
 *                    written; the mean kernel sees the status word and writes NaN
 *                    (the same holds for mxq_quant_error's workspace)
 */
mxq_status mxq_quant_error_noalloc(const void *X_bf16, int64_t rows, int64_t cols, const void *Rhat_bf16,
                                   const float *Lambda_or_null, float *out_group_err_or_null, double *out_mean,
                                   void *stream);

/*
 * The outlier-aware rotation search that builds R̂ offline (DuQuant++ write-up,
 * §3.2; its pitfalls section asks for the search on the smoothed activations
 * X / Λ, and its implementation notes for double precision).  Steps:
 *   1. the worst group: among the cols/32 channel groups, the [rows, 32] block
 *      of X / Λ with the largest max |value| (the first on ties);
 *   2. R = I;
 *   3. up to max_steps greedy steps.  Each step:
 *      - takes d, the first column of the block holding its largest |value|;
 *      - tries, for every other column j and every grid angle, the Givens
 *        rotation G(d, j) that maps column d to c x_d - s x_j and column j to
 *        s x_d + c x_j;
 *      - keeps the rotation that gives the smallest max |value| of block * G
 *        (the first in (j, angle) order on ties);
 *      - stops if no candidate is strictly below the current max;
 *      - sets R <- R G and block <- block * G.
 * The write-up leaves the angle open.  Here the grid has 2 * n_angle angles,
 * angle a at t = tan(θ/2) = (a' - n_angle) / n_angle with a' = a for
 * a < n_angle and a + 1 otherwise (t runs over [-1, 1] without 0).  Then
 * c = (1 - t²)/(1 + t²) and s = 2t/(1 + t²), each a plain IEEE double expression.
 * Every value a decision depends on is one IEEE double operation, and every
 * reduction is a max, so the result is the same bits as a sequential double
 * evaluation of these steps.
 *
 * All pointers are device memory of the current device; the work is queued on
 * `stream` (2 * max_steps + 6 kernel launches, no host synchronisation).
 *   X_bf16          in   [rows, cols] bf16 row-major, 16-byte aligned; rows >= 1,
 *                        cols >= 32 and a multiple of 32
 *   Lambda_or_null  in   [cols] fp32 per-channel divisor, or NULL for none
 *   max_steps       in   K, 0..65536 (the write-up uses 128)
 *   n_angle         in   1..128; 2 * n_angle angles are tried per column pair
 *   R_out           out  [32][32] double row-major [k][n], 8-byte aligned: the rotation
 *   Rhat_bf16_out_or_null  out  [32][32] bf16, R rounded to nearest even, 2-byte aligned
 *   trace_out_or_null      out  [max_steps][3] int32 (d, j, angle) per step taken
 *   linf_out_or_null       out  [max_steps + 1] double: the block's max |value|
 *                        before each step, and after the last one taken
 *   steps_out_or_null      out  one int32: the number of steps taken
 *   group_out_or_null      out  one int64: the worst group's index
 *   workspace       in   mxq_rotation_search_workspace_bytes(rows, cols, n_angle)
 *                        bytes, 256-byte aligned, caller-owned, overwritten
 * Entries of trace and linf beyond the steps taken are left untouched.
 * Errors: MXQ_ERR_INVALID_ARG for a bad size, a host pointer, a misaligned or
 * too-small buffer, or outputs that overlap X, Λ, each other or the workspace.
 */
size_t mxq_rotation_search_workspace_bytes(int64_t rows, int64_t cols, int n_angle);
mxq_status mxq_rotation_search(const void *X_bf16, int64_t rows, int64_t cols, const float *Lambda_or_null,
                               int max_steps, int n_angle, double *R_out, void *Rhat_bf16_out_or_null,
                               int32_t *trace_out_or_null, double *linf_out_or_null, int32_t *steps_out_or_null,
                               int64_t *group_out_or_null, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Synchronise `stream` and then read and clear the device status word.
 * Returns MXQ_ERR_CUDA if the stream reported an error and MXQ_ERR_TIMEOUT if
 * a kernel's bounded wait ran out since the last check; otherwise MXQ_OK.
 */
mxq_status mxq_sync_check(void *stream);

/*
 * Diagnostic for the failure-detection path (no counterpart on the pages).
 * Queues one single-thread kernel on `stream`.  It waits on a shared-memory
 * barrier that nothing ever completes, using the same bounded wait as the
 * fused kernel's pipeline.  After `timeout_ms` (1..10000) the wait gives up: it
 * sets MXQ_ERR_TIMEOUT in the device status word and writes 2 to
 * *result_device.  A following mxq_sync_check() then returns MXQ_ERR_TIMEOUT
 * and clears the word.  No GPU fault, trap or hang is involved.
 *
 *   result_device   out  one int of device memory, 4-byte aligned
 */
mxq_status mxq_selftest_bounded_wait(uint32_t timeout_ms, int *result_device, void *stream);

/* A static, human-readable string for a status code (never NULL). */
const char *mxq_status_string(mxq_status status);

/* The text of the last CUDA error this thread saw inside the library (static storage). */
const char *mxq_last_cuda_error(void);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int mxq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MXQ_H */
