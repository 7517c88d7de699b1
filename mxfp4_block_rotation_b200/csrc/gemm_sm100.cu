// gemm_sm100.cu -- the MXFP4 x MXFP4 consumer GEMM on Blackwell's block-scaled tensor cores (B200, sm_100a).
//
// The DuQuant++ write-up's inference step (§3.3): with X̂ = X·Λ⁻¹·R̂ quantised
// online and Ŵ = R̂ᵀ·Λ·W quantised offline, the layer computes X̂·Ŵ, which
// equals X·W up to the quantisation.  On Blackwell both operands stay MXFP4 in
// the MMA (§1 and §5.4 name the native MXFP4 tensor cores):
//   Y[m][n] = sum_k deq(A)[m][k] * deq(B)[n][k],   deq = E2M1 code * 2^(E8M0 byte - 127)
// A = the activations' codes [M, K/2] and scales [M, K/32]; B = the absorbed
// weights, stored transposed ([N, K/2], [N, K/32]), so both are K-major, exactly
// as the quantiser writes them.
//
// One persistent CTA per SM takes 128 x 256 output tiles.  Warp roles (320 threads):
//   warps 0-3  epilogue: TMEM -> registers -> fp32 or bf16 stores (warp w reads lane quarter w)
//   warp 4     TMA producer: per stage, 256 k of A (128 rows x 128 B) and B (256 rows x 128 B),
//              128-byte swizzle, zero fill past the matrix edges, plus the stage's scale atoms
//              (bulk copies of 512-byte atoms: 2 for A, 2 x 2 for B) on a barrier of their own
//   warp 5     TMEM owner and MMA issuer: four tcgen05.mma kind::mxf4 block32 of K = 64 per
//              stage, M = 128, N = 256, fp32 accumulator in TMEM columns 0-255
//   warps 6-9  scale movers: the stage's atoms from shared memory into TMEM with tcgen05.st,
//              in the layout the block-scaled MMA reads: the scales of row r, k-blocks
//              4c..4c+3, form one 32-bit word in lane r % 32 (of every lane quarter) and column
//              base + 4c + r / 32 (A; 8c + r / 32 for the 256 rows of B).  An atom (128 rows x
//              4 k-blocks, row r's word at byte 16 (r % 32) + 4 (r / 32)) holds, in lane l's 16
//              bytes, exactly the four words lane l stores.
// A K = 64 MMA takes two scales per row: bytes 0-1 (first half of a 128-k word) or 2-3,
// chosen by the top two bits of the scale address and the descriptor's scale ids.
// Every wait is bounded (2 s) and raises the status word; nothing waits on another CTA.
#include "pipeline_sm100.cuh"
#include "sm100_bulk.cuh"

namespace mxq {
namespace {

using namespace pipe;

// ------------------------------------------------------------------ PTX used only here

// D (+)= A * B with per-32-k E8M0 scales (MXFP4 operands in shared memory, scales in TMEM).
__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
        :
        : "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
}

// Eight / sixteen 32-bit registers of each lane into consecutive TMEM columns of its lane.
__device__ __forceinline__ void tmem_st_8cols(uint32_t taddr, const uint32_t (&r)[8])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 :
                 : "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                   "r"(r[7])
                 : "memory");
}

__device__ __forceinline__ void tmem_st_16cols(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};"
        :
        : "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Instruction descriptor, kind::mxf4 block-scaled: E2M1 A and B (format 1), UE8M0 scales,
// both K-major, M = 128, N = 256, K = 64; scale ids (the byte pair inside a scale word) added per MMA.
__host__ __device__ constexpr uint32_t idesc_mxf4(int m, int n)
{
    return (1u << 7)                                  // A format: E2M1
           | (1u << 10)                               // B format: E2M1
           | (static_cast<uint32_t>(n >> 3) << 17)    // N / 8
           | (1u << 23)                               // scale format: UE8M0
           | (static_cast<uint32_t>(m >> 4) << 24);   // M / 16
}

// ------------------------------------------------------------------ tiling

constexpr int kGM = 128;                      // tile rows (M)
constexpr int kGN = 256;                      // tile columns (N)
constexpr int kGK = 256;                      // k per stage (128 bytes of codes per row)
constexpr int kGStages = 4;
constexpr int kGAStage = kGM * 128;           // 16 KB
constexpr int kGBStage = kGN * 128;           // 32 KB
constexpr int kGSfStage = 3 * 1024;           // scale atoms: A 2 x 512 B, B 2 row blocks x 2 x 512 B
constexpr int kGStageBytes = kGAStage + kGBStage + kGSfStage;   // 51 KB, a multiple of 1 KB
constexpr int kGThreads = 10 * 32;
constexpr int kGTmaWarp = 4;
constexpr int kGMmaWarp = 5;
constexpr int kGSfWarp0 = 6;
constexpr int kGAccCols = kGN;                // fp32 accumulator: TMEM columns 0..255
constexpr int kGSfaCols = 2 * (kGM / 32);     // per stage: two 128-k words x 4 row blocks
constexpr int kGSfbCols = 2 * (kGN / 32);     // per stage: two 128-k words x 8 row blocks
constexpr int kGSfCols = kGSfaCols + kGSfbCols;
constexpr int kGSmem = kGStages * kGStageBytes + 1024 + 1024;
static_assert(kGAccCols + kGStages * kGSfCols <= 512, "TMEM budget");
static_assert(kGSmem <= 232448, "shared memory budget");

struct GemmBars {
    uint64_t full[kGStages];      // TMA bytes of a stage's operands landed
    uint64_t sf_in[kGStages];     // the stage's scale atoms landed in shared memory
    uint64_t sf_full[kGStages];   // the stage's scales are in TMEM (4 loader warps)
    uint64_t empty[kGStages];     // the stage's MMAs are done (smem and scale columns free)
    uint64_t acc_full;            // the tile's accumulator is complete
    uint64_t acc_empty;           // the epilogue has read the accumulator (4 warps)
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(GemmBars) <= 1024, "barrier block");

// TMEM columns of stage s's scales: all A words first, then all B words, so every
// tcgen05.st starts on a multiple of its width.
__device__ __forceinline__ uint32_t sfa_col(int s) { return kGAccCols + s * kGSfaCols; }
__device__ __forceinline__ uint32_t sfb_col(int s) { return kGAccCols + kGStages * kGSfaCols + s * kGSfbCols; }

__device__ __forceinline__ uint64_t policy_evict_last()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__global__ void __launch_bounds__(kGThreads, 1)
    mxfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const GemmArgs args, unsigned int *status)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *stages = align_1k(smem_raw);
    GemmBars *bars = reinterpret_cast<GemmBars *>(stages + kGStages * kGStageBytes);
    volatile int *abort = &bars->abort;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t tiles_n = (args.N + kGN - 1) / kGN;
    const int64_t n_tiles = ((args.M + kGM - 1) / kGM) * tiles_n;
    const int kt_n = static_cast<int>((args.K + kGK - 1) / kGK);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
            ptx::mbar_init(ptx::smem_addr(&bars->full[s]), 1);
            ptx::mbar_init(ptx::smem_addr(&bars->sf_in[s]), 1);
            ptx::mbar_init(ptx::smem_addr(&bars->sf_full[s]), 4);
            ptx::mbar_init(ptx::smem_addr(&bars->empty[s]), 1);
        }
        ptx::mbar_init(ptx::smem_addr(&bars->acc_full), 1);
        ptx::mbar_init(ptx::smem_addr(&bars->acc_empty), 4);
        ptx::mbar_init(ptx::smem_addr(&bars->drain), 1);
        bars->abort = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tmap_a);
        ptx::prefetch_tmap(&tmap_b);
    }
    if (warp == kGMmaWarp) {
        ptx::tmem_alloc(ptx::smem_addr(&bars->tmem_base), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::griddep_launch_dependents();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = bars->tmem_base;
    ptx::griddep_wait();

    if (warp == kGTmaWarp) {
        if (lane == 0) {
            const uint64_t pol = policy_evict_last();   // A and B tiles are re-read by other CTAs
            int it = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
                const int tm = static_cast<int>(t / tiles_n), tn = static_cast<int>(t % tiles_n);
                for (int kt = 0; kt < kt_n; ++kt, ++it) {
                    const int s = it % kGStages;
                    if (!wait_bar(&bars->empty[s], ((it / kGStages) & 1) ^ 1, abort, status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full = ptx::smem_addr(&bars->full[s]);
                    const uint32_t dst = ptx::smem_addr(stages + s * kGStageBytes);
                    // scale atoms of k-blocks 8kt..8kt+7: two atoms, or one at an odd-sized K tail
                    const int64_t cb0 = 2 * static_cast<int64_t>(kt);
                    const uint32_t n_at = cb0 + 1 < args.cb_n ? 2u : 1u;
                    const int64_t rb0 = 2 * static_cast<int64_t>(tn);
                    const uint32_t n_rb = rb0 + 1 < args.rb_b ? 2u : 1u;
                    // the scale atoms first, on their own barrier: the scale warps can move them
                    // into TMEM while the operand tiles are still in flight
                    const uint32_t sfb = ptx::smem_addr(&bars->sf_in[s]);
                    ptx::mbar_arrive_expect_tx(sfb, n_at * 512u * (1u + n_rb));
                    const uint32_t sf = dst + kGAStage + kGBStage;
                    ptx::bulk_load(sf, args.a_sf + (static_cast<int64_t>(tm) * args.cb_n + cb0) * 512, n_at * 512u, sfb,
                              pol);
                    for (uint32_t h = 0; h < n_rb; ++h)
                        ptx::bulk_load(sf + 1024u + h * 1024u, args.b_sf + ((rb0 + h) * args.cb_n + cb0) * 512,
                                  n_at * 512u, sfb, pol);
                    ptx::mbar_arrive_expect_tx(full, kGAStage + kGBStage);
                    ptx::tma_load_2d(dst, &tmap_a, kt * 128, tm * kGM, full, pol);
                    ptx::tma_load_2d(dst + kGAStage, &tmap_b, kt * 128, tn * kGN, full, pol);
                }
            }
            // let the last copy into each stage land before the CTA can exit
            for (int s = 0; s < kGStages && s < it; ++s) {
                const int last = it - 1 - ((it - 1 - s) % kGStages);
                wait_bar(&bars->full[s], (last / kGStages) & 1, nullptr, status);
                wait_bar(&bars->sf_in[s], (last / kGStages) & 1, nullptr, status);
            }
        }
    } else if (warp >= kGSfWarp0) {
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        int it = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
            const int64_t rb0 = 2 * (t % tiles_n);
            for (int kt = 0; kt < kt_n; ++kt, ++it) {
                const int s = it % kGStages;
                // sf_in[s] is armed only after the stage's previous MMAs freed it, so the scale
                // columns of slot s are free too
                int w_ok = 0;
                if (lane == 0) w_ok = wait_bar(&bars->sf_in[s], (it / kGStages) & 1, abort, status);
                if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
                    ok = false;
                    break;
                }
                const uint32_t sf = ptx::smem_addr(stages + s * kGStageBytes + kGAStage + kGBStage) + 16u * lane;
                uint32_t wa[8], wb[16];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const bool cv = 2 * static_cast<int64_t>(kt) + c < args.cb_n;
                    const uint4 va = cv ? ptx::ld_shared_v4(sf + c * 512) : make_uint4(0, 0, 0, 0);
                    wa[4 * c] = va.x;
                    wa[4 * c + 1] = va.y;
                    wa[4 * c + 2] = va.z;
                    wa[4 * c + 3] = va.w;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const bool v = cv && rb0 + h < args.rb_b;
                        const uint4 vb = v ? ptx::ld_shared_v4(sf + 1024 + h * 1024 + c * 512) : make_uint4(0, 0, 0, 0);
                        wb[8 * c + 4 * h] = vb.x;
                        wb[8 * c + 4 * h + 1] = vb.y;
                        wb[8 * c + 4 * h + 2] = vb.z;
                        wb[8 * c + 4 * h + 3] = vb.w;
                    }
                }
                tmem_st_8cols(tmem_base + lane_base + sfa_col(s), wa);
                tmem_st_16cols(tmem_base + lane_base + sfb_col(s), wb);
                tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&bars->sf_full[s]));
            }
        }
    } else if (warp == kGMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t idesc0 = idesc_mxf4(kGM, kGN);
            int it = 0, tile_i = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++tile_i) {
                if (!wait_bar(&bars->acc_empty, (tile_i & 1) ^ 1, abort, status)) break;
                ptx::tc_fence_after();
                for (int kt = 0; kt < kt_n; ++kt, ++it) {
                    const int s = it % kGStages;
                    const uint32_t par = (it / kGStages) & 1;
                    if (!wait_bar(&bars->full[s], par, abort, status) ||
                        !wait_bar(&bars->sf_full[s], par, abort, status)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_base = ptx::smem_addr(stages + s * kGStageBytes);
                    const uint32_t b_base = a_base + kGAStage;
#pragma unroll
                    for (int j = 0; j < kGK / 64; ++j) {
                        const uint32_t c = j >> 1, byte = 2u * (j & 1);   // 128-k word, byte pair in it
                        const uint32_t sfa = (tmem_base + sfa_col(s) + 4 * c) | (byte << 30);
                        const uint32_t sfb = (tmem_base + sfb_col(s) + 8 * c) | (byte << 30);
                        const uint32_t idesc = idesc0 | (byte << 29) | (byte << 4);
                        mma_mxf4(tmem_base, ptx::smem_desc_sw128(a_base + j * 32), ptx::smem_desc_sw128(b_base + j * 32),
                                 idesc, sfa, sfb, static_cast<uint32_t>(kt | j));
                    }
                    ptx::mma_commit(ptx::smem_addr(&bars->empty[s]));
                }
                if (!ok) break;
                ptx::mma_commit(ptx::smem_addr(&bars->acc_full));
            }
            ptx::mma_commit(ptx::smem_addr(&bars->drain));
            wait_bar(&bars->drain, 0, nullptr, status);
        }
    } else {
        // epilogue: warp w reads TMEM lanes 32w..32w+31 = tile rows 32w..32w+31
        const uint32_t t_row = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
        const bool vec = args.out_bf16 ? (args.N % 8 == 0) : (args.N % 4 == 0);
        int tile_i = 0;
        for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tile_i) {
            int w_ok = 0;
            if (lane == 0) w_ok = wait_bar(&bars->acc_full, tile_i & 1, abort, status);
            if (!__shfl_sync(0xffffffffu, w_ok, 0)) break;
            ptx::tc_fence_after();
            const int64_t row = (t / tiles_n) * kGM + warp * 32 + lane;
            const int64_t col_tile = (t % tiles_n) * kGN;
            uint32_t ra[32], rb[32];
            ptx::tmem_ld_32cols(t_row, ra);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int cb = 0; cb < kGN / 32; ++cb) {
                uint32_t(&cur)[32] = (cb & 1) ? rb : ra;
                uint32_t(&nxt)[32] = (cb & 1) ? ra : rb;
                if (cb + 1 < kGN / 32) ptx::tmem_ld_32cols(t_row + (cb + 1) * 32, nxt);
                const int64_t col0 = col_tile + cb * 32;
                if (row < args.M && col0 < args.N) {
                    if (args.out_bf16) {
                        uint16_t *dst = static_cast<uint16_t *>(args.y) + row * args.N + col0;
                        if (vec && col0 + 32 <= args.N) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                uint32_t w[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    w[e] = pack_bf16x2(__float2bfloat16_rn(__uint_as_float(cur[8 * i + 2 * e])),
                                                       __float2bfloat16_rn(__uint_as_float(cur[8 * i + 2 * e + 1])));
                                ptx::st_global_v4(dst + 8 * i, w[0], w[1], w[2], w[3]);
                            }
                        } else {
                            for (int i = 0; i < 32 && col0 + i < args.N; ++i)
                                dst[i] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(cur[i])));
                        }
                    } else {
                        float *dst = static_cast<float *>(args.y) + row * args.N + col0;
                        if (vec && col0 + 32 <= args.N) {
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                ptx::st_global_v4(dst + 4 * i, cur[4 * i], cur[4 * i + 1], cur[4 * i + 2],
                                                  cur[4 * i + 3]);
                        } else {
                            for (int i = 0; i < 32 && col0 + i < args.N; ++i) dst[i] = __uint_as_float(cur[i]);
                        }
                    }
                }
                if (cb + 1 < kGN / 32) ptx::tmem_wait_ld();
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&bars->acc_empty));
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kGMmaWarp) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, kTmemCols);
    }
}

// One thread per 16-byte row of an atom: row m0 of atom (rb, cb) holds, for the four
// 32-row slices m1, the scales of row rb*128 + 32 m1 + m0 at k-blocks 4cb..4cb+3.
__global__ void __launch_bounds__(256)
    scales_to_mma_kernel(const uint8_t *__restrict__ sc, int64_t rows, int64_t G, int64_t CB, int64_t n_rows16,
                         uint4 *__restrict__ out)
{
    const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
    if (i >= n_rows16) return;
    const int64_t atom = i / 32, m0 = i % 32;
    const int64_t rb = atom / CB, cb = atom % CB;
    uint32_t w[4];
#pragma unroll
    for (int m1 = 0; m1 < 4; ++m1) {
        const int64_t row = rb * 128 + m1 * 32 + m0;
        uint32_t v = 0;
        if (row < rows) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t kb = cb * 4 + j;
                if (kb < G) v |= static_cast<uint32_t>(sc[row * G + kb]) << (8 * j);
            }
        }
        w[m1] = v;
    }
    out[i] = make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace

cudaError_t launch_scales_to_mma(const uint8_t *scales, int64_t rows, int64_t G, uint8_t *out, cudaStream_t stream)
{
    const int64_t CB = (G + 3) / 4;
    const int64_t n = ((rows + 127) / 128) * CB * 32;
    if (n <= 0) return cudaSuccess;
    scales_to_mma_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(scales, rows, G, CB, n,
                                                                                    reinterpret_cast<uint4 *>(out));
    return cudaGetLastError();
}

cudaError_t launch_mxfp4_gemm(const CUtensorMap &tmap_a, const CUtensorMap &tmap_b, const GemmArgs &args,
                              int num_sms, cudaStream_t stream)
{
    const int64_t n_tiles = ((args.M + kGM - 1) / kGM) * ((args.N + kGN - 1) / kGN);
    if (n_tiles <= 0 || args.K <= 0) return cudaSuccess;
    const int grid = static_cast<int>(n_tiles < num_sms ? n_tiles : num_sms);
    unsigned int *status = status_word();
    if (!status) return cudaErrorInvalidSymbol;
    return launch_pdl(mxfp4_gemm_kernel, grid, kGThreads, kGSmem, stream, tmap_a, tmap_b, args, status);
}

}  // namespace mxq
