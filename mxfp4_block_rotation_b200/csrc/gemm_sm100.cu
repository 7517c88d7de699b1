// gemm_sm100.cu -- the MXFP4 x MXFP4 consumer GEMM on Blackwell's block-scaled tensor cores (B200, sm_100a).
//
// The DuQuant++ write-up's inference step (§3.3): with X̂ = X·Λ⁻¹·R̂ quantised
// online and Ŵ = R̂ᵀ·Λ·W quantised offline, the layer computes X̂·Ŵ, which
// equals X·W up to the quantisation.  On Blackwell both operands stay MXFP4 in
// the MMA (§1 and §5.4 name the native MXFP4 tensor cores):
//   Y[m][n] = sum_k deq(A)[m][k] * deq(B)[n][k],   deq = E2M1 code * 2^(E8M0 byte - 127)
// A = the activations' codes [M, K/2] and scales [M, K/32]; B = the absorbed
// weights, stored transposed ([N, K/2], [N, K/32]), so both are K-major, exactly
// as the quantiser writes them.  The scales come in the MMA's atom layout (512-byte
// atoms of 128 rows x 4 k-blocks; row r's word at byte 16 (r % 32) + 4 (r / 32)).
//
// CTA pairs (clusters of two, tcgen05 cta_group::2) share each 256 x 256 output tile:
// CTA r holds rows 128 r .. 128 r + 127 of the tile's A and rows (n) 128 r .. 128 r + 127
// of its B in shared memory, and its TMEM holds its 128 output rows x all 256 columns
// plus its own scales (A: its rows; B: all 256).  The even CTA issues one M = 256,
// N = 256, K = 64 MMA per step that reads both CTAs' tiles, so each CTA brings in only
// half of B: 35 KB per 256-k stage (A 16 KB + B 16 KB + scale atoms 3 KB) against 51 KB
// for a 128 x 256 tile on one CTA.  The mainloop is bound by the bytes in flight per SM
// (six stages fill shared memory), so fewer bytes per stage is what pays.  Warp roles
// (256 threads per CTA):
//   warps 0-3  epilogue (both CTAs): TMEM lanes 32w.. -> fp32 or bf16 stores, then an
//              arrival on the even CTA's acc_empty
//   warp 4     TMA (both CTAs): per stage its A rows, its half of B, its A row block's
//              scale atoms and both of B's row blocks' atoms, all counted on the even
//              CTA's full[s] (tensor copies with cta_group::2, each into its own CTA only)
//   warp 5     TMEM owner (both CTAs) and, in the even CTA, the MMA issuer: four
//              kind::mxf4 block32 MMAs per stage, fp32 accumulator in TMEM columns 0-255;
//              one commit multicast to both CTAs frees each stage (empty[s]) and one
//              completes each tile (acc_full)
//   warps 6-7  scale copies (even CTA): tcgen05.cp of the stage's atoms into both CTAs'
//              TMEM (32x128b, replicated over the four lane quarters), the copies of a
//              stage alternating between the two warps, each warp committing its own to
//              sf_ready[s] (two arrivals).  Issued from their own warps the copies run
//              ahead of the MMAs; issued by the MMA thread before each stage's MMAs they
//              cost a quarter of the time.  Two issuing warps instead of one: NVFP4's
//              twelve copies per stage 0.246 -> 0.217 ms at 8192x4096x14336, MXFP4's six
//              unchanged, bit-identical output.
// A K = 64 MMA takes two scales per row: bytes 0-1 (first half of a 128-k word) or 2-3,
// chosen by the top two bits of the scale address and the descriptor's scale ids.
// Every wait on a barrier is bounded (2 s) and raises the status word; the two CTAs
// of a pair meet at the hardware cluster barrier only at start and end.
#include "pipeline_sm100.cuh"
#include "sm100_bulk.cuh"

namespace mxq {
namespace {

using namespace pipe;

// ------------------------------------------------------------------ PTX used only here

// Instruction descriptor, kind::mxf4 block-scaled: E2M1 A and B (format 1), UE8M0 scales,
// both K-major, M = 128, N = 256, K = 64; scale ids (the byte pair inside a scale word) added per MMA.
__host__ __device__ constexpr uint32_t idesc_mxf4(int m, int n, bool e8m0 = true)
{
    return (1u << 7)                                  // A format: E2M1
           | (1u << 10)                               // B format: E2M1
           | (static_cast<uint32_t>(n >> 3) << 17)    // N / 8
           | ((e8m0 ? 1u : 0u) << 23)                 // scale format: UE8M0 (MXFP4) or UE4M3 (NVFP4)
           | (static_cast<uint32_t>(m >> 4) << 24);   // M / 16
}

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// The shared::cluster address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// A tile of this CTA's operand into its own shared memory; the bytes count on the
// mbarrier at bar_cluster (the even CTA's).  The data lands in this CTA only.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int32_t x, int32_t y,
                                                 uint32_t bar_cluster, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void mma_mxf4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
        :
        : "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
}

// The same with NVFP4 operands: E2M1 codes, one E4M3 scale per 16 k (a K = 64 MMA takes the
// four scales of a 32-bit TMEM word).
__device__ __forceinline__ void mma_nvf4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
        :
        : "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
}

// Arrive on the mbarrier at bar_cluster (either CTA's) once the pair MMAs issued so far are done.
__device__ __forceinline__ void commit_pair(uint32_t bar_cluster)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
                 : "memory");
}

// One commit whose arrival goes to the barrier at this CTA-relative shared-memory offset in
// both CTAs of the pair (CTA mask 0b11): half the commits of one per CTA, on the MMA
// thread that paces the mainloop (MXFP4 0.192 -> 0.185 ms at 8192 x 4096 x 14336).
__device__ __forceinline__ void commit_pair_both(uint32_t bar_local)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 ::"r"(bar_local), "h"(static_cast<uint16_t>(3))
                 : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_slot, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_slot), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// tcgen05.cp of one 512-byte scale atom (32 rows of 16 B) into TMEM, four columns from
// taddr, replicated over the four lane quarters, in both CTAs of the pair (each from its
// own shared memory at the same offset).
__device__ __forceinline__ void tmem_cp_atom_pair(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Shared-memory descriptor of a scale atom for tcgen05.cp: no swizzle, 8-row core
// matrices of 16-byte rows, 128 B apart (stride byte offset); one core matrix along K.
__device__ __forceinline__ uint64_t smem_desc_atom(uint32_t saddr)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);   // start address, 16-B units
    d |= static_cast<uint64_t>(128 >> 4) << 16;           // leading byte offset (one core matrix: unused)
    d |= static_cast<uint64_t>(128 >> 4) << 32;           // stride byte offset: next 8 rows
    d |= static_cast<uint64_t>(1) << 46;                  // descriptor version (sm100)
    return d;                                             // layout 0: no swizzle
}

__device__ __forceinline__ uint64_t policy_evict_last()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// 32 accumulator columns of one output row (col0 < N) as bf16 or fp32: 16-byte stores
// when the row's chunk is whole and aligned, element stores at the right edge.
__device__ __forceinline__ void store_row_chunk(const GemmArgs &args, int64_t row, int64_t col0,
                                                const uint32_t (&cur)[32], bool vec)
{
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
                ptx::st_global_v4(dst + 4 * i, cur[4 * i], cur[4 * i + 1], cur[4 * i + 2], cur[4 * i + 3]);
        } else {
            for (int i = 0; i < 32 && col0 + i < args.N; ++i) dst[i] = __uint_as_float(cur[i]);
        }
    }
}

constexpr int kGK = 256;                      // k per stage (128 bytes of codes per row)
constexpr int kGTmaWarp = 4;
constexpr int kGMmaWarp = 5;
constexpr int kGAccCols = 256;                // fp32 accumulator: TMEM columns 0..255

constexpr int kPM = 256;                      // pair tile rows (128 per CTA)
constexpr int kPN = 256;                      // pair tile columns
constexpr int kPAStage = 128 * 128;           // this CTA's 128 rows x 256 k: 16 KB
constexpr int kPBStage = 128 * 128;           // this CTA's half of B: 16 KB
constexpr int kPThreads = 8 * 32;             // warps 0-3 epilogue, 4 TMA, 5 MMA, 6-7 scale copies
constexpr int kPCpWarps = 2;                  // the copies alternate between them
constexpr int kPCpWarp = 6;
constexpr int kPMaxStages = 6;

// Per format: MXFP4 scales cover 32 k (a 512-byte atom = 128 rows x 128 k), NVFP4 scales 16 k
// (an atom = 128 rows x 64 k), so a 256-k stage holds 2 or 4 atoms per 128-row block.
template <bool kNv>
struct PairCfg {
    static constexpr int kAtoms = kNv ? 4 : 2;                       // atoms per stage per row block
    static constexpr int kStages = kNv ? 5 : 6;
    static constexpr int kSfStage = 3 * kAtoms * 512;                 // A: its row block; B: two row blocks
    static constexpr int kStageBytes = kPAStage + kPBStage + kSfStage;   // 35 KB or 38 KB
    static constexpr int kTx = 2 * kStageBytes;                      // bytes a stage brings into the pair
    static constexpr int kSmem = kStages * kStageBytes + 1024 + 1024;
    static constexpr int kSfaCols = 4 * kAtoms;                       // scale words x 4 row blocks
    static constexpr int kSfbCols = 8 * kAtoms;                       // x 8 row blocks
    static_assert(kStages <= kPMaxStages, "barrier arrays");
    static_assert(kGAccCols + kStages * (kSfaCols + kSfbCols) <= 512, "TMEM budget (pairs)");
    static_assert(kSmem <= 232448, "shared memory budget (pairs)");
    __device__ static uint32_t sfa_col(int s) { return kGAccCols + s * kSfaCols; }
    __device__ static uint32_t sfb_col(int s) { return kGAccCols + kStages * kSfaCols + s * kSfbCols; }
};

struct PairBars {
    uint64_t full[kPMaxStages];      // even CTA: both CTAs' operand and scale bytes of a stage landed
    uint64_t empty[kPMaxStages];     // the stage's pair MMAs are done (from the even CTA's commit)
    uint64_t sf_ready[kPMaxStages];  // even CTA: the stage's scales have been copied into both CTAs' TMEM
    uint64_t acc_full;               // the tile's accumulator is complete (from the even CTA's commit)
    uint64_t acc_empty;              // even CTA: both CTAs' epilogues have read the accumulator (8 warps)
    uint64_t drain;
    uint64_t cp_drain;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(PairBars) <= 1024, "barrier block (pairs)");

template <bool kNv>
__global__ void __launch_bounds__(kPThreads, 1)
    mxfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                      const GemmArgs args, unsigned int *status)
{
    using C = PairCfg<kNv>;
    constexpr int kPStages = C::kStages;
    constexpr int kPStageBytes = C::kStageBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *stages = align_1k(smem_raw);
    PairBars *bars = reinterpret_cast<PairBars *>(stages + kPStages * kPStageBytes);
    volatile int *abort = &bars->abort;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();   // 0: the even CTA, which issues the MMAs
    const int64_t pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    const int64_t tiles_n = (args.N + kPN - 1) / kPN;
    const int64_t n_tiles = ((args.M + kPM - 1) / kPM) * tiles_n;
    const int kt_n = static_cast<int>((args.K + kGK - 1) / kGK);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            ptx::mbar_init(ptx::smem_addr(&bars->full[s]), 1);
            ptx::mbar_init(ptx::smem_addr(&bars->empty[s]), 1);
            ptx::mbar_init(ptx::smem_addr(&bars->sf_ready[s]), kPCpWarps);
        }
        ptx::mbar_init(ptx::smem_addr(&bars->acc_full), 1);
        ptx::mbar_init(ptx::smem_addr(&bars->acc_empty), 8);
        ptx::mbar_init(ptx::smem_addr(&bars->drain), 1);
        ptx::mbar_init(ptx::smem_addr(&bars->cp_drain), kPCpWarps);
        bars->abort = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tmap_a);
        ptx::prefetch_tmap(&tmap_b);
        ptx::prefetch_tmap(&tmap_sfa);
        ptx::prefetch_tmap(&tmap_sfb);
    }
    if (warp == kGMmaWarp) {
        tmem_alloc_pair(ptx::smem_addr(&bars->tmem_base), kTmemCols);
        tmem_relinquish_pair();
    }
    ptx::griddep_launch_dependents();
    ptx::tc_fence_before();
    __syncthreads();
    cluster_sync();   // both CTAs' barriers exist before either signals the other's
    ptx::tc_fence_after();
    const uint32_t tmem_base = bars->tmem_base;
    ptx::griddep_wait();

    if (warp == kGTmaWarp) {
        if (lane == 0) {
            const uint64_t pol = policy_evict_last();   // A and B tiles are re-read by other pairs
            int it = 0;
            bool ok = true;
            for (int64_t t = pair; ok && t < n_tiles; t += n_pairs) {
                const int tm2 = static_cast<int>(t / tiles_n), tn = static_cast<int>(t % tiles_n);
                for (int kt = 0; kt < kt_n; ++kt, ++it) {
                    const int s = it % kPStages;
                    if (!wait_bar(&bars->empty[s], ((it / kPStages) & 1) ^ 1, abort, status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t dst = ptx::smem_addr(stages + s * kPStageBytes);
                    const uint32_t full0 = mapa(ptx::smem_addr(&bars->full[s]), 0);
                    if (rank == 0) ptx::mbar_arrive_expect_tx(ptx::smem_addr(&bars->full[s]), C::kTx);
                    // this CTA's A rows and half of B; its A row block's scale atoms and the atoms of
                    // both of B's row blocks (zero past the matrices' edges)
                    tma_load_2d_pair(dst, &tmap_a, kt * 128, tm2 * kPM + static_cast<int>(rank) * 128, full0, pol);
                    tma_load_2d_pair(dst + kPAStage, &tmap_b, kt * 128, tn * kPN + static_cast<int>(rank) * 128, full0,
                                     pol);
                    // scale atoms in boxes of two (256 words); NVFP4 has four per stage
                    const uint32_t sfd = dst + kPAStage + kPBStage;
#pragma unroll
                    for (int h2 = 0; h2 < C::kAtoms / 2; ++h2) {
                        const int x = kt * C::kAtoms * 128 + h2 * 256;
                        tma_load_2d_pair(sfd + h2 * 1024, &tmap_sfa, x, 2 * tm2 + static_cast<int>(rank), full0, pol);
                        tma_load_2d_pair(sfd + C::kAtoms * 512 + h2 * 2048, &tmap_sfb, x, 2 * tn, full0, pol);
                    }
                }
            }
            // the last copies into each stage land before the CTA can exit (the even CTA's
            // full[s] counts both CTAs' bytes; the cluster barrier at the end covers the odd CTA)
            if (rank == 0) {
                for (int s = 0; s < kPStages && s < it; ++s) {
                    const int last = it - 1 - ((it - 1 - s) % kPStages);
                    wait_bar(&bars->full[s], (last / kPStages) & 1, nullptr, status);
                }
            }
        }
    } else if (warp == kGMmaWarp) {
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc0 = idesc_mxf4(kPM, kPN, !kNv);
            int it = 0, tile_i = 0;
            bool ok = true;
            for (int64_t t = pair; ok && t < n_tiles; t += n_pairs, ++tile_i) {
                if (!wait_bar(&bars->acc_empty, (tile_i & 1) ^ 1, abort, status)) break;
                ptx::tc_fence_after();
                for (int kt = 0; kt < kt_n; ++kt, ++it) {
                    const int s = it % kPStages;
                    // full[s] then sf_ready[s] (both copy warps' copies of the stage's scales done)
                    if (!wait_bar(&bars->full[s], (it / kPStages) & 1, abort, status) ||
                        !wait_bar(&bars->sf_ready[s], (it / kPStages) & 1, abort, status)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_base = ptx::smem_addr(stages + s * kPStageBytes);
                    const uint32_t b_base = a_base + kPAStage;
#pragma unroll
                    for (int j = 0; j < kGK / 64; ++j) {
                        // MXFP4: a word holds the scales of 128 k, the MMA takes bytes 0-1 or 2-3;
                        // NVFP4: a word holds the four scales of 64 k, one word per MMA
                        const uint32_t c = kNv ? j : j >> 1, byte = kNv ? 0u : 2u * (j & 1);
                        const uint32_t sfa = (tmem_base + C::sfa_col(s) + 4 * c) | (byte << 30);
                        const uint32_t sfb = (tmem_base + C::sfb_col(s) + 8 * c) | (byte << 30);
                        const uint32_t idesc = idesc0 | (byte << 29) | (byte << 4);
                        const uint64_t ad = ptx::smem_desc_sw128(a_base + j * 32);
                        const uint64_t bd = ptx::smem_desc_sw128(b_base + j * 32);
                        if constexpr (kNv)
                            mma_nvf4_pair(tmem_base, ad, bd, idesc, sfa, sfb, static_cast<uint32_t>(kt | j));
                        else
                            mma_mxf4_pair(tmem_base, ad, bd, idesc, sfa, sfb, static_cast<uint32_t>(kt | j));
                    }
                    commit_pair_both(ptx::smem_addr(&bars->empty[s]));
                }
                if (!ok) break;
                commit_pair_both(ptx::smem_addr(&bars->acc_full));
            }
            commit_pair(mapa(ptx::smem_addr(&bars->drain), 0));
            wait_bar(&bars->drain, 0, nullptr, status);
        }
    } else if (warp >= kPCpWarp && warp < kPCpWarp + kPCpWarps) {
        const int cpw = warp - kPCpWarp;
        // the stages' scale atoms into both CTAs' TMEM, ahead of the MMAs that read them.  A
        // stage's columns are free once its bytes are back: the producer reloads a stage only
        // after the MMAs that read its previous contents (and scales) completed.
        if (lane == 0 && rank == 0) {
            int it = 0;
            bool ok = true;
            for (int64_t t = pair; ok && t < n_tiles; t += n_pairs) {
                for (int kt = 0; kt < kt_n; ++kt, ++it) {
                    const int s = it % kPStages;
                    if (!wait_bar(&bars->full[s], (it / kPStages) & 1, abort, status)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t sf_base = ptx::smem_addr(stages + s * kPStageBytes) + kPAStage + kPBStage;
                    // A's atoms c at sf_base + 512 c; B's (row block h, atom c) in boxes of two
                    // atoms by two row blocks: sf_base + 512 kAtoms + 2048 (c / 2) + 1024 h + 512 (c % 2)
#pragma unroll
                    for (int c = 0; c < C::kAtoms; ++c) {
                        // copy t = 3c (A's atom), 3c + 1 + h (B's): warp t % 2 issues it, so each
                        // warp's copies are half the stage's and its commit covers its own
                        if (cpw == (c & 1))
                            tmem_cp_atom_pair(tmem_base + C::sfa_col(s) + 4 * c, smem_desc_atom(sf_base + c * 512));
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            if (cpw == ((c + h + 1) & 1))
                                tmem_cp_atom_pair(tmem_base + C::sfb_col(s) + 8 * c + 4 * h,
                                                  smem_desc_atom(sf_base + C::kAtoms * 512 + (c / 2) * 2048 + h * 1024 +
                                                                 (c % 2) * 512));
                    }
                    commit_pair(mapa(ptx::smem_addr(&bars->sf_ready[s]), 0));
                }
            }
            commit_pair(mapa(ptx::smem_addr(&bars->cp_drain), 0));   // no copy in flight at exit
            wait_bar(&bars->cp_drain, 0, nullptr, status);
        }
    } else if (warp < 4) {
        // epilogue: warp w reads TMEM lanes 32w..32w+31 = this CTA's rows 32w..32w+31 of the tile
        const uint32_t t_row = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
        const bool vec = args.out_bf16 ? (args.N % 8 == 0) : (args.N % 4 == 0);
        const uint32_t acc_empty0 = mapa(ptx::smem_addr(&bars->acc_empty), 0);
        // NVFP4: the product of the two tensor scales multiplies every output
        const float alpha = kNv ? __fmul_rn(*args.a_tscale, *args.b_tscale) : 1.0f;
        int tile_i = 0;
        for (int64_t t = pair; t < n_tiles; t += n_pairs, ++tile_i) {
            int w_ok = 0;
            if (lane == 0) w_ok = wait_bar(&bars->acc_full, tile_i & 1, abort, status);
            if (!__shfl_sync(0xffffffffu, w_ok, 0)) break;
            ptx::tc_fence_after();
            const int64_t row = (t / tiles_n) * kPM + static_cast<int64_t>(rank) * 128 + warp * 32 + lane;
            const int64_t col_tile = (t % tiles_n) * kPN;
            uint32_t ra[32], rb[32];
            ptx::tmem_ld_32cols(t_row, ra);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int cb = 0; cb < kPN / 32; ++cb) {
                uint32_t(&cur)[32] = (cb & 1) ? rb : ra;
                uint32_t(&nxt)[32] = (cb & 1) ? ra : rb;
                if (cb + 1 < kPN / 32) ptx::tmem_ld_32cols(t_row + (cb + 1) * 32, nxt);
                const int64_t col0 = col_tile + cb * 32;
                if constexpr (kNv) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) cur[i] = __float_as_uint(__fmul_rn(__uint_as_float(cur[i]), alpha));
                }
                if (row < args.M && col0 < args.N) store_row_chunk(args, row, col0, cur, vec);
                if (cb + 1 < kPN / 32) ptx::tmem_wait_ld();
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty0);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    cluster_sync();   // neither CTA leaves while the other may still touch its barriers, smem or TMEM
    if (warp == kGMmaWarp) {
        ptx::tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
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

namespace {

template <bool kNv>
cudaError_t launch_pairs(const CUtensorMap &tmap_a, const CUtensorMap &tmap_b, const CUtensorMap &tmap_sfa,
                         const CUtensorMap &tmap_sfb, const GemmArgs &args, int num_sms, cudaStream_t stream)
{
    unsigned int *status = status_word();
    if (!status) return cudaErrorInvalidSymbol;
    // clusters of two CTAs, one pair per two SMs, persistent over the 256 x 256 tiles
    const int64_t n_tiles = ((args.M + kPM - 1) / kPM) * ((args.N + kPN - 1) / kPN);
    if (n_tiles <= 0 || args.K <= 0) return cudaSuccess;
    const int64_t pairs = n_tiles < num_sms / 2 ? n_tiles : num_sms / 2;
    constexpr int smem = PairCfg<kNv>::kSmem;
    const void *fn = reinterpret_cast<const void *>(mxfp4_gemm_kernel<kNv>);
    cudaError_t e = smem_optin(fn, smem, false);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    cfg.blockDim = dim3(kPThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, mxfp4_gemm_kernel<kNv>, tmap_a, tmap_b, tmap_sfa, tmap_sfb, args, status);
    if (e == cudaSuccess) return e;
    (void)cudaGetLastError();   // refused: set the opt-in again (a device reset clears it) and retry once
    if ((e = smem_optin(fn, smem, true)) != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, mxfp4_gemm_kernel<kNv>, tmap_a, tmap_b, tmap_sfa, tmap_sfb, args, status);
}

}  // namespace

cudaError_t launch_mxfp4_gemm(const CUtensorMap &tmap_a, const CUtensorMap &tmap_b, const CUtensorMap &tmap_sfa,
                              const CUtensorMap &tmap_sfb, const GemmArgs &args, int num_sms, cudaStream_t stream)
{
    return args.nvfp4 ? launch_pairs<true>(tmap_a, tmap_b, tmap_sfa, tmap_sfb, args, num_sms, stream)
                      : launch_pairs<false>(tmap_a, tmap_b, tmap_sfa, tmap_sfb, args, num_sms, stream);
}

}  // namespace mxq
