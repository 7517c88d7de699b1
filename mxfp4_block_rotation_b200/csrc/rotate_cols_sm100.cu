// rotate_cols_sm100.cu -- fused smooth -> rotate -> MXFP4-quantise kernel (B200, sm_100a).
//
// The online step of the DuQuant++ write-up (jsqmd.com/news/928156) with the
// SmoothQuant scale: X_hat = X * Lambda^-1 * R^ (§3.1, §3.3), quantised to MXFP4 as
// in §2.1.  The B operand depends on the channel group, B_g = diag(1/Lambda_g)·R^,
// so an MMA must hold one column group over 128 token rows.  A tile is 128 rows x
// 64 columns (2 groups): one 128-byte-swizzled TMA box.
//
// Warp roles as in the flat kernel, with four builder warps (10-13).  Per unit
// (4 row blocks of one column tile) they make the tile's two B_g in fp32: a
// reciprocal per channel plus its FMA residual, so R*(1/Lambda) is good to about
// an ulp.  Each B_g is split three ways into bf16, high + middle + low (~24 bits
// of B).  A builder thread owns one column n of R^ and one k-chunk of 8 for the
// whole kernel, so its R^ values stay in registers; a warp shares the k-chunk, so
// its reads of 1/Lambda are broadcasts and its stores hit distinct banks.  The three
// parts are stacked along N: one group's B is 96 rows (n of the high part, then
// the middle, then the low) x 32 k, so a K = 16 step is ONE MMA with N = 96.  An
// MMA's cost follows the bytes it reads from shared memory (A once, B's 96 rows),
// so one N = 96 MMA per step is cheaper than three N = 32 MMAs, each reading A.
// The epilogue adds the three 32-column partial results, (low + middle) + high,
// in fp32.  X stays the exact bf16 A operand, so the smoothing adds only ~2^-25
// relative error on top of fp32 accumulation.  Each epilogue warp stages its 32
// rows of codes (32 x 32 B, 32-byte swizzle so that the staging stores are
// conflict free; two buffers so that one store can be in flight) and writes them
// with its own TMA bulk tensor store; no warp waits for another.
//
// The MMA thread is the pipeline's critical path, so it does only waits, the MMAs
// and one commit per tile.  The tile order advances by additions (no division per
// tile), and the epilogue's leader, which sees each tile's MMAs complete, hands its
// shared-memory stage back to the TMA producer.
#include "pipeline_sm100.cuh"
#include "tile_order.cuh"

namespace mxq {
namespace {

using namespace pipe;

constexpr int kColTileCols = 64;                              // columns per tile
constexpr int kColTileG = kColTileCols / 32;                  // groups per tile
constexpr int kColParts = 3;                                  // bf16 parts of B, stacked along N
constexpr int kColN = 32 * kColParts;                         // MMA N per group: 96
constexpr int kColAcc = 2;                                    // accumulator stages
constexpr int kColAccCols = kColTileG * kColN;                // 192 TMEM columns per stage
constexpr int kColStageBytes = kTileM * kColTileCols * 2;     // 16 KB of bf16 per stage: one TMA box
constexpr int kBGroupBytes = kColN * 64;                      // one group's B: 96 rows x 64 B, 64-byte swizzle
constexpr int kBSlotBytes = kColTileG * kBGroupBytes;         // 12 KB
constexpr int kColStages = 6;
constexpr int kWarpCodeBytes = 32 * kColTileG * 16;           // one epilogue warp's 32 rows of codes (1 KB)
constexpr int kColStageOffset = kEpiWarps * 2 * kWarpCodeBytes;   // code staging first: 2 buffers per epilogue warp
constexpr int kColBOffset = kColStageOffset + kColStages * kColStageBytes;
constexpr int kColInvOffset = kColBOffset + 2 * kBSlotBytes;   // per slot: 1/Lambda of the tile's channels
constexpr int kColBarOffset = kColInvOffset + 2 * kColTileCols * 8;
constexpr int kColSmemBytes = kColBarOffset + 512 + 1024;
constexpr int kColBuildWarps = 4;                             // warps 10-13
constexpr int kColThreads = (kEpiWarps + 2 + kColBuildWarps) * 32;   // 448
static_assert(kColStages <= kMaxStages && kColStages % 2 == 0 && kColAcc == 2 && kColAcc * kColAccCols <= 512 &&
                  kColStageOffset % 1024 == 0 && kColBOffset % 1024 == 0 && kBGroupBytes % 512 == 0 &&
                  kColInvOffset % 16 == 0,
              "smoothing kernel layout (an epilogue group takes every other tile, so every other stage)");

// cur += part, element-wise in fp32 (round to nearest), two at a time with the packed add.
__device__ __forceinline__ void add_pairs(uint32_t (&cur)[32], const uint32_t (&part)[32])
{
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float2 v = __fadd2_rn(make_float2(__uint_as_float(cur[2 * i]), __uint_as_float(cur[2 * i + 1])),
                                    make_float2(__uint_as_float(part[2 * i]), __uint_as_float(part[2 * i + 1])));
        cur[2 * i] = __float_as_uint(v.x);
        cur[2 * i + 1] = __float_as_uint(v.y);
    }
}

template <RotOut kMode>
__global__ void __launch_bounds__(kColThreads, 1)
    rotate_cols_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_codes,
                       const RotArgs args, unsigned int *status)
{
    constexpr bool kCodes = kMode == RotOut::Quant || rot_nvfp4(kMode) || kMode == RotOut::QuantMma;   // codes via staging + TMA
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1k(smem_raw);
    uint8_t *code_tiles = smem;                       // two 2 KB staging buffers per epilogue warp
    uint8_t *stages = smem + kColStageOffset;
    uint8_t *bmat = smem + kColBOffset;
    float2 *inv_tab = reinterpret_cast<float2 *>(smem + kColInvOffset);   // [slot][channel] (1/L, residual)
    Bars *bars = reinterpret_cast<Bars *>(smem + kColBarOffset);
    volatile int *abort = &bars->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t rows = args.rows;
    const int64_t cols = args.cols;
    const int64_t G = cols / 32;
    const int n_ct = static_cast<int>((cols + kColTileCols - 1) / kColTileCols);
    const int n_rt = static_cast<int>((rows + kTileM - 1) / kTileM);
    const UnitSched sched(n_ct, n_rt, blockIdx.x, gridDim.x);

    const uint32_t tmem_base =
        kernel_setup(bars, SetupCfg{kColStages, kColAcc, 1, kColBuildWarps * 32, kMmaWarp}, &tmap_x,
                     kCodes ? &tmap_codes : nullptr);

    if (warp == kTmaWarp) {
        if (lane == 0) {
            const uint64_t pol = ptx::policy_evict_first();
            TileCursor cur(sched);
            int it = 0, s = 0, ph = 1;
            for (; it < sched.n_tiles; ++it, cur.next()) {
                // stage s is free once the epilogue has seen the MMAs that read it complete
                if (!wait_bar(&bars->empty[s], ph, abort, status)) break;
                const uint32_t full = ptx::smem_addr(&bars->full[s]);
                const uint32_t dst = ptx::smem_addr(stages + s * kColStageBytes);
                ptx::mbar_arrive_expect_tx(full, kColStageBytes);
                ptx::tma_load_2d(dst, &tmap_x, cur.ct * kColTileCols, cur.rtile() * kTileM, full, pol);
                if (++s == kColStages) {
                    s = 0;
                    ph ^= 1;
                }
            }
            drain_loads(bars, kColStages, it, status);
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, kColN);
            const uint32_t b_base0 = ptx::smem_addr(bmat);
            TileCursor cur(sched);
            int s = 0, s_ph = 0;
            for (int it = 0; it < sched.n_tiles; ++it, cur.next()) {
                const int a = it & (kColAcc - 1);
                const int slot = cur.ui & 1;
                if (!wait_bar(&bars->full[s], s_ph, abort, status)) break;
                if (!wait_bar(&bars->acc_empty[a], ((it >> 1) & 1) ^ 1, abort, status)) break;
                if (cur.sub == 0 && !wait_bar(&bars->b_full[slot], (cur.ui >> 1) & 1, abort, status)) break;
                ptx::tc_fence_after();
                // Descriptors built once per tile; each MMA adds a compile-time offset to the
                // start-address field (16-byte units; addresses stay below 256 KB, so no carry).
                const uint64_t ad0 = ptx::smem_desc_sw128(ptx::smem_addr(stages + s * kColStageBytes));
                const uint64_t bd0 = ptx::smem_desc_sw64(b_base0 + slot * kBSlotBytes);
                const uint32_t d_base = tmem_base + static_cast<uint32_t>(a * kColAccCols);
#pragma unroll
                for (int j = 0; j < kColTileG; ++j) {
#pragma unroll
                    for (int kh = 0; kh < 2; ++kh)
                        ptx::mma_bf16(d_base + j * kColN, ad0 + ((j * 64 + kh * 32) >> 4),
                                      bd0 + ((j * kBGroupBytes + kh * 32) >> 4), idesc, kh);
                }
                // one commit: the epilogue learns of the tile and frees its shared-memory stage
                ptx::mma_commit(ptx::smem_addr(&bars->acc_full[a]));
                if (cur.sub == cur.len - 1) ptx::mma_commit(ptx::smem_addr(&bars->b_empty[slot]));
                if (++s == kColStages) {
                    s = 0;
                    s_ph ^= 1;
                }
            }
            drain_mmas(bars, status);
        }
    } else if (warp >= kBuildWarp0) {
        // Builders: thread bt owns column n = bt % 32 of R^ and the k-chunk c = bt / 32 (k = 8c..8c+7)
        // for both groups of every tile, so its eight R^ values live in registers.  Per unit: 1/Lambda
        // of the tile's 64 channels (a reciprocal plus its FMA residual, so R*(1/Lambda) is good to
        // about an ulp) into shared memory, then per group the eight entries of B_g = diag(1/Lambda_g) R^
        // split three ways into bf16, stored to B rows n, 32 + n and 64 + n (16-byte chunk c; 64-byte
        // swizzle: chunk c of row r sits at chunk c ^ ((r >> 1) & 3)).  The weights' side (lam_mul)
        // uses Lambda itself: B_g = diag(Lambda_g) R^.
        const int bt = threadIdx.x - kBuildWarp0 * 32;   // 0..127
        constexpr int kB = kColBuildWarps * 32;
        const int bn = bt & 31, bc = bt >> 5;
        float rr[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) rr[e] = __bfloat162float(__ushort_as_bfloat16(rhat_at(args, bc * 8 + e, bn)));
        TileCursor cur(sched);
        int built0 = -1, built1 = -1;   // column tile whose B_g each slot holds
        for (int ui = 0; ui < sched.n_units_cta; ++ui, cur.next_unit()) {
            const int slot = ui & 1;
            // one thread waits (bounded) for the slot; the verdict goes to all builders
            // (the flag alternates per unit, so a slow reader never sees the next unit's value)
            if (bt == 0) bars->bl_ok[ui & 1] = wait_bar(&bars->b_empty[slot], ((ui >> 1) & 1) ^ 1, abort, status);
            __syncwarp();
            ptx::named_bar_sync(3, kB);
            if (!*reinterpret_cast<volatile int *>(&bars->bl_ok[ui & 1])) break;
            const int ct = cur.ct;
            if ((slot ? built1 : built0) != ct) {
                if (slot)
                    built1 = ct;
                else
                    built0 = ct;
                const int64_t ch_tile = static_cast<int64_t>(ct) * kColTileCols;
                float2 *inv = inv_tab + slot * kColTileCols;
                if (bt < kColTileCols) {
                    const int64_t ch = ch_tile + bt;
                    float ih = 0.0f, il = 0.0f;
                    if (ch < cols) {
                        const float lam = args.lambda[ch];
                        if (args.lam_mul) {
                            ih = lam;   // the weights' side: R * Lambda, one rounding
                        } else {
                            ih = __frcp_rn(lam);
                            il = __fmul_rn(__fmaf_rn(-lam, ih, 1.0f), ih);   // 1/lam - ih, to working precision
                        }
                    }
                    inv[bt] = make_float2(ih, il);
                }
                ptx::named_bar_sync(3, kB);
                uint8_t *bs = bmat + slot * kBSlotBytes;
#pragma unroll
                for (int j = 0; j < kColTileG; ++j) {
                    const float4 *iv4 = reinterpret_cast<const float4 *>(inv + j * 32 + bc * 8);
                    uint32_t hw[4], mw[4], lw[4];
#pragma unroll
                    for (int e2 = 0; e2 < 4; ++e2) {
                        const float4 iv = iv4[e2];   // (1/L, residual) of k = 8c + 2 e2 and 8c + 2 e2 + 1
                        __nv_bfloat16 h[2], m[2], l[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const float r = rr[2 * e2 + u];
                            const float val = __fmaf_rn(r, u ? iv.z : iv.x, __fmul_rn(r, u ? iv.w : iv.y));   // R / Lambda
                            // val = hi + mid + lo to ~24 bits; each residual is exact in fp32
                            h[u] = __float2bfloat16_rn(val);
                            const float r1 = val - __bfloat162float(h[u]);
                            m[u] = __float2bfloat16_rn(r1);
                            l[u] = __float2bfloat16_rn(r1 - __bfloat162float(m[u]));
                        }
                        hw[e2] = pack_bf16x2(h[0], h[1]);
                        mw[e2] = pack_bf16x2(m[0], m[1]);
                        lw[e2] = pack_bf16x2(l[0], l[1]);
                    }
                    uint8_t *bg = bs + j * kBGroupBytes;
                    const uint4 v3[3] = {make_uint4(hw[0], hw[1], hw[2], hw[3]), make_uint4(mw[0], mw[1], mw[2], mw[3]),
                                         make_uint4(lw[0], lw[1], lw[2], lw[3])};
#pragma unroll
                    for (int pp = 0; pp < 3; ++pp) {
                        const uint32_t row = static_cast<uint32_t>(pp * 32 + bn);
                        *reinterpret_cast<uint4 *>(bg + row * 64 + ((static_cast<uint32_t>(bc) ^ ((row >> 1) & 3u)) << 4)) =
                            v3[pp];
                    }
                }
                ptx::fence_proxy_async_smem();
            }
            ptx::mbar_arrive(ptx::smem_addr(&bars->b_full[slot]));
        }
    } else {
        const int q = warp & 3;
        const int ewg = warp >> 2;
        // NVFP4: the tensor scale s_t and r_t = 1 / (6 s_t), once per thread
        float nv_st = 0.0f, nv_rt = 0.0f;
        if constexpr (rot_nvfp4(kMode)) {
            nv_st = *args.nv_scale;
            nv_rt = __frcp_rn(__fmul_rn(6.0f, nv_st));
        }
        const bool scale_vec = (G % 2 == 0) && ((reinterpret_cast<uintptr_t>(args.scales) & 1) == 0);
        // NVFP4 scales are 2 bytes per group: a tile's 4 bytes go as one word when aligned
        const bool nv_vec = (G % 2 == 0) && ((reinterpret_cast<uintptr_t>(args.scales) & 3) == 0);
        // Each warp stages its own 32 rows' codes (32 rows x 32 B, 32-byte swizzle, two buffers)
        // and stores them with its own TMA store, so the warps of a group never wait for one another.
        const uint32_t wbuf0 = ptx::smem_addr(code_tiles + warp * 2 * kWarpCodeBytes);
        int n_st = 0;
        TileCursor cur(sched);
        if (ewg) cur.next();
        // this group's tiles are it = ewg, ewg + 2, ...; tile it used stage it % kColStages
        int s = ewg;
        for (int it = ewg; it < sched.n_tiles; it += 2, cur.next(), cur.next()) {
            const int a = it & (kColAcc - 1);
            int ok = 0;
            if (lane == 0) {
                ok = wait_bar(&bars->acc_full[a], (it >> 1) & 1, abort, status);
                // the tile's MMAs are complete, so its shared-memory stage can be refilled
                if (ok && q == 0) ptx::mbar_arrive(ptx::smem_addr(&bars->empty[s]));
                // this warp's next staging buffer must have been read by the store that used it
                if constexpr (kCodes) ptx::bulk_wait_group_read1();
            }
            if ((s += 2) >= kColStages) s -= kColStages;
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            ptx::tc_fence_after();
            const int ctile = cur.ct, rtile = cur.rtile();
            const uint32_t wbuf = wbuf0 + (n_st & 1) * kWarpCodeBytes;
            const int r_local = q * 32 + lane;
            const int64_t row = static_cast<int64_t>(rtile) * kTileM + r_local;
            const bool row_ok = row < rows;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * kColAccCols;
            uint32_t sc_word = 0;
            double err_acc = 0.0;   // Err mode: this row's groups of the tile, in order
#pragma unroll
            for (int j = 0; j < kColTileG; ++j) {
                // the group's value = (low + middle) + high: the three 32-column partials
                uint32_t cur[32], part[32], hi[32];
                const uint32_t tg = t_row + j * kColN;
                ptx::tmem_ld_32cols(tg + 64, cur);    // low
                ptx::tmem_ld_32cols(tg + 32, part);   // middle
                ptx::tmem_ld_32cols(tg, hi);          // high: all three loads in flight, one wait
                ptx::tmem_wait_ld();
                add_pairs(cur, part);
                if (j == kColTileG - 1) {
                    // the tile's last TMEM reads have landed: free the accumulator stage now
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(ptx::smem_addr(&bars->acc_empty[a]));
                }
                add_pairs(cur, hi);
                const int64_t g = static_cast<int64_t>(ctile) * kColTileG + j;
                if constexpr (kMode == RotOut::F32) {
                    if (g < G && row_ok) {
                        float *dst = args.y + row * cols + g * 32;
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            ptx::st_global_v4(dst + 4 * i, cur[4 * i], cur[4 * i + 1], cur[4 * i + 2],
                                              cur[4 * i + 3]);
                    }
                } else if constexpr (kMode == RotOut::Err) {
                    if (g < G && row_ok) {
                        uint32_t w[4];
                        float e;
                        quantize_group_err(cur, w, e);
                        if (args.err) args.err[row * G + g] = e;
                        err_acc += static_cast<double>(e);
                    }
                } else if constexpr (rot_nvfp4(kMode)) {
                    uint32_t w[4];
                    const uint32_t bytes = quantize_group_nv(cur, w, nv_rt, nv_st);
                    // 32-byte swizzle: chunk j of row lane sits at chunk j ^ ((lane >> 2) & 1)
                    ptx::st_shared_v4(wbuf + lane * 32 + ((j ^ ((lane >> 2) & 1)) << 4), w[0], w[1], w[2], w[3]);
                    if (kMode == RotOut::QuantNvMma || nv_vec)
                        sc_word |= bytes << (16 * j);
                    else if (g < G && row_ok)
                        reinterpret_cast<uint16_t *>(args.scales)[row * G + g] = static_cast<uint16_t>(bytes);
                } else {
                    uint32_t w[4];
                    const uint32_t byte = quantize_group(cur, w);
                    ptx::st_shared_v4(wbuf + lane * 32 + ((j ^ ((lane >> 2) & 1)) << 4), w[0], w[1], w[2], w[3]);
                    if (kMode == RotOut::QuantMma || scale_vec)
                        sc_word |= byte << (8 * j);
                    else if (g < G && row_ok)
                        args.scales[row * G + g] = static_cast<uint8_t>(byte);
                }
            }
            if constexpr (kMode == RotOut::Err) {
                const double sum = warp_sum(err_acc);
                if (lane == 0) args.partials[(static_cast<int64_t>(rtile) * n_ct + ctile) * 4 + q] = sum;
            }
            if constexpr (kCodes) {
                if constexpr (kMode == RotOut::QuantNv) {
                    // two groups x two E4M3 bytes: 4 bytes at group 2 ctile of the row
                    if (nv_vec && row_ok)
                        reinterpret_cast<uint32_t *>(args.scales)[(row * G) / 2 + ctile] = sc_word;
                } else if constexpr (kMode == RotOut::QuantNvMma) {
                    // the tile's blocks 4 ctile .. 4 ctile + 3 fill one 4-byte word of the atom: one
                    // 32-bit store, or 16 bits for a last odd group
                    if (row_ok) {
                        const int64_t g0 = static_cast<int64_t>(ctile) * kColTileG;
                        uint8_t *dst = args.sf_mma + sf_mma_offset(row, 2 * g0, (2 * G + 3) >> 2);
                        if (g0 + 1 < G)
                            *reinterpret_cast<uint32_t *>(dst) = sc_word;
                        else
                            *reinterpret_cast<uint16_t *>(dst) = static_cast<uint16_t>(sc_word);
                    }
                } else if constexpr (kMode == RotOut::QuantMma) {
                    // the tile's groups 2 ctile and 2 ctile + 1 share one 4-byte word of the atom
                    // (from an even byte): one 16-bit store, or one byte for a last odd group
                    if (row_ok) {
                        const int64_t g0 = static_cast<int64_t>(ctile) * kColTileG;
                        uint8_t *dst = args.sf_mma + sf_mma_offset(row, g0, (G + 3) >> 2);
                        if (g0 + 1 < G)
                            *reinterpret_cast<uint16_t *>(dst) = static_cast<uint16_t>(sc_word);
                        else
                            *dst = static_cast<uint8_t>(sc_word);
                    }
                } else if (scale_vec && row_ok) {
                    *reinterpret_cast<uint16_t *>(args.scales + row * G + static_cast<int64_t>(ctile) * kColTileG) =
                        static_cast<uint16_t>(sc_word);
                }
                // this warp's 32 rows complete -> one bulk store (rows/columns past the tensor are clipped)
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    ptx::tma_store_2d(&tmap_codes, ctile * (kColTileCols / 2), rtile * kTileM + q * 32, wbuf);
                    ptx::bulk_commit_group();
                }
                ++n_st;
            }
        }
        if constexpr (kCodes) {
            if (lane == 0) ptx::bulk_wait_group0();   // stores done before the CTA's shared memory goes
        }
    }
    kernel_teardown(tmem_base, kMmaWarp);
}

static_assert(kColSmemBytes <= 232448, "shared memory budget");

}  // namespace

cudaError_t launch_rotate_cols(const CUtensorMap &tmap_x, const CUtensorMap &tmap_codes, const RotArgs &args,
                               RotOut mode, int num_sms, cudaStream_t stream)
{
    const int64_t n_tiles = ((args.rows + kTileM - 1) / kTileM) * ((args.cols + kColTileCols - 1) / kColTileCols);
    if (n_tiles <= 0) return cudaSuccess;
    const int grid = static_cast<int>(n_tiles < num_sms ? n_tiles : num_sms);
    unsigned int *status = status_word();
    if (!status) return cudaErrorInvalidSymbol;
    if (mode == RotOut::Quant)
        return launch_pdl(rotate_cols_kernel<RotOut::Quant>, grid, kColThreads, kColSmemBytes, stream, tmap_x,
                          tmap_codes, args, status);
    if (mode == RotOut::QuantMma)
        return launch_pdl(rotate_cols_kernel<RotOut::QuantMma>, grid, kColThreads, kColSmemBytes, stream, tmap_x,
                          tmap_codes, args, status);
    if (mode == RotOut::QuantNvMma)
        return launch_pdl(rotate_cols_kernel<RotOut::QuantNvMma>, grid, kColThreads, kColSmemBytes, stream, tmap_x,
                          tmap_codes, args, status);
    if (mode == RotOut::Err)
        return launch_pdl(rotate_cols_kernel<RotOut::Err>, grid, kColThreads, kColSmemBytes, stream, tmap_x,
                          tmap_codes, args, status);
    if (mode == RotOut::QuantNv)
        return launch_pdl(rotate_cols_kernel<RotOut::QuantNv>, grid, kColThreads, kColSmemBytes, stream, tmap_x,
                          tmap_codes, args, status);
    return launch_pdl(rotate_cols_kernel<RotOut::F32>, grid, kColThreads, kColSmemBytes, stream, tmap_x, tmap_codes,
                      args, status);
}

int64_t rotate_cols_partials(int64_t rows, int64_t cols)
{
    return ((rows + kTileM - 1) / kTileM) * ((cols + kColTileCols - 1) / kColTileCols) * 4;
}

}  // namespace mxq
