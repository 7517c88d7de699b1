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
// of B).  The three parts are stacked along N: one group's B is 96 rows (n of the
// high part, then the middle, then the low) x 32 k, so a K = 16 step is ONE MMA
// with N = 96 instead of three with N = 32; the small MMAs' fixed cost in the
// tensor pipe, not HBM, bounded the three-MMA form.  The epilogue adds the three
// 32-column partial results, (low + middle) + high, in fp32.  X stays the exact
// bf16 A operand, so the smoothing adds only ~2^-25 relative error on top of
// fp32 accumulation.  Each epilogue warp stages its 32 rows of codes (32 x 32 B,
// two buffers so that one store can be in flight) and writes them with its own
// TMA bulk tensor store; no warp waits for another.
#include "pipeline_sm100.cuh"

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
constexpr int kColRtOffset = kColBOffset + 2 * kBSlotBytes;
constexpr int kColInvOffset = kColRtOffset + 32 * 32 * 4;     // per slot: 1/Lambda of the tile's channels
constexpr int kColBarOffset = kColInvOffset + 2 * kColTileCols * 8;
constexpr int kColSmemBytes = kColBarOffset + 512 + 1024;
constexpr int kColBuildWarps = 4;                             // warps 10-13
constexpr int kColThreads = (kEpiWarps + 2 + kColBuildWarps) * 32;   // 448
static_assert(kColStages <= kMaxStages && kColAcc * kColAccCols <= 512 && kColStageOffset % 1024 == 0 &&
                  kColBOffset % 1024 == 0 && kBGroupBytes % 512 == 0,
              "smoothing kernel layout");

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
    constexpr bool kCodes = kMode == RotOut::Quant || kMode == RotOut::QuantNv;   // codes via staging + TMA
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align_1k(smem_raw);
    uint8_t *code_tiles = smem;                       // two 2 KB staging buffers per epilogue warp
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
    const int n_ct = static_cast<int>((cols + kColTileCols - 1) / kColTileCols);
    const int n_rt = static_cast<int>((rows + kTileM - 1) / kTileM);
    const UnitSched sched(n_ct, n_rt, blockIdx.x, gridDim.x);

    const uint32_t tmem_base =
        kernel_setup(bars, SetupCfg{kColStages, kColAcc, 1, kColBuildWarps * 32, kMmaWarp}, &tmap_x,
                     kCodes ? &tmap_codes : nullptr);

    if (warp == kTmaWarp) {
        if (lane == 0) {
            const uint64_t pol = ptx::policy_evict_first();
            int it = 0;
            for (; it < sched.n_tiles; ++it) {
                const int s = it % kColStages;
                if (!wait_bar(&bars->empty[s], ((it / kColStages) & 1) ^ 1, abort, status)) break;
                int ui, sub, len;
                sched.at(it, ui, sub, len);
                const int ctile = sched.ct_of_unit(ui), rtile = sched.rt0_of_unit(ui) + sub;
                const uint32_t full = ptx::smem_addr(&bars->full[s]);
                const uint32_t dst = ptx::smem_addr(stages + s * kColStageBytes);
                ptx::mbar_arrive_expect_tx(full, kColStageBytes);
                ptx::tma_load_2d(dst, &tmap_x, ctile * kColTileCols, rtile * kTileM, full, pol);
            }
            drain_loads(bars, kColStages, it, status);
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, kColN);
            const uint32_t b_base0 = ptx::smem_addr(bmat);
            for (int it = 0; it < sched.n_tiles; ++it) {
                const int s = it % kColStages;
                const int a = it % kColAcc;
                int ui, sub, len;
                sched.at(it, ui, sub, len);
                const int slot = ui & 1;
                if (!wait_bar(&bars->full[s], (it / kColStages) & 1, abort, status)) break;
                if (!wait_bar(&bars->acc_empty[a], ((it / kColAcc) & 1) ^ 1, abort, status)) break;
                if (sub == 0 && !wait_bar(&bars->b_full[slot], (ui >> 1) & 1, abort, status)) break;
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
                ptx::mma_commit(ptx::smem_addr(&bars->empty[s]));
                ptx::mma_commit(ptx::smem_addr(&bars->acc_full[a]));
                if (sub == len - 1) ptx::mma_commit(ptx::smem_addr(&bars->b_empty[slot]));
            }
            drain_mmas(bars, status);
        }
    } else if (warp >= kBuildWarp0) {
        // Builders: R^ in fp32, transposed to [n][k]; then per tile 1/Lambda of its 64
        // channels (a reciprocal plus its FMA residual, so R*(1/Lambda) is good to about
        // an ulp), then the two B_g = diag(1/Lambda_g) R^ split three ways into bf16.
        // The weights' side (lam_mul) uses Lambda itself: B_g = diag(Lambda_g) R^.
        const int bt = threadIdx.x - kBuildWarp0 * 32;   // 0..127
        constexpr int kB = kColBuildWarps * 32;
        for (int i = bt; i < 32 * 32; i += kB) {
            const int k = i >> 5, n = i & 31;
            rt[n * 32 + k] = __bfloat162float(__ushort_as_bfloat16(rhat_at(args, k, n)));
        }
        ptx::named_bar_sync(3, kB);
        int built0 = -1, built1 = -1;   // column tile whose B_g each slot holds
        for (int ui = 0; ui < sched.n_units_cta; ++ui) {
            const int slot = ui & 1;
            // one thread waits (bounded) for the slot; the verdict goes to all builders
            // (the flag alternates per unit, so a slow reader never sees the next unit's value)
            if (bt == 0) bars->bl_ok[ui & 1] = wait_bar(&bars->b_empty[slot], ((ui >> 1) & 1) ^ 1, abort, status);
            __syncwarp();
            ptx::named_bar_sync(3, kB);
            if (!*reinterpret_cast<volatile int *>(&bars->bl_ok[ui & 1])) break;
            const int ct = sched.ct_of_unit(ui);
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
                // 2 groups x 32 rows (n) x 4 chunks of 8 k = 256 chunk tasks.  Part p of row n
                // goes to B row p * 32 + n (64-byte swizzle: 16-byte chunk c of row r sits at
                // chunk c ^ ((r >> 1) & 3)).
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
                    uint8_t *bg = bs + j * kBGroupBytes;
                    const uint32_t rows3[3] = {static_cast<uint32_t>(n), static_cast<uint32_t>(32 + n),
                                               static_cast<uint32_t>(64 + n)};
                    const uint4 v3[3] = {make_uint4(hw[0], hw[1], hw[2], hw[3]), make_uint4(mw[0], mw[1], mw[2], mw[3]),
                                         make_uint4(lw[0], lw[1], lw[2], lw[3])};
#pragma unroll
                    for (int pp = 0; pp < 3; ++pp)
                        *reinterpret_cast<uint4 *>(bg + rows3[pp] * 64 + ((c ^ ((rows3[pp] >> 1) & 3u)) << 4)) = v3[pp];
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
        if constexpr (kMode == RotOut::QuantNv) {
            nv_st = *args.nv_scale;
            nv_rt = __frcp_rn(__fmul_rn(6.0f, nv_st));
        }
        const bool scale_vec = (G % 2 == 0) && ((reinterpret_cast<uintptr_t>(args.scales) & 1) == 0);
        // NVFP4 scales are 2 bytes per group: a tile's 4 bytes go as one word when aligned
        const bool nv_vec = (G % 2 == 0) && ((reinterpret_cast<uintptr_t>(args.scales) & 3) == 0);
        // Each warp stages its own 32 rows' codes (32 rows x 32 B, plain layout, two buffers)
        // and stores them with its own TMA store, so the warps of a group never wait for one another.
        const uint32_t wbuf0 = ptx::smem_addr(code_tiles + warp * 2 * kWarpCodeBytes);
        int n_st = 0;
        for (int it = ewg; it < sched.n_tiles; it += 2) {
            const int a = it % kColAcc;
            int ok = 0;
            if (lane == 0) {
                ok = wait_bar(&bars->acc_full[a], (it / kColAcc) & 1, abort, status);
                // this warp's next staging buffer must have been read by the store that used it
                if constexpr (kCodes) ptx::bulk_wait_group_read1();
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            ptx::tc_fence_after();
            int ui, sub, len;
            sched.at(it, ui, sub, len);
            const int ctile = sched.ct_of_unit(ui), rtile = sched.rt0_of_unit(ui) + sub;
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
                } else if constexpr (kMode == RotOut::QuantNv) {
                    uint32_t w[4];
                    const uint32_t bytes = quantize_group_nv(cur, w, nv_rt, nv_st);
                    ptx::st_shared_v4(wbuf + lane * (kColTileG * 16) + j * 16, w[0], w[1], w[2], w[3]);
                    if (nv_vec)
                        sc_word |= bytes << (16 * j);
                    else if (g < G && row_ok)
                        reinterpret_cast<uint16_t *>(args.scales)[row * G + g] = static_cast<uint16_t>(bytes);
                } else {
                    uint32_t w[4];
                    const uint32_t byte = quantize_group(cur, w);
                    ptx::st_shared_v4(wbuf + lane * (kColTileG * 16) + j * 16, w[0], w[1], w[2], w[3]);
                    if (scale_vec)
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
