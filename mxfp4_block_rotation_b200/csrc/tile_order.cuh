// tile_order.cuh -- the tile order of the column-tiled smoothing kernel
// (rotate_cols_sm100.cu): tiles of 128 rows x one column tile, walked in units of
// kUnitRows row blocks of one column tile, so that one build of the column tile's B
// operand serves a whole unit.
#pragma once

namespace mxq {
namespace pipe {

// Tile order.  A unit is kUnitRows consecutive row
// blocks of one column tile, so one B_g build serves kUnitRows tiles.  Units are
// numbered band-major (u = band * n_ct + ct) and dealt round robin to the CTAs.
// At any moment the CTAs' units therefore cover whole rows of a couple of row
// bands, which DRAM reads well.  Only the last band can be shorter than
// kUnitRows, and a CTA meets it only in its last units (from unit k_full on).
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
};

// A CTA's tiles in order, advanced by additions only: the unit's column tile ct and
// first row tile rt0, the position sub inside the unit and the unit's length.  Unit
// ui + 1 is unit ui moved by grid in the band-major numbering, i.e. by grid % n_ct
// column tiles and grid / n_ct bands, with a carry into the band.
struct TileCursor {
    int sub, len, ui, ct, rt0;
    int n_ct, step_ct, step_rt, k_full, r_last;
    __device__ explicit TileCursor(const UnitSched &s)
        : sub(0), ui(0), n_ct(s.n_ct), step_ct(s.grid % s.n_ct), step_rt((s.grid / s.n_ct) * kUnitRows),
          k_full(s.k_full), r_last(s.r_last)
    {
        ct = s.cta % s.n_ct;
        rt0 = (s.cta / s.n_ct) * kUnitRows;
        len = k_full > 0 ? kUnitRows : r_last;
    }
    __device__ int rtile() const { return rt0 + sub; }
    // Step to the next unit (the builders walk units, not tiles).
    __device__ void next_unit()
    {
        sub = 0;
        ++ui;
        ct += step_ct;
        rt0 += step_rt;
        if (ct >= n_ct) {
            ct -= n_ct;
            rt0 += kUnitRows;
        }
        len = ui < k_full ? kUnitRows : r_last;
    }
    __device__ void next()
    {
        if (++sub == len) next_unit();
    }
};

}  // namespace pipe
}  // namespace mxq
