// search_sm100.cu -- the outlier-aware rotation search (B200, sm_100a).
//
// The DuQuant++ write-up's §3.2 builds the shared 32x32 rotation R̂ offline:
//   1. the worst group is the [rows, 32] channel block of X / Λ with the
//      largest L-infinity norm (the write-up's §3.1 smoothing comes first; its
//      pitfalls section asks for the search on the smoothed activations);
//   2. R starts as the identity;
//   3. up to K greedy steps.  Each step:
//      - finds the column d that holds the block's largest magnitude;
//      - tries a Givens rotation of d with each of the other 31 columns;
//      - keeps the rotation that lowers the block's L-infinity norm most;
//      - applies it to R and to the block;
//   4. R is shared by every group.
// The write-up asks for the search and the matrix in double precision; so
// does this file.  Each candidate's angle comes from a grid on t = tan(θ/2),
// so c and s come from a few IEEE operations rather than from trigonometric
// functions.
//
// Every floating-point operation that a decision depends on is written with
// the round-to-nearest intrinsics (__dmul_rn, __dadd_rn, __dsub_rn,
// __ddiv_rn), so the compiler cannot contract it into an FMA.  The reductions
// are maxima, which are exact in any order.  So every decision, and every bit
// of R, equals that of a plain sequential double-precision evaluation of the
// same steps.
//
// Kernels, in stream order (no kernel waits on another inside the GPU):
//   init     zero the column maxima, the search state and the two candidate tables; R = I
//   colmax   per column of X, the largest |x| (bf16 magnitude bits, NaN skipped)
//   pick     per group, max_k colmax_k / |Λ_k|; the first group with the largest
//   gather   the worst group's block, divided by Λ, column-major in double; its column maxima
//   cand     (per step) for every j != d and every angle, the rotated block's
//            max |value| over columns d and j, by row chunks (rows that cannot
//            hold the max left out), combined with atomicMax
//   select   (per step, one block per row range) the best candidate, found by
//            every block; each block rotates its rows of the two columns; block 0
//            updates R and the trace; the last block to finish sets the two new
//            column maxima.  The candidate tables alternate by step parity, so
//            the next step's table is cleared while this one is read.
//   finish   R in bf16; the step count and the group
#include <cuda_bf16.h>
#include <math_constants.h>

#include "mxq_internal.h"

namespace mxq {
namespace {

constexpr int kGroup = 32;
constexpr int kCandThreads = 256;
constexpr int kCandChunk = 1024;      // rows per cand CTA
constexpr int kSelectThreads = 256;
constexpr int kPickThreads = 512;
constexpr int kSelectWarps = kSelectThreads / 32;
constexpr int kColmaxThreads = 256;

// Search state, at the start of the workspace.  colmax holds the bit patterns of
// non-negative, non-NaN doubles, whose order as unsigned integers is their order
// as numbers, so atomicMax on the bits is a max of the values.
struct SearchState {
    unsigned long long colmax[kGroup];
    unsigned long long nm[2];     // the two rotated columns' new maxima, during a select
    long long group;
    int done;
    int steps;
    unsigned int ticket;          // blocks of the current select that have finished
};
static_assert(sizeof(SearchState) <= 512, "search state must fit its slot");

__device__ __forceinline__ double bits_to_double(unsigned long long b)
{
    return __longlong_as_double(static_cast<long long>(b));
}
__device__ __forceinline__ unsigned long long double_to_bits(double v)
{
    return static_cast<unsigned long long>(__double_as_longlong(v));
}

// Givens grid: angle a of 2n, t = (a' - n) / n with a' = a (a < n) or a + 1,
// c = (1 - t^2) / (1 + t^2), s = 2t / (1 + t^2).
__device__ __forceinline__ void givens_cs(int a, int n, double &c, double &s)
{
    const int ap = a < n ? a : a + 1;
    const double t = __ddiv_rn(static_cast<double>(ap - n), static_cast<double>(n));
    const double t2 = __dmul_rn(t, t);
    const double den = __dadd_rn(1.0, t2);
    c = __ddiv_rn(__dsub_rn(1.0, t2), den);
    s = __ddiv_rn(__dmul_rn(2.0, t), den);
}

// The first column holding the largest value (values are non-negative, non-NaN).
__device__ __forceinline__ int first_argmax32(const double *v)
{
    int d = 0;
    for (int k = 1; k < kGroup; ++k)
        if (v[k] > v[d]) d = k;
    return d;
}

__global__ void __launch_bounds__(1024)
    search_init_kernel(unsigned int *colmax_x, int64_t cols, SearchState *st, unsigned long long *cand, int n_cand,
                       double *R)
{
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (int64_t i = t0; i < cols; i += stride) colmax_x[i] = 0u;
    for (int64_t i = t0; i < n_cand; i += stride) cand[i] = 0ull;
    for (int64_t i = t0; i < kGroup * kGroup; i += stride) R[i] = (i / kGroup == i % kGroup) ? 1.0 : 0.0;
    if (t0 < kGroup) st->colmax[t0] = 0ull;
    if (t0 < 2) st->nm[t0] = 0ull;
    if (t0 == 0) {
        st->ticket = 0u;
        st->group = 0;
        st->done = 0;
        st->steps = 0;
    }
}

// Per column, the largest bf16 magnitude over the rows, as magnitude bits (the
// sign bit cleared).  For non-NaN bf16 values the magnitude bits order like the
// magnitudes; NaN (magnitude bits above 0x7F80) is skipped.  Each thread owns 8
// adjacent columns (one 16-byte load per row) and a strided subset of the rows.
__global__ void __launch_bounds__(kColmaxThreads)
    search_colmax_kernel(const uint4 *__restrict__ X, int64_t rows, int64_t cols, unsigned int *colmax_x)
{
    const int64_t nvec = cols / 8;
    const int64_t v = static_cast<int64_t>(blockIdx.x) * kColmaxThreads + threadIdx.x;
    if (v >= nvec) return;
    unsigned int acc[4] = {0u, 0u, 0u, 0u};
    int64_t r = blockIdx.y;
    const int64_t rs = gridDim.y;
    for (; r + 3 * rs < rows; r += 4 * rs) {
        uint4 q[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) q[u] = __ldcs(X + (r + u * rs) * nvec + v);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const unsigned int w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const unsigned int mag = w[h] & 0x7FFF7FFFu;
                acc[h] = __vmaxu2(acc[h], mag & __vcmpleu2(mag, 0x7F807F80u));
            }
        }
    }
    for (; r < rows; r += rs) {
        const uint4 q = __ldcs(X + r * nvec + v);
        const unsigned int w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const unsigned int mag = w[h] & 0x7FFF7FFFu;
            acc[h] = __vmaxu2(acc[h], mag & __vcmpleu2(mag, 0x7F807F80u));
        }
    }
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const unsigned int lo = acc[h] & 0xFFFFu, hi = acc[h] >> 16;
        if (lo) atomicMax(colmax_x + v * 8 + 2 * h, lo);
        if (hi) atomicMax(colmax_x + v * 8 + 2 * h + 1, hi);
    }
}

// The worst group: per group, the largest |x| / |Λ| over its 32 columns and all
// rows, then the first group holding the largest value.  Division by a fixed
// positive number, rounded to nearest, never reverses an order, so
// max_r (|x_r| / |Λ|) = (max_r |x_r|) / |Λ| exactly: one division per column.
// A NaN quotient (0/0, inf/inf, NaN Λ) is skipped, as it would be element by
// element.
__global__ void __launch_bounds__(kPickThreads)
    search_pick_kernel(const unsigned int *__restrict__ colmax_x, const float *__restrict__ lam, int64_t n_groups,
                       SearchState *st)
{
    double best = -1.0;
    long long bg = 0;
    for (int64_t g = threadIdx.x; g < n_groups; g += kPickThreads) {
        double m = 0.0;
        for (int k = 0; k < kGroup; ++k) {
            const unsigned int mb = colmax_x[g * kGroup + k];
            double v = static_cast<double>(__uint_as_float(mb << 16));
            if (lam) v = __ddiv_rn(v, fabs(static_cast<double>(lam[g * kGroup + k])));
            if (v > m) m = v;
        }
        if (m > best) {
            best = m;
            bg = g;
        }
    }
    // larger value wins; equal values: the smaller group
    __shared__ double sv[kPickThreads / 32];
    __shared__ long long sg[kPickThreads / 32];
    for (int o = 16; o >= 1; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, best, o);
        const long long og = __shfl_xor_sync(0xffffffffu, bg, o);
        if (ov > best || (ov == best && og < bg)) {
            best = ov;
            bg = og;
        }
    }
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (lane == 0) {
        sv[warp] = best;
        sg[warp] = bg;
    }
    __syncthreads();
    if (warp == 0) {
        best = lane < (kPickThreads / 32) ? sv[lane] : -1.0;
        bg = lane < (kPickThreads / 32) ? sg[lane] : 0;
        for (int o = 16; o >= 1; o >>= 1) {
            const double ov = __shfl_xor_sync(0xffffffffu, best, o);
            const long long og = __shfl_xor_sync(0xffffffffu, bg, o);
            if (ov > best || (ov == best && og < bg)) {
                best = ov;
                bg = og;
            }
        }
        if (lane == 0) st->group = bg;
    }
}

// The worst group's block B = X[:, g*32 : g*32+32] / Λ in double, stored
// column-major (B[k * rows + r]) so that one column is contiguous, and the
// maxima of its columns.  One warp per row at a time, lane k = column k.
__global__ void __launch_bounds__(256)
    search_gather_kernel(const uint16_t *__restrict__ X, int64_t rows, int64_t cols, const float *__restrict__ lam,
                         SearchState *st, double *__restrict__ B)
{
    const int lane = threadIdx.x % 32;
    const int64_t g = st->group;
    const int64_t c = g * kGroup + lane;
    const double lk = lam ? static_cast<double>(lam[c]) : 1.0;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
    double m = 0.0;
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32; r < rows; r += warps) {
        const unsigned int xb = X[r * cols + c];
        double v = static_cast<double>(__uint_as_float(xb << 16));
        if (lam) v = __ddiv_rn(v, lk);
        B[lane * rows + r] = v;
        const double a = fabs(v);
        if (a > m) m = a;
    }
    if (m > 0.0) atomicMax(&st->colmax[lane], double_to_bits(m));
}

// Block-wide max of non-negative, non-NaN doubles (every thread gets it).
template <int kThreads>
__device__ __forceinline__ double block_max(double m, double *red)
{
    for (int o = 16; o >= 1; o >>= 1) {
        const double om = __shfl_xor_sync(0xffffffffu, m, o);
        if (om > m) m = om;
    }
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    __syncthreads();
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = lane < kThreads / 32 ? red[lane] : 0.0;
    for (int o = 16; o >= 1; o >>= 1) {
        const double om = __shfl_xor_sync(0xffffffffu, m, o);
        if (om > m) m = om;
    }
    return m;
}

// One greedy step's candidates.  Block (x, y): rows [x*kCandChunk, ...) of the
// block, partner column j = y.
// A row r can be left out when it cannot hold any candidate's max:
//   - its rotated pair (u, w) is bounded by b_r = fl(|x_d| + |x_j|).  Rounding
//     is monotone and |c|, |s| <= 1, so |fl(fl(c x_d) - fl(s x_j))| <= b_r, and
//     the same holds for w;
//   - at the row r* with the largest b, for every angle,
//     max(|u|, |w|) >= sqrt((x_d² + x_j²) / 2) >= b_r* / 2, less a few ulps;
//   - so a row with b_r < 0.499 b_r* never holds a candidate's max, and the max
//     over the rows kept is the max over all rows, bit for bit.
// With an infinite b_r* nothing is left out, because an infinite pair can
// rotate to NaN.  The rows kept are packed in shared memory.  Warp w evaluates
// angles w, w + 8, ... over them.  The largest |rotated value| of the two
// columns goes to cand[j * 2n + angle] by atomicMax on the bits.  The other 30
// columns do not change under G(d, j); the select kernel adds their maxima.
__global__ void __launch_bounds__(kCandThreads)
    search_cand_kernel(const double *__restrict__ B, int64_t rows, int n_angle, const SearchState *st,
                       unsigned long long *cand)
{
    constexpr int kPer = kCandChunk / kCandThreads;
    __shared__ double sx[2][kCandChunk];
    __shared__ double cm[kGroup];
    __shared__ double red[kCandThreads / 32];
    __shared__ int n_kept;
    if (st->done) return;
    if (threadIdx.x < kGroup) cm[threadIdx.x] = bits_to_double(st->colmax[threadIdx.x]);
    if (threadIdx.x == 0) n_kept = 0;
    __syncthreads();
    const int d = first_argmax32(cm);
    const int j = blockIdx.y;
    if (j == d) return;
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kCandChunk;
    const int n = static_cast<int>(rows - r0 < kCandChunk ? rows - r0 : kCandChunk);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    double xd[kPer], xj[kPer], b[kPer];
    double bmax = 0.0;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int i = threadIdx.x + u * kCandThreads;
        xd[u] = i < n ? B[d * rows + r0 + i] : 0.0;
        xj[u] = i < n ? B[j * rows + r0 + i] : 0.0;
        b[u] = __dadd_rn(fabs(xd[u]), fabs(xj[u]));
        if (b[u] > bmax) bmax = b[u];
    }
    bmax = block_max<kCandThreads>(bmax, red);
    const double thr = bmax == CUDART_INF ? 0.0 : __dmul_rn(bmax, 0.4990234375);
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int i = threadIdx.x + u * kCandThreads;
        const bool keep = i < n && b[u] >= thr;
        const unsigned int ballot = __ballot_sync(0xffffffffu, keep);
        int base = 0;
        if (lane == 0 && ballot) base = atomicAdd(&n_kept, __popc(ballot));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (keep) {
            const int pos = base + __popc(ballot & ((1u << lane) - 1u));
            sx[0][pos] = xd[u];
            sx[1][pos] = xj[u];
        }
    }
    __syncthreads();
    const int nk = n_kept;
    const int n_cand_j = 2 * n_angle;
    for (int a = warp; a < n_cand_j; a += kCandThreads / 32) {
        double c, s;
        givens_cs(a, n_angle, c, s);
        double m = 0.0;
        for (int i = lane; i < nk; i += 32) {
            const double x0 = sx[0][i], x1 = sx[1][i];
            const double u = __dsub_rn(__dmul_rn(c, x0), __dmul_rn(s, x1));
            const double w = __dadd_rn(__dmul_rn(s, x0), __dmul_rn(c, x1));
            const double au = fabs(u), aw = fabs(w);
            if (au > m) m = au;
            if (aw > m) m = aw;
        }
        for (int o = 16; o >= 1; o >>= 1) {
            const double om = __shfl_xor_sync(0xffffffffu, m, o);
            if (om > m) m = om;
        }
        if (lane == 0 && m > 0.0) atomicMax(cand + j * n_cand_j + a, double_to_bits(m));
    }
}

// Step `step` of the search, after its cand kernel (or, at step == K, only the
// final L-infinity norm).  Every block takes the same decision from the same
// data:
//   - cur = the block's L-infinity norm (the largest column maximum), column d
//     its first holder;
//   - a candidate's norm is max(its cand entry, the maxima of the 30 other columns);
//   - the first candidate with the smallest norm below cur wins; with none, the
//     search stops.
// Each block then applies B <- B G to its own rows of columns d and j and adds
// their maxima to st->nm by atomicMax.  Block 0 applies R <- R G and records
// the trace.  The last block to finish (a ticket counter; nothing waits) moves
// the two new maxima into st->colmax.  The next step's candidate table is
// cleared here: nobody reads it during this kernel.
__global__ void __launch_bounds__(kSelectThreads)
    search_select_kernel(double *__restrict__ B, int64_t rows, int64_t rows_per_block, int n_angle, int step, int K,
                         SearchState *st, const unsigned long long *__restrict__ cand, unsigned long long *cand_next,
                         double *__restrict__ R, int32_t *trace, double *linf)
{
    __shared__ double cm[kGroup];
    __shared__ double other[kGroup];
    __shared__ double red[kSelectWarps];
    __shared__ double sv[kSelectWarps];
    __shared__ int sc[kSelectWarps];
    if (st->done) return;
    const bool lead = blockIdx.x == 0 && threadIdx.x == 0;
    if (threadIdx.x < kGroup) cm[threadIdx.x] = bits_to_double(st->colmax[threadIdx.x]);
    __syncthreads();
    const int d = first_argmax32(cm);
    const double cur = cm[d];
    if (lead && linf) linf[step] = cur;
    if (step == K) {
        if (lead) st->steps = K;
        return;
    }
    if (threadIdx.x < kGroup) {
        const int j = threadIdx.x;
        double v = 0.0;
        for (int k = 0; k < kGroup; ++k)
            if (k != d && k != j && cm[k] > v) v = cm[k];
        other[j] = v;
    }
    __syncthreads();
    const int n_cand_j = 2 * n_angle;
    const int n_cand = kGroup * n_cand_j;
    double bv = 0.0;
    int bc = -1;
    for (int ci = threadIdx.x; ci < n_cand; ci += kSelectThreads) {
        const int j = ci / n_cand_j;
        if (j == d) continue;
        double v = other[j];
        const double cv = bits_to_double(cand[ci]);
        if (cv > v) v = cv;
        if (v < cur && (bc < 0 || v < bv)) {
            bv = v;
            bc = ci;
        }
    }
    // smallest value wins; equal values: the smaller candidate index; bc < 0 loses
    for (int o = 16; o >= 1; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oc = __shfl_xor_sync(0xffffffffu, bc, o);
        if (oc >= 0 && (bc < 0 || ov < bv || (ov == bv && oc < bc))) {
            bv = ov;
            bc = oc;
        }
    }
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (lane == 0) {
        sv[warp] = bv;
        sc[warp] = bc;
    }
    __syncthreads();
    bv = lane < kSelectWarps ? sv[lane] : 0.0;
    bc = lane < kSelectWarps ? sc[lane] : -1;
    for (int o = 16; o >= 1; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oc = __shfl_xor_sync(0xffffffffu, bc, o);
        if (oc >= 0 && (bc < 0 || ov < bv || (ov == bv && oc < bc))) {
            bv = ov;
            bc = oc;
        }
    }
    for (int i = blockIdx.x * kSelectThreads + threadIdx.x; i < n_cand; i += gridDim.x * kSelectThreads)
        cand_next[i] = 0ull;
    if (bc < 0) {
        if (lead) {
            st->done = 1;
            st->steps = step;
        }
        return;
    }
    const int j = bc / n_cand_j, a = bc % n_cand_j;
    double c, s;
    givens_cs(a, n_angle, c, s);
    if (blockIdx.x == 0 && threadIdx.x < kGroup) {
        double *row = R + threadIdx.x * kGroup;
        const double rd = row[d], rj = row[j];
        row[d] = __dsub_rn(__dmul_rn(c, rd), __dmul_rn(s, rj));
        row[j] = __dadd_rn(__dmul_rn(s, rd), __dmul_rn(c, rj));
    }
    if (lead && trace) {
        trace[3 * step] = d;
        trace[3 * step + 1] = j;
        trace[3 * step + 2] = a;
    }
    double *bd = B + d * rows;
    double *bj = B + j * rows;
    const int64_t lo = static_cast<int64_t>(blockIdx.x) * rows_per_block;
    const int64_t hi = lo + rows_per_block < rows ? lo + rows_per_block : rows;
    double md = 0.0, mj = 0.0;
    for (int64_t r = lo + threadIdx.x; r < hi; r += kSelectThreads) {
        const double xd = bd[r], xj = bj[r];
        const double u = __dsub_rn(__dmul_rn(c, xd), __dmul_rn(s, xj));
        const double w = __dadd_rn(__dmul_rn(s, xd), __dmul_rn(c, xj));
        bd[r] = u;
        bj[r] = w;
        const double au = fabs(u), aw = fabs(w);
        if (au > md) md = au;
        if (aw > mj) mj = aw;
    }
    md = block_max<kSelectThreads>(md, red);
    mj = block_max<kSelectThreads>(mj, red);
    if (threadIdx.x == 0) {
        if (md > 0.0) atomicMax(&st->nm[0], double_to_bits(md));
        if (mj > 0.0) atomicMax(&st->nm[1], double_to_bits(mj));
        __threadfence();
        if (atomicAdd(&st->ticket, 1u) == gridDim.x - 1) {
            __threadfence();
            st->colmax[d] = atomicExch(&st->nm[0], 0ull);
            st->colmax[j] = atomicExch(&st->nm[1], 0ull);
            st->ticket = 0u;
            st->steps = step + 1;
        }
    }
}

// R in bf16 (round to nearest even, straight from double), the step count and the group.
__global__ void __launch_bounds__(kGroup * kGroup)
    search_finish_kernel(const double *__restrict__ R, const SearchState *st, uint16_t *rhat, int32_t *steps_out,
                         int64_t *group_out)
{
    if (rhat) rhat[threadIdx.x] = __bfloat16_as_ushort(__double2bfloat16(R[threadIdx.x]));
    if (threadIdx.x == 0) {
        if (steps_out) *steps_out = st->steps;
        if (group_out) *group_out = st->group;
    }
}

}  // namespace

namespace {

constexpr int64_t align256(int64_t n) { return (n + 255) / 256 * 256; }

struct SearchLayout {
    int64_t cand, colmax_x, block, total;
};

SearchLayout search_layout(int64_t rows, int64_t cols, int n_angle)
{
    SearchLayout L{};
    L.cand = 512;
    L.colmax_x = L.cand + align256(2 * static_cast<int64_t>(kGroup) * 2 * n_angle * 8);   // two tables
    L.block = L.colmax_x + align256(cols * 4);
    L.total = L.block + rows * kGroup * 8;
    return L;
}

}  // namespace

size_t rotation_search_workspace(int64_t rows, int64_t cols, int n_angle)
{
    return static_cast<size_t>(search_layout(rows, cols, n_angle).total);
}

cudaError_t launch_rotation_search(const SearchArgs &a, int num_sms, cudaStream_t stream)
{
    const SearchLayout L = search_layout(a.rows, a.cols, a.n_angle);
    char *ws = static_cast<char *>(a.workspace);
    SearchState *st = reinterpret_cast<SearchState *>(ws);
    unsigned long long *cand = reinterpret_cast<unsigned long long *>(ws + L.cand);
    unsigned int *colmax_x = reinterpret_cast<unsigned int *>(ws + L.colmax_x);
    double *B = reinterpret_cast<double *>(ws + L.block);
    const int n_cand = kGroup * 2 * a.n_angle;

    search_init_kernel<<<num_sms, 1024, 0, stream>>>(colmax_x, a.cols, st, cand, 2 * n_cand, a.R);
    const int64_t nvec = a.cols / 8;
    const int64_t gx = (nvec + kColmaxThreads - 1) / kColmaxThreads;
    int64_t gy = (static_cast<int64_t>(num_sms) * 4 + gx - 1) / gx;
    if (gy > a.rows) gy = a.rows;
    if (gy > 65535) gy = 65535;
    if (gy < 1) gy = 1;
    search_colmax_kernel<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), kColmaxThreads, 0, stream>>>(
        static_cast<const uint4 *>(a.X), a.rows, a.cols, colmax_x);
    search_pick_kernel<<<1, kPickThreads, 0, stream>>>(colmax_x, a.lambda, a.cols / kGroup, st);
    int64_t gb = (a.rows + 7) / 8;
    if (gb > static_cast<int64_t>(num_sms) * 4) gb = static_cast<int64_t>(num_sms) * 4;
    search_gather_kernel<<<static_cast<unsigned>(gb), 256, 0, stream>>>(static_cast<const uint16_t *>(a.X), a.rows,
                                                                        a.cols, a.lambda, st, B);
    const unsigned chunks = static_cast<unsigned>((a.rows + kCandChunk - 1) / kCandChunk);
    int64_t sel_blocks = (a.rows + 2 * kSelectThreads - 1) / (2 * kSelectThreads);
    if (sel_blocks > 2 * static_cast<int64_t>(num_sms)) sel_blocks = 2 * static_cast<int64_t>(num_sms);
    const int64_t rows_per_block = (a.rows + sel_blocks - 1) / sel_blocks;
    for (int step = 0; step < a.max_steps; ++step) {
        unsigned long long *tab = cand + (step & 1) * n_cand;
        unsigned long long *next = cand + ((step + 1) & 1) * n_cand;
        search_cand_kernel<<<dim3(chunks, kGroup), kCandThreads, 0, stream>>>(B, a.rows, a.n_angle, st, tab);
        search_select_kernel<<<static_cast<unsigned>(sel_blocks), kSelectThreads, 0, stream>>>(
            B, a.rows, rows_per_block, a.n_angle, step, a.max_steps, st, tab, next, a.R, a.trace, a.linf);
    }
    search_select_kernel<<<1, kSelectThreads, 0, stream>>>(B, a.rows, a.rows, a.n_angle, a.max_steps, a.max_steps,
                                                           st, cand, cand + n_cand, a.R, a.trace, a.linf);
    search_finish_kernel<<<1, kGroup * kGroup, 0, stream>>>(a.R, st, a.rhat, a.steps, a.group);
    return cudaGetLastError();
}

int rotation_search_launches(int max_steps) { return 2 * max_steps + 6; }

}  // namespace mxq
