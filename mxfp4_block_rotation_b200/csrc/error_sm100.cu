// error_sm100.cu -- mean of the per-group MXFP4 quantisation errors (B200, sm_100a).
//
// The error metric of the DuQuant++ write-up's §4.1 (Figure 1: the normalised
// quantisation error inside each MXFP4 group, averaged over a layer's groups,
// compared for the original activations, a random Hadamard block rotation and
// the outlier-aware rotation).  The rotate kernels' Err mode computes each
// group's error ||Q(y) - y|| / ||y|| in their epilogue.  Each warp adds its
// groups in a fixed order and leaves one partial sum per (stage or tile, warp)
// in a caller-provided workspace.  This kernel adds the partial sums, again in
// a fixed order, so the mean is the same on every run and for any grid size.
#include "mxq_internal.h"

namespace mxq {
namespace {

constexpr int kMeanThreads = 1024;

__global__ void __launch_bounds__(kMeanThreads)
    error_mean_kernel(const double *__restrict__ partials, int64_t n, int64_t n_groups, double *__restrict__ out)
{
    __shared__ double red[kMeanThreads];
    const int64_t per = (n + kMeanThreads - 1) / kMeanThreads;
    const int64_t lo = static_cast<int64_t>(threadIdx.x) * per;
    const int64_t hi = lo + per < n ? lo + per : n;
    double s = 0.0;
    for (int64_t i = lo; i < hi; ++i) s += partials[i];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int step = kMeanThreads / 2; step >= 1; step >>= 1) {
        if (static_cast<int>(threadIdx.x) < step) red[threadIdx.x] += red[threadIdx.x + step];
        __syncthreads();
    }
    if (threadIdx.x == 0) *out = red[0] / static_cast<double>(n_groups);
}

}  // namespace

cudaError_t launch_error_mean(const double *partials, int64_t n_partials, int64_t n_groups, double *out,
                              cudaStream_t stream)
{
    error_mean_kernel<<<1, kMeanThreads, 0, stream>>>(partials, n_partials, n_groups, out);
    return cudaGetLastError();
}

}  // namespace mxq
