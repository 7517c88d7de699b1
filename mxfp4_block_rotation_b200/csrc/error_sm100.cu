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
#include "pipeline_sm100.cuh"

namespace mxq {
namespace {

constexpr int kMeanThreads = 1024;
constexpr int kMeanUnroll = 8;   // loads in flight per thread

// Fixed-order sum of 32 lanes' values (the same tree every run); lane 0 holds it.
__device__ __forceinline__ double warp_tree_sum(double v)
{
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v += __shfl_down_sync(0xffffffffu, v, off);
    return v;
}

// One block.  Thread t adds the elements t + kMeanThreads * (kMeanUnroll * r + u) into
// accumulator u, so each warp load reads 256 contiguous bytes and kMeanUnroll loads per
// thread are in flight together; the accumulators, the lanes and the warps are then
// combined in a fixed order.  The partial sums were just written and sit in L2, so the
// kernel is bound by L2 latency: about n / (kMeanThreads * kMeanUnroll) round trips.
// It is launched as a programmatic dependent of the rotate kernel, so its launch
// overlaps that kernel's tail; griddepcontrol.wait then holds it until every partial
// sum is written and visible.  A rotate kernel whose bounded wait ran out leaves some
// partial sums unwritten and the timeout bit in the status word; the mean is then NaN.
__global__ void __launch_bounds__(kMeanThreads)
    error_mean_kernel(const double *__restrict__ partials, int64_t n, int64_t n_groups, double *__restrict__ out,
                      const unsigned int *status)
{
    __shared__ double red[kMeanThreads / 32];
    ptx::griddep_wait();
    if (*reinterpret_cast<const volatile unsigned int *>(status) & kStatusTimeout) {
        if (threadIdx.x == 0) *out = __longlong_as_double(0x7FF8000000000000ll);
        return;
    }
    double acc[kMeanUnroll];
#pragma unroll
    for (int u = 0; u < kMeanUnroll; ++u) acc[u] = 0.0;
    constexpr int64_t kStep = static_cast<int64_t>(kMeanThreads) * kMeanUnroll;
    for (int64_t base = threadIdx.x; base < n; base += kStep) {
        double v[kMeanUnroll];
#pragma unroll
        for (int u = 0; u < kMeanUnroll; ++u) {
            const int64_t i = base + static_cast<int64_t>(u) * kMeanThreads;
            v[u] = i < n ? partials[i] : 0.0;
        }
#pragma unroll
        for (int u = 0; u < kMeanUnroll; ++u) acc[u] += v[u];
    }
    double s = acc[0];
#pragma unroll
    for (int u = 1; u < kMeanUnroll; ++u) s += acc[u];
    s = warp_tree_sum(s);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x < 32) {
        s = warp_tree_sum(red[threadIdx.x]);
        if (threadIdx.x == 0) *out = s / static_cast<double>(n_groups);
    }
}

}  // namespace

cudaError_t launch_error_mean(const double *partials, int64_t n_partials, int64_t n_groups, double *out,
                              cudaStream_t stream)
{
    unsigned int *status = status_word();
    if (!status) return cudaErrorInvalidSymbol;
    return pipe::launch_pdl(error_mean_kernel, 1, kMeanThreads, 0, stream, partials, n_partials, n_groups, out,
                            static_cast<const unsigned int *>(status));
}

}  // namespace mxq
