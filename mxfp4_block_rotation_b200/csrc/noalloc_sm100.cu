// noalloc_sm100.cu -- mxq_quant_error for callers that cannot allocate device memory.
//
// Some callers have no way to obtain scratch memory.  Examples:
//   - a plug-in handed only input and output pointers, with no allocator;
//   - a serving process whose framework has already reserved the GPU's free
//     memory, so cudaMalloc fails;
//   - a latency-critical path that must not take cudaMalloc's implicit device
//     synchronisation.
// For them, mxq_quant_error_noalloc keeps the per-warp partial sums that
// mxq_quant_error needs in a fixed array of device memory that belongs to this
// library.  The array is 1 MiB of doubles: 131072 partial sums.  Without the
// smoothing that covers 131072 * 128 = 16,777,216 groups of 32 values
// (536,870,912 elements); with it, one sum covers 32 rows x 64 columns, so half
// as many elements.  Larger inputs are rejected.
//
// Every GPU that loads the library holds the array until the process exits.
// All calls share it.  Each call writes every slot it later reads, so nothing
// needs clearing between calls; the one exception is a kernel whose bounded wait
// runs out, whose missing slots make the mean kernel write NaN instead (it reads
// the status word).  Two calls whose work overlaps on the GPU race on the array,
// so the caller must order them (one stream, or events).
#include <cstdio>

#include "../../include/mxq.h"
#include "mxq_internal.h"

namespace {

constexpr int64_t kNoAllocPartials = 131072;   // doubles in the array (1 MiB)

static __device__ __align__(256) double g_noalloc_partials[kNoAllocPartials];

// The array's device address on the current device.  Host code may not use the
// symbol itself as a pointer (on the host it names a stand-in object, not device
// memory), so the address is looked up with cudaGetSymbolAddress, with the device
// current, on every call.  Nothing is kept between calls, so the address stays right
// even after a device reset has reloaded the module and moved the array.
mxq_status noalloc_scratch(double **out)
{
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_partials);
    if (e != cudaSuccess || p == nullptr) {
        char msg[160];
        std::snprintf(msg, sizeof msg, "cudaGetSymbolAddress of the no-alloc scratch: %s", cudaGetErrorString(e));
        mxq::set_last_error(msg);
        return MXQ_ERR_CUDA;
    }
    *out = static_cast<double *>(p);
    return MXQ_OK;
}

}  // namespace

extern "C" mxq_status mxq_quant_error_noalloc(const void *X_bf16, int64_t rows, int64_t cols, const void *Rhat_bf16,
                                              const float *Lambda_or_null, float *out_group_err_or_null,
                                              double *out_mean, void *stream)
{
    const size_t need = mxq_quant_error_workspace_bytes(rows, cols, Lambda_or_null != nullptr);
    if (need > sizeof(g_noalloc_partials)) {
        char msg[200];
        std::snprintf(msg, sizeof msg,
                      "invalid argument: %lld x %lld needs %zu bytes of scratch; mxq_quant_error_noalloc has %zu "
                      "(at most 16777216 groups of 32, half that with Lambda)",
                      static_cast<long long>(rows), static_cast<long long>(cols), need, sizeof(g_noalloc_partials));
        mxq::set_last_error(msg);
        return MXQ_ERR_INVALID_ARG;
    }
    double *scratch = nullptr;
    const mxq_status st = noalloc_scratch(&scratch);
    if (st != MXQ_OK) return st;
    // Everything else (argument checks, the two launches) is mxq_quant_error's, with
    // the library's array as the workspace.
    return mxq_quant_error(X_bf16, rows, cols, Rhat_bf16, Lambda_or_null, out_group_err_or_null, out_mean, scratch,
                           sizeof(g_noalloc_partials), stream);
}
