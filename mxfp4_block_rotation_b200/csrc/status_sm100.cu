// status_sm100.cu -- the library's device status word, its bounded-wait
// self-test and the host-side read-and-clear.
//
// The kernels' bounded waits record MXQ_ERR_TIMEOUT here (atomicOr).  The word is
// a file-scope __device__ variable, one per device that loads the library.
// Kernels get its device address as an argument, so every translation unit
// shares the one word.
#include <mutex>

#include "pipeline_sm100.cuh"

namespace mxq {

namespace {

__device__ unsigned int g_status;

using namespace pipe;

// Diagnostic: one thread waits on an mbarrier phase that nothing completes, so the
// bounded wait must run out, set the status word and return.  It exercises the
// same wait routine as the pipelines, without any TMA, MMA or TMEM in play.
__global__ void bounded_wait_selftest(uint64_t timeout_ns, int *result, unsigned int *status)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    abort_flag = 0;
    ptx::mbar_init(ptx::smem_addr(&bar), 1);
    ptx::fence_mbar_init();
    const bool ok = wait_bar(&bar, 0, &abort_flag, status, timeout_ns);
    *result = ok ? 1 : (abort_flag ? 2 : 3);
    ptx::mbar_arrive(ptx::smem_addr(&bar));   // complete the phase before exit
}

// (kernel, device, bytes) triples whose shared-memory opt-in has been set.
struct OptIn {
    const void *func;
    int dev;
    int smem;
};
std::mutex g_optin_mu;
OptIn g_optin[256];
int g_n_optin = 0;

}  // namespace

unsigned int *status_word()
{
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    return static_cast<unsigned int *>(p);
}

cudaError_t smem_optin(const void *func, int smem, bool force)
{
    if (smem <= 48 * 1024) return cudaSuccess;   // below the default limit no opt-in is needed
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_optin_mu);
    int slot = -1;
    for (int i = 0; i < g_n_optin; ++i)
        if (g_optin[i].func == func && g_optin[i].dev == dev) slot = i;
    if (slot >= 0 && g_optin[slot].smem >= smem && !force) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (slot < 0 && g_n_optin < 256) slot = g_n_optin++;
    if (slot >= 0) g_optin[slot] = OptIn{func, dev, smem};
    return cudaSuccess;
}

cudaError_t launch_wait_selftest(uint64_t timeout_ns, int *result, cudaStream_t stream)
{
    unsigned int *status = status_word();
    if (!status) return cudaErrorInvalidSymbol;
    bounded_wait_selftest<<<1, 32, 0, stream>>>(timeout_ns, result, status);
    return cudaGetLastError();
}

cudaError_t read_and_clear_status(unsigned int *host_status, cudaStream_t stream)
{
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(host_status, g_status, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_status, &zero, sizeof(unsigned int));
}

}  // namespace mxq
