// status.cu -- the per-device status word written by kernels whose bounded waits
// expire (word 0: error bits, word 1: tag of the first wait that gave up).
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx.cuh"

namespace cpattn {

__device__ int g_status_word[2];

cudaError_t status_word(int **ptr)
{
    // the symbol's device address differs per device: look it up for the current one
    constexpr int kMaxDevices = 64;
    static int *cached[kMaxDevices] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices && cached[dev]) {
        *ptr = cached[dev];
        return cudaSuccess;
    }
    void *addr = nullptr;
    e = cudaGetSymbolAddress(&addr, g_status_word);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices) cached[dev] = static_cast<int *>(addr);
    *ptr = static_cast<int *>(addr);
    return cudaSuccess;
}

cudaError_t set_smem_per_device(const void *fn, int bytes, unsigned long long *done)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
    if (bit && (__atomic_load_n(done, __ATOMIC_ACQUIRE) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) __atomic_fetch_or(done, bit, __ATOMIC_RELEASE);
    return e;
}

namespace {

// One warp waits on an mbarrier that nothing ever arrives at; the bounded wait runs
// out after limit_ns and reports through the status word, the way every wait in the
// attention kernels does.  The kernel then returns normally.
__global__ void wait_timeout_kernel(int *status, uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t mbar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&mbar), 1);
        abort_flag = 0;
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        WaitCtx w{&abort_flag, status, 99};
        mbar_wait_limit(smem_u32(&mbar), 0, w, limit_ns);
    }
    __syncthreads();
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(uint64_t limit_ns, cudaStream_t stream)
{
    int *word = nullptr;
    cudaError_t e = status_word(&word);
    if (e != cudaSuccess) return e;
    wait_timeout_kernel<<<1, 32, 0, stream>>>(word, limit_ns);
    return cudaGetLastError();
}

// Streaming multiprocessors of the current device (looked up once per device).
int sm_count()
{
    static int counts[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 0 || dev >= 64) return 148;
    if (!counts[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        counts[dev] = n;
    }
    return counts[dev];
}

}  // namespace cpattn
