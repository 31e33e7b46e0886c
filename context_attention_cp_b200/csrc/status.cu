// status.cu -- the per-device status word written by kernels whose bounded waits
// expire (word 0: error bits, word 1: tag of the first wait that gave up).
#include <cuda_runtime.h>

#include "kernels.h"

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

}  // namespace cpattn
