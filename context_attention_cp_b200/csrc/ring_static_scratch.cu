// ring_static_scratch.cu -- the stepwise ring for callers that cannot allocate
// device memory.
//
// Some callers of this library have no way to call cudaMalloc: a plug-in hosted by
// an engine that owns every byte of device memory and only hands the plug-in its
// input and output pointers, or a latency-critical caller that must not pay the
// implicit device synchronisation an allocation can bring.  The stepwise ring
// (cp_ring_attn_fwd with CP_RING_STEPWISE) needs a workspace for its running fp32
// output and the per-step partials; this entry point takes that workspace from a
// static array that lives in the library's device image instead of from the caller.
//
// Costs and rules:
//   - every GPU on which this code is loaded holds CP_STATIC_SCRATCH_BYTES of device
//     memory for the array until the process exits;
//   - problems whose workspace exceeds CP_STATIC_SCRATCH_BYTES are rejected with
//     CP_ERR_UNSUPPORTED before anything is launched;
//   - all calls on one device share the array: two calls whose work overlaps on the
//     GPU (different streams, or different host threads) race on it;
//   - the array keeps the previous call's contents; the stepwise ring writes every
//     byte it later reads (step 0 stores the running result, every later step stores
//     its whole partial before the merge reads it), so nothing has to be cleared;
//   - the first call on a device looks up the array's device address (a host-side
//     reference to the array is not a device address); make that first call before
//     any stream capture on that device;
//   - the looked-up address is kept for the life of the process; a device reset
//     (cudaDeviceReset) unloads the array, after which this entry point must not be
//     called on that device.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/cpattn.h"
#include "kernels.h"

namespace {

static __device__ __align__(256) unsigned char g_ring_scratch[CP_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_ring_scratch on the current device, looked up once per device.
cp_status scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cpattn::report_error(CP_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return cpattn::report_error(CP_ERR_UNSUPPORTED, "device %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_ring_scratch);
        if (e != cudaSuccess || !ptr)
            return cpattn::report_error(CP_ERR_CUDA, "cudaGetSymbolAddress of the static scratch: %s",
                                        cudaGetErrorString(e));
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
    return CP_OK;
}

}  // namespace

extern "C" cp_status cp_ring_attn_fwd_static_scratch(int32_t layout, int32_t N, int32_t causal, const cp_tensor *q,
                                                     const cp_tensor *k, const cp_tensor *v, float softmax_scale,
                                                     cp_tensor *o, cp_tensor *lse, void *stream)
{
    if (!q) return cpattn::report_error(CP_ERR_INVALID_ARG, "q is NULL");
    const size_t need = cp_ring_workspace_bytes(layout, N, CP_RING_STEPWISE, q->dtype, q->shape[0], q->shape[1],
                                                q->shape[2], q->shape[3]);
    if (need > CP_STATIC_SCRATCH_BYTES)
        return cpattn::report_error(CP_ERR_UNSUPPORTED,
                                    "this problem needs %zu bytes of scratch; the static scratch holds %zu bytes",
                                    need, (size_t)CP_STATIC_SCRATCH_BYTES);
    void *scratch = nullptr;
    cp_status s = scratch_address(&scratch);
    if (s != CP_OK) return s;
    return cp_ring_attn_fwd(layout, N, causal, q, k, v, softmax_scale, o, lse, CP_RING_STEPWISE, scratch,
                            CP_STATIC_SCRATCH_BYTES, stream);
}
