// peer.cu -- other ranks' device blocks mapped into this process (CUDA IPC).
//
// "上下文并行与 Ring Attention" (hs-black.github.io), section Ring Attention: at
// step r rank i attends its Q to the K/V block that rank (i - r) mod N started
// with.  Between the processes of one node nobody needs to send: every rank maps
// the others' blocks into its own address space once; at step r it pulls rank
// (i - r) mod N's block across the link (the forward copies it one step ahead
// into a local buffer with the copy engines, so it crosses once however many CTAs
// read it), or works on it where it lies (the backward's key-tile CTAs read each
// K/V tile once and add their dK, dV shares into the owner's accumulator with
// plain loads and stores).  No load anywhere uses cluster multicast.
//
// cp_peer_export describes a block (the IPC handle of the allocation holding it and
// the block's offset in that allocation); the handle bytes go to the other ranks
// by any host channel; cp_peer_import maps the allocation on the current device
// (lazily enabling peer access when it lives on another GPU) and returns the
// block's address there; cp_peer_close drops the mapping.  Mappings are counted
// per (device, allocation), so blocks that share an allocation map it once.
// cp_peer_copy pulls a mapped block into this GPU's memory with the copy engines,
// for readers that would otherwise cross the link many times (every query-tile CTA
// of the forward reads every K/V tile of the block).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "../../include/cpattn.h"
#include "kernels.h"

namespace {

static_assert(sizeof(cudaIpcMemHandle_t) == sizeof(((cp_peer_handle *)nullptr)->ipc),
              "cp_peer_handle.ipc must hold a cudaIpcMemHandle_t");

typedef CUresult (*AddressRangeFn)(CUdeviceptr *, size_t *, CUdeviceptr);

AddressRangeFn address_range_fn()
{
    static AddressRangeFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &ptr, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<AddressRangeFn>(ptr);
    }
    return fn;
}

struct Mapping {
    void *base;
    int refs;
};
using Key = std::pair<int, std::string>;  // (device, handle bytes)
std::mutex g_peer_mu;
std::map<Key, Mapping> g_peer_maps;

cp_status current_key(const cp_peer_handle *h, Key *key)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cpattn::report_error(CP_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    *key = Key(dev, std::string(reinterpret_cast<const char *>(h->ipc), sizeof h->ipc));
    return CP_OK;
}

}  // namespace

extern "C" cp_status cp_peer_export(const void *ptr, cp_peer_handle *out)
{
    if (!ptr || !out) return cpattn::report_error(CP_ERR_INVALID_ARG, "ptr or out is NULL");
    AddressRangeFn range = address_range_fn();
    if (!range) return cpattn::report_error(CP_ERR_CUDA, "cuMemGetAddressRange is not available");
    CUdeviceptr base = 0;
    size_t size = 0;
    if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS)
        return cpattn::report_error(CP_ERR_INVALID_ARG, "%p is not device memory allocated in this process", ptr);
    cudaIpcMemHandle_t h;
    cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base));
    if (e != cudaSuccess)
        return cpattn::report_error(CP_ERR_CUDA, "cudaIpcGetMemHandle (memory from cudaMalloc only): %s",
                                    cudaGetErrorString(e));
    std::memcpy(out->ipc, &h, sizeof h);
    out->offset = (uint64_t)(reinterpret_cast<CUdeviceptr>(ptr) - base);
    out->bytes = (uint64_t)size - out->offset;
    return CP_OK;
}

extern "C" cp_status cp_peer_import(const cp_peer_handle *h, void **ptr)
{
    if (!h || !ptr) return cpattn::report_error(CP_ERR_INVALID_ARG, "h or ptr is NULL");
    Key key;
    cp_status s = current_key(h, &key);
    if (s != CP_OK) return s;
    std::lock_guard<std::mutex> lk(g_peer_mu);
    auto it = g_peer_maps.find(key);
    if (it == g_peer_maps.end()) {
        cudaIpcMemHandle_t ipc;
        std::memcpy(&ipc, h->ipc, sizeof ipc);
        void *base = nullptr;
        cudaError_t e = cudaIpcOpenMemHandle(&base, ipc, cudaIpcMemLazyEnablePeerAccess);
        if (e != cudaSuccess)
            return cpattn::report_error(CP_ERR_CUDA, "cudaIpcOpenMemHandle (a handle of another process): %s",
                                        cudaGetErrorString(e));
        it = g_peer_maps.emplace(key, Mapping{base, 0}).first;
    }
    it->second.refs += 1;
    *ptr = static_cast<char *>(it->second.base) + h->offset;
    return CP_OK;
}

extern "C" cp_status cp_peer_close(const cp_peer_handle *h)
{
    if (!h) return cpattn::report_error(CP_ERR_INVALID_ARG, "h is NULL");
    Key key;
    cp_status s = current_key(h, &key);
    if (s != CP_OK) return s;
    std::lock_guard<std::mutex> lk(g_peer_mu);
    auto it = g_peer_maps.find(key);
    if (it == g_peer_maps.end())
        return cpattn::report_error(CP_ERR_INVALID_ARG, "this handle is not mapped on the current device");
    if (--it->second.refs > 0) return CP_OK;
    cudaError_t e = cudaIpcCloseMemHandle(it->second.base);
    g_peer_maps.erase(it);
    if (e != cudaSuccess)
        return cpattn::report_error(CP_ERR_CUDA, "cudaIpcCloseMemHandle: %s", cudaGetErrorString(e));
    return CP_OK;
}

extern "C" cp_status cp_peer_copy(void *dst, const void *src, size_t bytes, void *stream)
{
    if (bytes == 0) return CP_OK;
    if (!dst || !src) return cpattn::report_error(CP_ERR_INVALID_ARG, "dst or src is NULL");
    cudaError_t e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cpattn::report_error(CP_ERR_CUDA, "cudaMemcpyAsync: %s", cudaGetErrorString(e));
    return CP_OK;
}
