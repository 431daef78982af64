// ipc.cpp - mapping another process's device buffers into this one, so that
// the pointer tables of the collectives can name peers' memory.
//
// In a data-parallel job each rank owns its gradients and its shard; TIDE-RS
// reads chunk r of every rank's gradients and TIDE-AG places every rank's
// shard (weekinpapers.com, Abstract; kongchang.com, "TIDE's Design Approach").
// With one process per GPU, the peers' buffers reach this process through
// CUDA IPC: the owner exports the allocation that holds a buffer, every other
// rank maps it on ITS OWN device, where the mapping enables peer access to the
// owner's GPU (over NVLink on B200 systems), and the kernels then load from it
// like from local memory.  Nothing here waits on another process; ordering
// between ranks is the caller's (host barriers).
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>

#include "tide_internal.h"

namespace {

// cuMemGetAddressRange, from the driver through the runtime (the library links
// the runtime statically and does not link libcuda itself).
using GetRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

GetRangeFn get_range_fn() {
    static GetRangeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<GetRangeFn>(p);
        (void)cudaGetLastError();
    });
    return fn;
}

// Runs f with `device` current and restores the caller's device.
template <class F>
tide_status_t on_device(int device, F f) {
    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) {
        (void)cudaGetLastError();
        return TIDE_ERR_CUDA;
    }
    if (device != prev && cudaSetDevice(device) != cudaSuccess) {
        (void)cudaGetLastError();
        return TIDE_ERR_DEVICE;
    }
    tide_status_t st = f();
    if (device != prev) cudaSetDevice(prev);
    if (st != TIDE_OK) (void)cudaGetLastError();
    return st;
}

}  // namespace

static_assert(sizeof(cudaIpcMemHandle_t) == TIDE_IPC_HANDLE_BYTES, "IPC handle size");

extern "C" tide_status_t tide_ipc_export(const void* dev_ptr, void* handle, int64_t* offset,
                                         int32_t* device) {
    if (dev_ptr == nullptr || handle == nullptr || offset == nullptr) return TIDE_ERR_INVALID_ARG;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, dev_ptr) != cudaSuccess) {
        (void)cudaGetLastError();
        return TIDE_ERR_INVALID_ARG;
    }
    if (attr.type != cudaMemoryTypeDevice) return TIDE_ERR_INVALID_ARG;
    GetRangeFn range = get_range_fn();
    if (range == nullptr) return TIDE_ERR_CUDA;
    return on_device(attr.device, [&]() -> tide_status_t {
        CUdeviceptr base = 0;
        size_t size = 0;
        if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
            return TIDE_ERR_INVALID_ARG;
        cudaIpcMemHandle_t h;
        if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) return TIDE_ERR_CUDA;
        std::memcpy(handle, &h, sizeof(h));
        *offset = static_cast<int64_t>(reinterpret_cast<uintptr_t>(dev_ptr) - static_cast<uintptr_t>(base));
        if (device != nullptr) *device = attr.device;
        return TIDE_OK;
    });
}

extern "C" tide_status_t tide_ipc_open(const void* handle, int32_t device, void** base) {
    if (handle == nullptr || base == nullptr || device < 0) return TIDE_ERR_INVALID_ARG;
    int n_dev = 0;
    if (cudaGetDeviceCount(&n_dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return TIDE_ERR_CUDA;
    }
    if (device >= n_dev) return TIDE_ERR_DEVICE;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof(h));
    return on_device(device, [&]() -> tide_status_t {
        void* p = nullptr;
        if (cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return TIDE_ERR_CUDA;
        *base = p;
        return TIDE_OK;
    });
}

extern "C" tide_status_t tide_ipc_close(void* base, int32_t device) {
    if (base == nullptr || device < 0) return TIDE_ERR_INVALID_ARG;
    return on_device(device, [&]() -> tide_status_t {
        return cudaIpcCloseMemHandle(base) == cudaSuccess ? TIDE_OK : TIDE_ERR_CUDA;
    });
}

extern "C" tide_status_t tide_peer_access(int32_t device, int32_t peer, int32_t* can_access) {
    if (can_access == nullptr || device < 0 || peer < 0) return TIDE_ERR_INVALID_ARG;
    int v = 0;
    if (device == peer) {
        *can_access = 1;
        return TIDE_OK;
    }
    if (cudaDeviceCanAccessPeer(&v, device, peer) != cudaSuccess) {
        (void)cudaGetLastError();
        return TIDE_ERR_DEVICE;
    }
    *can_access = v;
    return TIDE_OK;
}
