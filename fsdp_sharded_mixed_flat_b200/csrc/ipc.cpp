// ipc.cpp -- another process's device memory, mapped for this library's kernels
// (host only).
//
// The D-GPU form of the step ("7.10 — Fully-sharded data parallel (FSDP /
// ZeRO-3)", §4 and §5.1) lets the fused kernel on rank r read slice P_r of
// every rank's gradient, and the gather kernel read every rank's shard,
// straight from the other GPUs' memory.  Each rank exports the allocation that
// holds its buffer (a CUDA IPC handle plus the buffer's offset in it); every
// other rank maps that allocation into the address space of ITS OWN current
// device with lazy peer access, so that its kernels, launched on that device,
// reach the memory with plain loads and stores over NVLink.  (Mapping it under
// the owning GPU's device instead would leave the kernels' device without a
// peer mapping.)
//
// A second open of a handle that a process has mapped already is not something
// the CUDA runtime promises to allow, while several buffers of one rank often
// share an allocation; imports are therefore counted per handle and share one
// mapping, which the last close releases.
#include <cuda.h>  // CUresult and CUdeviceptr for the driver entry point (no link to libcuda)
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <string>

#include "zero3.h"

static_assert(sizeof(cudaIpcMemHandle_t) == Z3_IPC_HANDLE_BYTES, "IPC handle size");

namespace {

using GetAddressRange = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

// cuMemGetAddressRange through the runtime's driver entry point, so the library
// needs no link against the driver library.
GetAddressRange address_range() {
    static const GetAddressRange fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return GetAddressRange(nullptr);
        }
        return reinterpret_cast<GetAddressRange>(p);
    }();
    return fn;
}

struct Mapping {
    void* base;
    int64_t refs;
};

std::mutex g_mu;
std::map<std::string, Mapping> g_by_handle;  // handle bytes -> mapping
std::map<void*, std::string> g_by_base;      // mapping -> handle bytes

}  // namespace

extern "C" Z3_API int zero3_ipc_export(const void* ptr, void* handle_out, int64_t* offset_out, int64_t* size_out) {
    if (ptr == nullptr || handle_out == nullptr || offset_out == nullptr || size_out == nullptr) return Z3_EINVAL;
    const GetAddressRange range = address_range();
    if (range == nullptr) return Z3_ECUDA;
    CUdeviceptr base = 0;
    size_t size = 0;
    if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return Z3_EINVAL;
    const uintptr_t p = reinterpret_cast<uintptr_t>(ptr);
    if (p < uintptr_t(base) || p - uintptr_t(base) >= size) return Z3_EINVAL;  // not inside the range reported
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) {
        cudaGetLastError();
        return Z3_ECUDA;
    }
    std::memcpy(handle_out, &h, sizeof h);
    *offset_out = int64_t(reinterpret_cast<uintptr_t>(ptr) - uintptr_t(base));
    *size_out = int64_t(size);
    return Z3_OK;
}

extern "C" Z3_API int zero3_ipc_import(const void* handle, int64_t offset, void** ptr_out, void** base_out) {
    if (handle == nullptr || offset < 0 || ptr_out == nullptr || base_out == nullptr) return Z3_EINVAL;
    std::string key;
    try {
        key.assign(static_cast<const char*>(handle), Z3_IPC_HANDLE_BYTES);
    } catch (...) {
        return Z3_ENOMEM;
    }
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_by_handle.find(key);
    if (it == g_by_handle.end()) {
        cudaIpcMemHandle_t h;
        std::memcpy(&h, handle, sizeof h);
        void* base = nullptr;
        if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
            cudaGetLastError();
            return Z3_ECUDA;
        }
        try {  // record the mapping; if the bookkeeping cannot allocate, unmap again
            it = g_by_handle.emplace(key, Mapping{base, 0}).first;
            try {
                g_by_base.emplace(base, key);
            } catch (...) {
                g_by_handle.erase(it);
                throw;
            }
        } catch (...) {
            cudaIpcCloseMemHandle(base);
            cudaGetLastError();
            return Z3_ENOMEM;
        }
    }
    ++it->second.refs;
    *base_out = it->second.base;
    *ptr_out = static_cast<char*>(it->second.base) + offset;
    return Z3_OK;
}

extern "C" Z3_API int zero3_ipc_close(void* base) {
    if (base == nullptr) return Z3_EINVAL;
    std::lock_guard<std::mutex> lk(g_mu);
    auto b = g_by_base.find(base);
    if (b == g_by_base.end()) return Z3_EINVAL;
    auto it = g_by_handle.find(b->second);
    if (--it->second.refs > 0) return Z3_OK;
    g_by_handle.erase(it);
    g_by_base.erase(b);
    if (cudaIpcCloseMemHandle(base) != cudaSuccess) {
        cudaGetLastError();
        return Z3_ECUDA;
    }
    return Z3_OK;
}
