// Peer mappings between processes for the expert-parallel calls: CUDA IPC handles of
// caller-allocated buffers, opened in the other ranks' processes as plain peer mappings
// (no multicast object is created, so no rank's memory is ever bound to one).
//
// A buffer inside a larger allocation (a caching allocator's segment) is exported as the
// handle of the enclosing allocation plus the buffer's byte offset in it; the importing
// process maps the whole allocation and adds the offset.
#include <cuda.h>
#include <cuda_runtime.h>
#include <string.h>

#include <map>
#include <mutex>
#include <string>

#include "moedisp.h"

namespace {

typedef CUresult (*GetAddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);

// cuMemGetAddressRange through the runtime's driver entry point (no link against the
// driver library).
GetAddressRangeFn address_range_fn() {
    static std::once_flag once;
    static GetAddressRangeFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<GetAddressRangeFn>(p);
        (void)cudaGetLastError();
    });
    return fn;
}

// One mapping per exported allocation, shared by every buffer imported from it (an
// allocation is opened once per process and closed with its last buffer).
struct Mapping {
    uintptr_t base;
    int refs;
};
std::mutex g_mu;
std::map<std::string, Mapping> g_maps;             // handle bytes -> mapping
std::map<uintptr_t, std::string> g_opened;         // returned pointer -> handle bytes

}  // namespace

extern "C" {

int moedisp_ipc_export(const void* dev_ptr, void* handle, int64_t* offset) {
    if (!dev_ptr || !handle || !offset) return MOEDISP_ERR_NULLPTR;
    GetAddressRangeFn range = address_range_fn();
    if (!range) return MOEDISP_ERR_CUDA;
    CUdeviceptr base = 0;
    size_t size = 0;
    if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
        return MOEDISP_ERR_INVALID;                 // not device memory of this process
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) {
        (void)cudaGetLastError();
        return MOEDISP_ERR_CUDA;
    }
    static_assert(sizeof(h) == MOEDISP_IPC_HANDLE_BYTES, "IPC handle size");
    memcpy(handle, &h, sizeof(h));
    *offset = (int64_t)(reinterpret_cast<uintptr_t>(dev_ptr) - (uintptr_t)base);
    return MOEDISP_OK;
}

int moedisp_ipc_import(const void* handle, int64_t offset, void** dev_ptr) {
    if (!handle || !dev_ptr) return MOEDISP_ERR_NULLPTR;
    if (offset < 0) return MOEDISP_ERR_INVALID;
    const std::string key(static_cast<const char*>(handle), MOEDISP_IPC_HANDLE_BYTES);
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = g_maps.find(key);
    if (it == g_maps.end()) {
        cudaIpcMemHandle_t h;
        memcpy(&h, handle, sizeof(h));
        void* base = nullptr;
        if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
            (void)cudaGetLastError();
            return MOEDISP_ERR_CUDA;
        }
        it = g_maps.emplace(key, Mapping{reinterpret_cast<uintptr_t>(base), 0}).first;
    }
    const uintptr_t p = it->second.base + (uintptr_t)offset;
    if (g_opened.count(p)) return MOEDISP_ERR_INVALID;        // already imported
    it->second.refs += 1;
    g_opened[p] = key;
    *dev_ptr = reinterpret_cast<void*>(p);
    return MOEDISP_OK;
}

int moedisp_ipc_close(void* dev_ptr) {
    if (!dev_ptr) return MOEDISP_ERR_NULLPTR;
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = g_opened.find(reinterpret_cast<uintptr_t>(dev_ptr));
    if (it == g_opened.end()) return MOEDISP_ERR_INVALID;
    auto m = g_maps.find(it->second);
    g_opened.erase(it);
    if (--m->second.refs > 0) return MOEDISP_OK;
    const uintptr_t base = m->second.base;
    g_maps.erase(m);
    if (cudaIpcCloseMemHandle(reinterpret_cast<void*>(base)) != cudaSuccess) {
        (void)cudaGetLastError();
        return MOEDISP_ERR_CUDA;
    }
    return MOEDISP_OK;
}

}  // extern "C"
