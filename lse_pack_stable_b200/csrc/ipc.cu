// Mapping a peer rank's buffers into this process, for the pull-based exchange
// (cp_pull_combine): CUDA IPC memory handles, exported by the owner and opened
// by every reader in the reader's current-device context with lazy peer
// access, so that the reader's kernels address the owner's HBM over NVLink.
//
// Plain device-memory IPC only: no multicast object, no fabric handle, nothing
// bound to the NVLink switch. Host code only; no kernels here.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "cplse.h"

// defined in api.cu: records the message that cp_last_error() returns
cp_status cplse_set_error(cp_status st, const char* msg);

namespace {

cp_status ipc_fail(cp_status st, const char* fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    return cplse_set_error(st, buf);
}

typedef int (*AddressRangeFn)(unsigned long long* base, size_t* size, unsigned long long p);

// cuMemGetAddressRange through the runtime's driver entry point: the base and
// size of the allocation that contains p (an IPC handle names a whole
// allocation, so the exported offset is p - base).
cudaError_t allocation_range(const void* p, uintptr_t& base, size_t& size)
{
    // looked up once per process (thread-safe static initialisation)
    static const AddressRangeFn fn = []() -> AddressRangeFn {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &f, 12000, cudaEnableDefault,
                                             &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        return reinterpret_cast<AddressRangeFn>(f);
    }();
    if (fn == nullptr) return cudaErrorSymbolNotFound;
    unsigned long long b = 0;
    size_t s = 0;
    if (fn(&b, &s, (unsigned long long)(uintptr_t)p) != 0) return cudaErrorInvalidValue;
    base = (uintptr_t)b;
    size = s;
    return cudaSuccess;
}

}  // namespace

extern "C" {

cp_status cp_ipc_export(const void* p, cp_ipc_handle* h)
{
    if (p == nullptr) return ipc_fail(CP_ERR_ARG, "p is NULL");
    if (h == nullptr) return ipc_fail(CP_ERR_ARG, "h is NULL");
    cudaPointerAttributes at;
    cudaError_t e = cudaPointerGetAttributes(&at, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return ipc_fail(CP_ERR_ARG, "p: cudaPointerGetAttributes failed (%s)", cudaGetErrorString(e));
    }
    if (at.type != cudaMemoryTypeDevice)
        return ipc_fail(CP_ERR_ARG, "p is not device memory");
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || at.device != dev) {
        cudaGetLastError();
        return ipc_fail(CP_ERR_ARG, "p lives on device %d, not on the current device", at.device);
    }
    uintptr_t base = 0;
    size_t size = 0;
    e = allocation_range(p, base, size);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return ipc_fail(CP_ERR_CUDA, "allocation range of p: %s", cudaGetErrorString(e));
    }
    cudaIpcMemHandle_t mh;
    e = cudaIpcGetMemHandle(&mh, reinterpret_cast<void*>(base));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return ipc_fail(CP_ERR_CUDA, "cudaIpcGetMemHandle: %s (the memory must come from cudaMalloc)",
                        cudaGetErrorString(e));
    }
    static_assert(sizeof(mh) == sizeof(h->handle), "IPC handle size");
    memcpy(h->handle, &mh, sizeof(mh));
    h->offset = (int64_t)((uintptr_t)p - base);
    h->alloc_bytes = (int64_t)size;
    h->device = dev;
    h->reserved = 0;
    return cplse_set_error(CP_OK, "");
}

cp_status cp_ipc_import(const cp_ipc_handle* h, void** base, void** p)
{
    if (h == nullptr || base == nullptr || p == nullptr)
        return ipc_fail(CP_ERR_ARG, "h, base and p must not be NULL");
    if (h->offset < 0 || h->offset >= h->alloc_bytes)
        return ipc_fail(CP_ERR_ARG, "offset %lld is outside the %lld-byte allocation",
                        (long long)h->offset, (long long)h->alloc_bytes);
    cudaIpcMemHandle_t mh;
    memcpy(&mh, h->handle, sizeof(mh));
    void* b = nullptr;
    const cudaError_t e = cudaIpcOpenMemHandle(&b, mh, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return ipc_fail(CP_ERR_CUDA, "cudaIpcOpenMemHandle: %s", cudaGetErrorString(e));
    }
    *base = b;
    *p = static_cast<char*>(b) + h->offset;
    return cplse_set_error(CP_OK, "");
}

cp_status cp_ipc_close(void* base)
{
    if (base == nullptr) return ipc_fail(CP_ERR_ARG, "base is NULL");
    const cudaError_t e = cudaIpcCloseMemHandle(base);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return ipc_fail(CP_ERR_CUDA, "cudaIpcCloseMemHandle: %s", cudaGetErrorString(e));
    }
    return cplse_set_error(CP_OK, "");
}

}  // extern "C"
