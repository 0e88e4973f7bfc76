// peer.cu -- device buffers shared between processes, and device-to-device copies.
//
// MoE-latency article, section "跨 GPU 时,激活要出门": with the experts spread over GPUs,
// a token's activation row travels to the GPU that holds its expert and the expert's
// output travels back, every layer.  The expert-parallel layer can move those rows
// itself, by copies into buffers of the other ranks' GPUs, instead of through a
// collective library.  These calls give it the pieces: a buffer exported by one
// process and mapped by another (CUDA IPC), and one asynchronous copy per contiguous
// range of rows.  Nothing here waits on another process; ordering between the ranks
// is the caller's (a host-side barrier after each rank's copies have completed).
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstring>

#include "../../include/moe.h"
#include "internal.h"

namespace {

using GetAddressRange = int (*)(uintptr_t *base, size_t *size, uintptr_t ptr);

// The allocation that contains ptr (driver call, looked up once): IPC handles name a
// whole allocation, so a buffer inside one travels as the handle plus its offset.
bool allocation_base(const void *ptr, uintptr_t *base)
{
    static GetAddressRange fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &p, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<GetAddressRange>(p);
    }();
    size_t size = 0;
    return fn && fn(base, &size, reinterpret_cast<uintptr_t>(ptr)) == 0;
}

}  // namespace

extern "C" {

moe_status_t moe_ipc_export(const void *ptr, void *handle, size_t *offset)
{
    if (!ptr || !handle || !offset) return MOE_ERR_INVALID_ARG;
    uintptr_t base = 0;
    if (!allocation_base(ptr, &base)) return MOE_ERR_UNSUPPORTED;
    cudaIpcMemHandle_t h;
    const cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_UNSUPPORTED;  // e.g. memory the IPC API cannot share (virtual-memory mapped)
    }
    static_assert(sizeof(h) == MOE_IPC_HANDLE_BYTES, "IPC handle size");
    std::memcpy(handle, &h, sizeof h);
    *offset = reinterpret_cast<uintptr_t>(ptr) - base;
    return MOE_OK;
}

moe_status_t moe_ipc_import(const void *handle, size_t offset, void **ptr)
{
    if (!handle || !ptr) return MOE_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof h);
    void *base = nullptr;
    const cudaError_t e = cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    *ptr = static_cast<uint8_t *>(base) + offset;
    return MOE_OK;
}

moe_status_t moe_ipc_close(void *ptr, size_t offset)
{
    if (!ptr) return MOE_ERR_INVALID_ARG;
    const cudaError_t e = cudaIpcCloseMemHandle(static_cast<uint8_t *>(ptr) - offset);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

moe_status_t moe_copy_async(void *dst, const void *src, size_t bytes, void *stream)
{
    if (bytes == 0) return MOE_OK;
    if (!dst || !src) return MOE_ERR_INVALID_ARG;
    const cudaError_t e =
        cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

}  // extern "C"
