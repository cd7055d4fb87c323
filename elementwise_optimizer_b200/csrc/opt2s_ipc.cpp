// opt2s_ipc.cpp -- peer mappings for the sharded step between processes.
//
// opt2s_shard_step reads every rank's gradient buffer and writes every rank's
// param buffer, so each rank needs the other ranks' buffers mapped into its
// own address space.  With one process per GPU that is CUDA IPC: a rank
// exports a handle to the allocation that holds its buffer, the handles and
// the buffers' offsets inside their allocations travel over the process
// group, and each rank opens the others' handles.  Across GPUs of one node
// the mapping enables peer access on first use, so the kernel's plain loads
// and stores cross NVLink; on one GPU the mapping is plain device memory.
// Nothing here uses TMA or multicast.

#include <cstdint>
#include <cstring>

#include <cuda.h>
#include <cuda_runtime.h>

#include "opt2s.h"
#include "opt2s_internal.h"

#define OPT2S_API extern "C" __attribute__((visibility("default")))

static_assert(sizeof(opt2s_ipc_handle) == sizeof(cudaIpcMemHandle_t), "IPC handle size");

namespace {

// cuMemGetAddressRange (CUDA 12 ABI) through the runtime's driver entry
// point, so the library needs no link-time dependency on the driver library.
using AddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

cudaError_t allocation_base(const void* ptr, void** base)
{
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    cudaError_t e = cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &fn, 12000,
                                                     cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
    CUdeviceptr b = 0;
    size_t size = 0;
    if (reinterpret_cast<AddressRangeFn>(fn)(&b, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    *base = reinterpret_cast<void*>(b);
    return cudaSuccess;
}

}  // namespace

OPT2S_API int opt2s_ipc_export(const void* ptr, opt2s_ipc_handle* handle, int64_t* offset)
{
    if (!ptr || !handle || !offset) return OPT2S_ERR_INVALID_ARG;
    void* base = nullptr;
    cudaError_t e = allocation_base(ptr, &base);
    if (e != cudaSuccess) return opt2s::record_cuda_error(e);
    cudaIpcMemHandle_t h;
    e = cudaIpcGetMemHandle(&h, base);
    if (e != cudaSuccess) return opt2s::record_cuda_error(e);
    std::memcpy(handle, &h, sizeof(h));
    *offset = static_cast<const char*>(ptr) - static_cast<const char*>(base);
    return OPT2S_OK;
}

OPT2S_API int opt2s_ipc_open(const opt2s_ipc_handle* handle, int64_t offset, void** base, void** ptr)
{
    if (!handle || !base || !ptr || offset < 0) return OPT2S_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof(h));
    void* b = nullptr;
    const cudaError_t e = cudaIpcOpenMemHandle(&b, h, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return opt2s::record_cuda_error(e);
    *base = b;
    *ptr = static_cast<char*>(b) + offset;
    return OPT2S_OK;
}

OPT2S_API int opt2s_ipc_close(void* base)
{
    if (!base) return OPT2S_ERR_INVALID_ARG;
    const cudaError_t e = cudaIpcCloseMemHandle(base);
    if (e != cudaSuccess) return opt2s::record_cuda_error(e);
    return OPT2S_OK;
}
