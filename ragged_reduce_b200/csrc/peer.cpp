// CUDA IPC for one rank per GPU (include/h3rr.h, h3_ipc_*): export a device
// buffer as (allocation handle, offset), map a peer's buffer, unmap it.
//
// cudaIpcGetMemHandle wants the base of a cudaMalloc allocation, while a
// framework's caching allocator hands out buffers inside larger allocations;
// the base is found with the driver's cuMemGetAddressRange, fetched through
// the runtime's driver entry-point query (no link against libcuda).
//
// A process may map a given allocation's handle only once per device, yet
// two exported buffers often share one allocation.  Mappings are therefore
// counted per (device, handle): the first open maps, later opens reuse the
// mapping, and the last close unmaps it.
#include <array>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

#include <cuda.h>

#include "context.h"
#include "h3rr_internal.h"

using namespace h3rr;

static_assert(sizeof(cudaIpcMemHandle_t) == H3_IPC_HANDLE_BYTES, "IPC handle size");

namespace {

using AddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

// cuMemGetAddressRange with the CUDA 12 signature, or null if unavailable.
AddressRangeFn address_range_fn()
{
    static std::once_flag once;
    static AddressRangeFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<AddressRangeFn>(p);
    });
    return fn;
}

struct Mapping {
    void* base = nullptr;
    int64_t refs = 0;
};

// Mappings belong to a context: after cudaDeviceReset the device's next
// context holds none of them, so the key carries the context's id (0 when
// the driver cannot say).
using MappingKey =
    std::tuple<int, unsigned long long, std::array<unsigned char, H3_IPC_HANDLE_BYTES>>;

std::mutex g_map_mutex;
std::map<MappingKey, Mapping> g_mappings;

MappingKey key_of(int device, const h3_ipc_handle* handle)
{
    unsigned long long ctx = 0;
    if (!current_context_id(&ctx))
        ctx = 0;
    std::array<unsigned char, H3_IPC_HANDLE_BYTES> bytes;
    std::memcpy(bytes.data(), handle->handle, H3_IPC_HANDLE_BYTES);
    return MappingKey(device, ctx, bytes);
}

}  // namespace

extern "C" {

h3_status h3_ipc_export(const void* ptr, h3_ipc_handle* out)
{
    if (!ptr || !out)
        return H3_ERR_INVALID_ARG;
    std::memset(out, 0, sizeof(*out));
    AddressRangeFn range = address_range_fn();
    if (!range)
        return record_cuda_failure(cudaErrorNotSupported);
    CUdeviceptr base = 0;
    size_t size = 0;
    if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS)
        return record_cuda_failure(cudaErrorInvalidValue);
    cudaIpcMemHandle_t h;
    const cudaError_t err = cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base));
    if (err != cudaSuccess)
        return record_cuda_failure(err);
    std::memcpy(out->handle, &h, sizeof(h));
    out->offset = int64_t(reinterpret_cast<uintptr_t>(ptr) - uintptr_t(base));
    out->alloc_bytes = int64_t(size);
    return H3_OK;
}

h3_status h3_ipc_open(const h3_ipc_handle* handle, void** ptr)
{
    if (!handle || !ptr)
        return H3_ERR_INVALID_ARG;
    *ptr = nullptr;
    if (handle->offset < 0 || handle->offset >= handle->alloc_bytes)
        return H3_ERR_INVALID_ARG;
    int device = 0;
    cudaError_t err = cudaGetDevice(&device);
    if (err != cudaSuccess)
        return record_cuda_failure(err);
    std::lock_guard<std::mutex> lock(g_map_mutex);
    Mapping& m = g_mappings[key_of(device, handle)];
    if (m.refs == 0) {
        cudaIpcMemHandle_t h;
        std::memcpy(&h, handle->handle, sizeof(h));
        err = cudaIpcOpenMemHandle(&m.base, h, cudaIpcMemLazyEnablePeerAccess);
        if (err != cudaSuccess) {
            g_mappings.erase(key_of(device, handle));
            return record_cuda_failure(err);
        }
    }
    ++m.refs;
    *ptr = static_cast<char*>(m.base) + handle->offset;
    return H3_OK;
}

h3_status h3_ipc_close(void* ptr, const h3_ipc_handle* handle)
{
    if (!ptr || !handle || handle->offset < 0)
        return H3_ERR_INVALID_ARG;
    int device = 0;
    cudaError_t err = cudaGetDevice(&device);
    if (err != cudaSuccess)
        return record_cuda_failure(err);
    std::lock_guard<std::mutex> lock(g_map_mutex);
    auto it = g_mappings.find(key_of(device, handle));
    if (it == g_mappings.end() || it->second.base != static_cast<char*>(ptr) - handle->offset)
        return H3_ERR_INVALID_ARG;  // not a mapping this process holds on this device
    if (--it->second.refs > 0)
        return H3_OK;
    err = cudaIpcCloseMemHandle(it->second.base);
    g_mappings.erase(it);
    if (err != cudaSuccess)
        return record_cuda_failure(err);
    return H3_OK;
}

}  // extern "C"
