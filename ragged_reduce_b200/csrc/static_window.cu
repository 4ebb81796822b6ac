// h3_seq_to_head_staged_noalloc: the staged sequence->head relayout with its
// window in a device array owned by the library, for callers that cannot
// allocate device memory (see include/h3rr.h).  Nothing here allocates or
// frees device memory; the array itself is reserved when the CUDA runtime
// loads this file's device module into a context (on the first call in that
// context, under lazy module loading).
#include <map>
#include <mutex>
#include <utility>

#include "context.h"
#include "h3rr_internal.h"

namespace h3rr {

// The window of every h3_seq_to_head_staged_noalloc call on a device.  Host
// code must not pass this symbol to a kernel: on the host it names a
// stand-in, not device memory.  Its device address is looked up below.
static __device__ __align__(256) unsigned char g_static_window[H3RR_STATIC_WINDOW_BYTES];

namespace {

// Device address of g_static_window in the current context.  Looked up with
// cudaGetSymbolAddress once per device and context, with that device
// current, and kept under the context's id: after cudaDeviceReset the
// device's next context has a new id and may hold the array elsewhere, so
// the lookup runs again there.  Without a context id the lookup runs on
// every call.
cudaError_t static_window_address(void** ptr)
{
    static std::mutex mu;
    static std::map<std::pair<int, unsigned long long>, void*> addresses;
    int device = 0;
    cudaError_t err = cudaGetDevice(&device);
    if (err != cudaSuccess)
        return err;
    unsigned long long ctx = 0;
    bool keyed = current_context_id(&ctx);
    if (keyed) {
        std::lock_guard<std::mutex> lock(mu);
        auto it = addresses.find({device, ctx});
        if (it != addresses.end()) {
            *ptr = it->second;
            return cudaSuccess;
        }
    }
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_static_window);
    if (err != cudaSuccess)
        return err;
    // The lookup makes the device's primary context current if nothing was.
    if (!keyed)
        keyed = current_context_id(&ctx);
    if (keyed) {
        std::lock_guard<std::mutex> lock(mu);
        addresses[{device, ctx}] = p;
    }
    *ptr = p;
    return cudaSuccess;
}

}  // namespace
}  // namespace h3rr

extern "C" h3_status h3_seq_to_head_staged_noalloc(const void* const* send, void* const* recv,
                                                   int64_t n_tokens, int32_t planes,
                                                   int32_t n_heads, int32_t head_dim,
                                                   int32_t world, int64_t window_bytes,
                                                   void* stream, h3_exec_info* info)
{
    if (info)
        *info = h3_exec_info{};
    if (window_bytes < 0 || window_bytes > H3RR_STATIC_WINDOW_BYTES)
        return H3_ERR_UNSUPPORTED;  // more window than the library's static array holds
    if (window_bytes == 0)
        window_bytes = H3RR_STATIC_WINDOW_BYTES;
    void* window = nullptr;
    const cudaError_t err = h3rr::static_window_address(&window);
    if (err != cudaSuccess)
        return h3rr::record_cuda_failure(err);
    return h3rr::staged_relayout_with_window(true, send, recv, n_tokens, planes, n_heads, head_dim,
                                             world, window, window_bytes, stream, info);
}
