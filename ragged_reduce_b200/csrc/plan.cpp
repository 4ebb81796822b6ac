// Host-side partition plan: quotient/remainder splits, segment clipping,
// overlap checks and the per-device launch caches.
//
// "Distributed H3 Execution", "Partition Contract": head ownership is
// balanced and may be ragged (W=6 -> 10,10,9,9,9,9: the first ranks take the
// remainder); token ranges use the same split; segment boundaries are clipped
// to each rank's token interval and rebased before AdaLN modulation and
// residual gating.
#include <mutex>
#include <unordered_map>

#include <cuda.h>

#include "context.h"
#include "h3rr_internal.h"

namespace h3rr {

Split make_split(int64_t n, int32_t w)
{
    Split s;
    s.w = w;
    s.q = n / w;
    s.m = n % w;
    return s;
}

namespace {

// Token ranges of one plane group moving `planes` planes per launch.
h3_status plan_ranges(const Split& ts, const Split& hs, int64_t n_tokens, int64_t planes,
                      uint64_t row_bytes, uint64_t head_bytes, uint64_t window,
                      int64_t* per_group, int64_t* tokens)
{
    const int64_t tmax = ts.largest();
    const uint64_t send_token = uint64_t(planes) * row_bytes;  // one token of a rank, every plane moved
    const uint64_t recv_token = uint64_t(planes) * uint64_t(hs.largest()) * head_bytes;
    if (uint64_t(tmax) * send_token <= window && uint64_t(n_tokens) * recv_token <= window) {
        *per_group = 1;
        *tokens = tmax;
        return H3_OK;
    }
    // A full range sends L tokens from every rank and gives every head rank L
    // tokens from each of the W ranks.
    const uint64_t by_send = window / send_token;
    const uint64_t by_recv = window / (uint64_t(ts.w) * recv_token);
    const uint64_t most = by_send < by_recv ? by_send : by_recv;
    if (most < 1)
        return H3_ERR_WINDOW;
    // Fewest ranges, then equal lengths: ceil(tmax / L) is again k, so every
    // range but the last is full and the last is not empty.
    const int64_t k = (tmax + int64_t(most) - 1) / int64_t(most);
    *per_group = k;
    *tokens = (tmax + k - 1) / k;
    return H3_OK;
}

}  // namespace

h3_status plan_relayout(const Split& ts, const Split& hs, int64_t n_tokens, int32_t planes,
                        uint64_t row_bytes, uint64_t head_bytes, int64_t window_bytes,
                        bool token_ranges, RelayoutChunks* out)
{
    if (window_bytes <= 0) {
        out->plane_groups = 1;
        out->per_launch = planes;
        out->per_group = 1;
        out->tokens = ts.largest();
        return H3_OK;
    }
    out->plane_groups = token_ranges ? 1 : planes;
    out->per_launch = token_ranges ? planes : 1;
    return plan_ranges(ts, hs, n_tokens, out->per_launch, row_bytes, head_bytes, uint64_t(window_bytes),
                       &out->per_group, &out->tokens);
}

void chunk_split(const Split& ts, const RelayoutChunks& ch, int64_t c, int64_t* cq, int64_t* cm,
                 int64_t* t0)
{
    *t0 = c * ch.tokens;
    if (c + 1 < ch.per_group) {
        *cq = ch.tokens;
        *cm = 0;
    } else {
        *cq = ts.q - *t0;
        *cm = ts.m;
    }
}

int32_t clip_segments(const int64_t* bounds, int32_t n_segs, int64_t ts, int64_t te,
                      int64_t* local_bounds, int32_t* seg_ids)
{
    // Segments tile [0, T) in order, so the pieces inside [ts, te) are the
    // segments from the one holding ts up to the one holding te-1.
    int32_t pieces = 0;
    for (int32_t k = 0; k < n_segs; ++k) {
        const int64_t lo = bounds[k] < ts ? ts : bounds[k];
        const int64_t hi = bounds[k + 1] > te ? te : bounds[k + 1];
        if (hi <= lo)
            continue;
        local_bounds[pieces] = lo - ts;
        seg_ids[pieces] = k;
        ++pieces;
    }
    local_bounds[pieces] = te - ts;
    return pieces;
}

bool ranges_overlap(uintptr_t a, uint64_t na, uintptr_t b, uint64_t nb)
{
    if (na == 0 || nb == 0)
        return false;
    return a < b + nb && b < a + na;
}

namespace {

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// The driver's cuCtxGetCurrent and cuCtxGetId (CUDA 12.0), fetched through
// the runtime's entry-point query (no link against libcuda); null if
// unavailable.
struct ContextQuery {
    CtxGetCurrentFn current = nullptr;
    CtxGetIdFn id = nullptr;
};

const ContextQuery& context_query()
{
    static std::once_flag once;
    static ContextQuery q;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult r = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &r) ==
                cudaSuccess &&
            r == cudaDriverEntryPointSuccess)
            q.current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        r = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &r) ==
                cudaSuccess &&
            r == cudaDriverEntryPointSuccess)
            q.id = reinterpret_cast<CtxGetIdFn>(p);
    });
    return q;
}

}  // namespace

bool current_context_id(unsigned long long* id)
{
    const ContextQuery& q = context_query();
    if (!q.current || !q.id)
        return false;
    CUcontext ctx = nullptr;
    if (q.current(&ctx) != CUDA_SUCCESS || !ctx)
        return false;
    return q.id(ctx, id) == CUDA_SUCCESS;
}

int current_sm_count(int* device)
{
    static std::mutex mu;
    static std::unordered_map<int, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return 0;
    if (device)
        *device = dev;
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(dev);
    if (it != cache.end())
        return it->second;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    cache.emplace(dev, n);
    return n;
}

cudaError_t allow_dynamic_smem(const void* kernel, size_t smem, int device)
{
    // The opt-in is one value per kernel, so it is raised once per kernel and
    // context to the device's whole opt-in limit; any later launch with a
    // smaller ring then stays within it.  (Setting it to each launch's own
    // size would lower it under a later, larger launch.)  It belongs to the
    // context: after cudaDeviceReset the next context starts from the
    // default, so the cache is keyed by the context's id; without an id the
    // opt-in is set on every call.
    if (smem <= 48 * 1024)
        return cudaSuccess;
    struct Key {
        const void* k;
        int dev;
        unsigned long long ctx;
        bool operator==(const Key& o) const { return k == o.k && dev == o.dev && ctx == o.ctx; }
    };
    struct Hash {
        size_t operator()(const Key& x) const
        {
            return std::hash<const void*>()(x.k) ^ size_t(x.dev) ^ std::hash<unsigned long long>()(x.ctx);
        }
    };
    static std::mutex mu;
    static std::unordered_map<Key, int, Hash> limit;
    unsigned long long ctx = 0;
    const bool keyed = current_context_id(&ctx);
    std::lock_guard<std::mutex> lock(mu);
    const Key key{kernel, device, ctx};
    if (keyed) {
        auto it = limit.find(key);
        if (it != limit.end())
            return smem <= size_t(it->second) ? cudaSuccess : cudaErrorInvalidValue;
    }
    int optin = 0;
    cudaError_t err = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
    if (err != cudaSuccess)
        return err;
    if (smem > size_t(optin))
        return cudaErrorInvalidValue;
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (err == cudaSuccess && keyed)
        limit.emplace(key, optin);
    return err;
}

cudaError_t launch_kernel(const void* kernel, int64_t grid, int block, size_t smem,
                          cudaStream_t stream, void** params, bool programmatic)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid));
    cfg.blockDim = dim3(unsigned(block));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    if (programmatic) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelExC(&cfg, kernel, params);
}

}  // namespace h3rr
