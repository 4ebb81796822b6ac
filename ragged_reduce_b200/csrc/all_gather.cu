// Ragged all-gather of token rows for sm_100a.
//
// "Distributed H3 Execution", intro: ragged row gathering (its temporary
// collective padding is removed before model operations); "Validation":
// ragged gather and reduce-scatter behaviour.  Rank r holds rows
// ts_r .. te_r-1 of a [T, C] activation as a [T_r, C] block; after the gather
// every rank holds all T rows.  With every virtual rank in one GPU's memory
// there is nothing to pad: each row is read once from its owner's block and
// written to each of the W outputs.  A bulk-copy variant (H3_VARIANT_BULK)
// moves whole rows through shared memory instead of registers.
//
// A CTA of NT threads takes one token row per iteration (grid-stride); thread
// i owns the row's vectors i, i+NT, ... (32 bytes when every pointer and the
// row allow it, else 16), loads all of them, then stores each to the W
// outputs.  Non-coherent streaming loads (inputs never overlap outputs; the
// host checks this), streaming stores.
#include "bulk_copy.cuh"
#include "device_access.cuh"
#include "h3rr_internal.h"

namespace h3rr {

// Count of bounded waits that expired in the bulk all-gather kernel (per device).
__device__ unsigned int g_gather_wait_timeouts = 0;

namespace {

template <int VW, int NT, int VPT>
__global__ void __launch_bounds__(NT) all_gather_vec_kernel(const __grid_constant__ GatherArgs a)
{
    constexpr int kUnits = VW / kVecBytes;
    const int32_t row_v = a.row_vecs / kUnits;
    // Programmatic launch: the previous kernel in the stream completes before
    // the first memory access.
    pdl_wait_prerequisites();
    pdl_allow_dependents();
    for (int64_t t64 = blockIdx.x; t64 < a.T; t64 += gridDim.x) {
        const int32_t t = int32_t(t64);
        const int32_t s = split_owner(t, a.tq, a.tm);
        const int32_t tl = t - split_start(s, a.tq, a.tm);
        const char* src = a.in[s] + int64_t(tl) * a.row_bytes;
        const int64_t dst_off = int64_t(t) * a.row_bytes;
        Vec<VW> v[VPT];
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int32_t c = threadIdx.x + k * NT;
            if (c < row_v)
                ld_stream(v[k], src + int64_t(c) * VW);
        }
        for (int j = 0; j < a.W; ++j) {
            char* dst = a.out[j] + dst_off;
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                const int32_t c = threadIdx.x + k * NT;
                if (c < row_v)
                    st_stream(dst + int64_t(c) * VW, v[k]);
            }
        }
    }
}

// Any row width: 16-byte vectors, one vector per thread at a time.
constexpr int kGenericThreads = 128;

__global__ void __launch_bounds__(kGenericThreads) all_gather_generic_kernel(const __grid_constant__ GatherArgs a)
{
    // Programmatic launch: the previous kernel in the stream completes before
    // the first memory access.
    pdl_wait_prerequisites();
    pdl_allow_dependents();
    for (int64_t t64 = blockIdx.x; t64 < a.T; t64 += gridDim.x) {
        const int32_t t = int32_t(t64);
        const int32_t s = split_owner(t, a.tq, a.tm);
        const int32_t tl = t - split_start(s, a.tq, a.tm);
        const char* src = a.in[s] + int64_t(tl) * a.row_bytes;
        const int64_t dst_off = int64_t(t) * a.row_bytes;
        for (int32_t c = threadIdx.x; c < a.row_vecs; c += kGenericThreads) {
            Vec<16> v;
            ld_stream(v, src + int64_t(c) * kVecBytes);
            for (int j = 0; j < a.W; ++j)
                st_stream(a.out[j] + dst_off + int64_t(c) * kVecBytes, v);
        }
    }
}

// ---------------------------------------------------------------------------
// bulk variant: a CTA is one warp and gathers kBulkRows consecutive token
// rows; lane r bulk-loads row r once into its own shared-memory stage, waits
// on its own mbarrier and bulk-stores the stage to each of the W outputs (the
// copy engine does the fan-out).  One CTA per row group, scheduled by the
// hardware (not persistent); no multicast, no L2 cache hint.  Waits are
// bounded; expiries are counted in g_gather_wait_timeouts and reported with
// the relayout's count.
// ---------------------------------------------------------------------------
constexpr int kBulkRows = 4;
constexpr int kBulkBarrierBytes = 128;  // the lanes' mbarriers, padded to keep stages aligned

__global__ void __launch_bounds__(32) all_gather_bulk_kernel(const __grid_constant__ GatherArgs a)
{
    static_assert(kBulkRows <= 32 && kBulkRows * 8 <= kBulkBarrierBytes, "bulk CTA shape");
    extern __shared__ __align__(128) unsigned char smem[];
    const int lane = int(threadIdx.x);
    const bool driver = lane < kBulkRows;
    const uint32_t row_bytes = uint32_t(a.row_bytes);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem) + (driver ? lane : 0);
    unsigned char* stage = smem + kBulkBarrierBytes + size_t(driver ? lane : 0) * row_bytes;
    if (driver) {
        mbar_init(bar, 1);
        mbar_fence_init();
    }
    // Programmatic launch: the previous kernel in the stream completes before
    // the first global access.
    pdl_wait_prerequisites();
    pdl_allow_dependents();
    if (!driver)
        return;
    const int64_t stride = int64_t(gridDim.x) * kBulkRows;
    uint32_t parity = 0;
    for (int64_t t64 = int64_t(blockIdx.x) * kBulkRows + lane; t64 < a.T; t64 += stride) {
        if (t64 >= stride)
            bulk_wait_read<0>();  // a later row: the stage's previous stores have read it
        const int32_t t = int32_t(t64);
        const int32_t s = split_owner(t, a.tq, a.tm);
        const int32_t tl = t - split_start(s, a.tq, a.tm);
        mbar_arrive_expect_tx(bar, row_bytes);
        bulk_load(stage, a.in[s] + int64_t(tl) * row_bytes, row_bytes, bar);
        if (!mbar_wait(bar, parity)) {
            atomicAdd(&g_gather_wait_timeouts, 1u);
            mbar_wait(bar, parity);  // give the copy in flight one more bounded wait
            break;
        }
        parity ^= 1u;
        for (int j = 0; j < a.W; ++j)
            bulk_store(a.out[j] + int64_t(t) * row_bytes, stage, row_bytes);
        bulk_commit();
    }
    bulk_wait_all();
}

struct GatherChoice {
    const void* fn = nullptr;
    int threads = 0;
    size_t smem = 0;
    int variant = H3_VARIANT_GATHER;
};

template <int VW, int NT>
bool pick(int need, GatherChoice* gc)
{
#define H3RR_GATHER_VPT(V)                                             \
    if (need <= V) {                                                   \
        gc->fn = (const void*)all_gather_vec_kernel<VW, NT, V>;        \
        gc->threads = NT;                                              \
        return true;                                                   \
    }
    H3RR_GATHER_VPT(1)
    H3RR_GATHER_VPT(2)
    H3RR_GATHER_VPT(4)
    H3RR_GATHER_VPT(7)
    H3RR_GATHER_VPT(8)
#undef H3RR_GATHER_VPT
    return false;
}

bool wide_ok(const GatherArgs& a)
{
    if ((a.row_bytes % 32) != 0)
        return false;
    for (int r = 0; r < a.n_in; ++r)
        if (reinterpret_cast<uintptr_t>(a.in[r]) & 31u)
            return false;
    for (int j = 0; j < a.W; ++j)
        if (reinterpret_cast<uintptr_t>(a.out[j]) & 31u)
            return false;
    return true;
}

}  // namespace

bool all_gather_bulk_fits(const GatherArgs& a, int device)
{
    int max_smem = 0;
    if (cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) != cudaSuccess)
        return false;
    return size_t(kBulkBarrierBytes) + size_t(kBulkRows) * size_t(a.row_bytes) <= size_t(max_smem);
}

cudaError_t launch_all_gather(const GatherArgs& a, int variant, int ctas_per_sm, cudaStream_t stream,
                              LaunchShape* shape, bool programmatic)
{
    int device = 0;
    const int sms = current_sm_count(&device);
    if (sms <= 0)
        return cudaErrorNoDevice;
    GatherChoice gc;
    if (variant == H3_VARIANT_BULK) {
        if (!all_gather_bulk_fits(a, device))
            return cudaErrorInvalidConfiguration;
        gc.fn = (const void*)all_gather_bulk_kernel;
        gc.threads = 32;
        gc.smem = size_t(kBulkBarrierBytes) + size_t(kBulkRows) * size_t(a.row_bytes);
        gc.variant = H3_VARIANT_BULK;
        const cudaError_t err = allow_dynamic_smem(gc.fn, gc.smem, device);
        if (err != cudaSuccess)
            return err;
    } else {
        bool ok = false;
        if (wide_ok(a))
            ok = pick<32, 64>((a.row_vecs / 2 + 63) / 64, &gc);
        if (!ok)
            ok = pick<16, 128>((a.row_vecs + 127) / 128, &gc);
        if (!ok) {
            gc.fn = (const void*)all_gather_generic_kernel;
            gc.threads = kGenericThreads;
        }
    }
    // One CTA per token row (per kBulkRows rows for the bulk kernel) by
    // default, scheduled by the hardware: on B200 that measured 6.6-6.8 TB/s
    // against 5.6-6.0 TB/s for persistent grid-stride launches.
    // ctas_per_sm > 0 caps the grid (grid-stride).
    const int64_t needed = gc.variant == H3_VARIANT_BULK ? (int64_t(a.T) + kBulkRows - 1) / kBulkRows
                                                          : int64_t(a.T);
    int64_t grid = needed;
    if (ctas_per_sm > 0)
        grid = int64_t(sms) * ctas_per_sm;
    if (grid > needed)
        grid = needed;
    if (grid < 1)
        grid = 1;
    if (shape) {
        shape->grid = int(grid);
        shape->block = gc.threads;
        shape->variant = gc.variant;
    }
    // Every all-gather kernel follows the griddepcontrol protocol.
    void* params[] = {const_cast<GatherArgs*>(&a)};
    return launch_kernel(gc.fn, grid, gc.threads, gc.smem, stream, params, programmatic);
}

cudaError_t read_gather_wait_timeouts(unsigned int* count, bool reset, cudaStream_t stream)
{
    cudaError_t err = cudaMemcpyFromSymbolAsync(count, g_gather_wait_timeouts, sizeof(unsigned int), 0,
                                                cudaMemcpyDeviceToHost, stream);
    if (err == cudaSuccess)
        err = cudaStreamSynchronize(stream);
    if (err == cudaSuccess && reset) {
        static const unsigned int zero = 0;
        err = cudaMemcpyToSymbolAsync(g_gather_wait_timeouts, &zero, sizeof(zero), 0,
                                      cudaMemcpyHostToDevice, stream);
        if (err == cudaSuccess)
            err = cudaStreamSynchronize(stream);
    }
    return err;
}

}  // namespace h3rr
