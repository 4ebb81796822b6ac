// Tensor-mode ragged reduce-scatter kernel for sm_100a.
//
// "Distributed H3 Execution", "Partition Contract": each rank computes a
// partial output, a ragged reduce-scatter sums the partials and assigns token
// rows, and the projection bias, left out of the partials, is added exactly
// once after the reduction.  Token rows go to ranks by the quotient/remainder
// split.
//
// Per output element: the rank-ordered binary32 sum of bf16_sum.cuh.
//
// Layout of the work: one CTA per token row; each thread owns column vectors
// tid, tid+NT, ... of the row and, for U of them at once, issues all W
// partial loads before the first add, so U*W vector loads per thread are in
// flight.  The row's owner rank is computed once per row.  With every row
// and pointer 32-byte aligned (the H3 case, C = 7168) the kernel moves
// 32-byte vectors (16 BF16 values), two per thread, 128 threads for W <= 6
// and 64 for W = 7, 8: 5-7 % faster on B200 than 16-byte vectors.  Otherwise
// 16-byte vectors with 128 threads; W > 8 loads the partials in batches of 8.
// The gated variant is in reduce_scatter_gated.cu.
#include "bf16_sum.cuh"
#include "h3rr_internal.h"

namespace h3rr {
namespace {

constexpr int kThreads = kReduceThreads;

// 32-byte vectors, W fixed at compile time (1..8), U vectors per thread at
// once: all U*W partial loads are issued before the first add.
template <int kW, int U, int NT>
__global__ void __launch_bounds__(NT) reduce_scatter_wide_kernel(const __grid_constant__ ReduceArgs a)
{
    const int32_t row_v = a.row_vecs / 2;  // 32-byte vectors per row
    pdl_wait_prerequisites();
    pdl_allow_dependents();
    for (int64_t t64 = blockIdx.x; t64 < a.T; t64 += gridDim.x) {
        const int32_t t = int32_t(t64);
        const int32_t s = split_owner(t, a.tq, a.tm);
        const int32_t tl = t - split_start(s, a.tq, a.tm);
        const int64_t in_off = int64_t(t) * a.row_bytes;
        char* orow = a.out[s] + int64_t(tl) * a.row_bytes;
        for (int32_t c0 = threadIdx.x; c0 < row_v; c0 += NT * U) {
            Vec<32> x[U][kW];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int b = 0; b < kW; ++b)
                    if (c0 + u * NT < row_v)
                        ld_stream(x[u][b], a.part[b] + in_off + int64_t(c0 + u * NT) * 32);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (c0 + u * NT >= row_v)
                    continue;
                float acc[16];
                widen(x[u][0], acc);
#pragma unroll
                for (int b = 1; b < kW; ++b)
                    add_widened(x[u][b], acc);
                if (a.bias != nullptr) {
                    Vec<32> bv;
                    ld_cached(bv, a.bias + int64_t(c0 + u * NT) * 32);
                    add_widened(bv, acc);
                }
                st_stream(orow + int64_t(c0 + u * NT) * 32, narrow_rne<32>(acc));
            }
        }
    }
}

// kW > 0: W fixed at compile time, all loads issued before the adds.
// kW == 0: W from the arguments, loaded in batches of 8 ranks (still summed
// strictly in rank order).
template <int kW, int U>
__global__ void __launch_bounds__(kThreads) reduce_scatter_kernel(const __grid_constant__ ReduceArgs a)
{
    constexpr int kBatch = kW > 0 ? kW : 8;
    // Programmatic launch: the previous kernel in the stream completes before
    // the first memory access.
    pdl_wait_prerequisites();
    pdl_allow_dependents();
    for (int64_t t64 = blockIdx.x; t64 < a.T; t64 += gridDim.x) {
        const int32_t t = int32_t(t64);
        const int32_t s = split_owner(t, a.tq, a.tm);
        const int32_t tl = t - split_start(s, a.tq, a.tm);
        const int64_t in_off = int64_t(t) * a.row_bytes;
        char* orow = a.out[s] + int64_t(tl) * a.row_bytes;
        for (int32_t c0 = threadIdx.x; c0 < a.row_vecs; c0 += kThreads * U) {
            float acc[U][8];
            bool live[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                live[u] = c0 + u * kThreads < a.row_vecs;
            const int W = kW > 0 ? kW : a.W;
            for (int w0 = 0; w0 < W; w0 += kBatch) {
                Vec<16> x[U][kBatch];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int64_t off = in_off + int64_t(c0 + u * kThreads) * kVecBytes;
#pragma unroll
                    for (int b = 0; b < kBatch; ++b)
                        if (live[u] && w0 + b < W)
                            ld_stream(x[u][b], a.part[w0 + b] + off);
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (!live[u])
                        continue;
#pragma unroll
                    for (int b = 0; b < kBatch; ++b) {
                        if (w0 + b >= W)
                            break;
                        if (w0 + b == 0)
                            widen(x[u][b], acc[u]);
                        else
                            add_widened(x[u][b], acc[u]);
                    }
                }
            }
            if (a.bias != nullptr) {
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (live[u]) {
                        Vec<16> bv;
                        ld_cached(bv, a.bias + int64_t(c0 + u * kThreads) * kVecBytes);
                        add_widened(bv, acc[u]);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (live[u])
                    st_stream(orow + int64_t(c0 + u * kThreads) * kVecBytes, narrow_rne<16>(acc[u]));
        }
    }
}

// The 32-byte kernel for W <= 8 (nullptr otherwise) and its block size.
const void* pick_wide_reduce_kernel(int W, int* threads)
{
    *threads = W <= 6 ? 128 : 64;
    switch (W) {
        case 1: return (const void*)reduce_scatter_wide_kernel<1, 2, 128>;
        case 2: return (const void*)reduce_scatter_wide_kernel<2, 2, 128>;
        case 3: return (const void*)reduce_scatter_wide_kernel<3, 2, 128>;
        case 4: return (const void*)reduce_scatter_wide_kernel<4, 2, 128>;
        case 5: return (const void*)reduce_scatter_wide_kernel<5, 2, 128>;
        case 6: return (const void*)reduce_scatter_wide_kernel<6, 2, 128>;
        case 7: return (const void*)reduce_scatter_wide_kernel<7, 2, 64>;
        case 8: return (const void*)reduce_scatter_wide_kernel<8, 2, 64>;
        default: return nullptr;
    }
}

const void* pick_reduce_kernel(int W)
{
    switch (W) {
        case 1: return (const void*)reduce_scatter_kernel<1, 2>;
        case 2: return (const void*)reduce_scatter_kernel<2, 2>;
        case 3: return (const void*)reduce_scatter_kernel<3, 1>;
        case 4: return (const void*)reduce_scatter_kernel<4, 1>;
        case 5: return (const void*)reduce_scatter_kernel<5, 1>;
        case 6: return (const void*)reduce_scatter_kernel<6, 1>;
        case 7: return (const void*)reduce_scatter_kernel<7, 1>;
        case 8: return (const void*)reduce_scatter_kernel<8, 1>;
        default: return (const void*)reduce_scatter_kernel<0, 1>;
    }
}

}  // namespace

cudaError_t launch_reduce_scatter(const ReduceArgs& a, int ctas_per_sm, cudaStream_t stream,
                                  LaunchShape* shape, bool programmatic)
{
    const void* kernel = pick_reduce_kernel(a.W);
    int threads = kThreads;
    if (wide_rows_ok(a)) {
        int wide_threads = 0;
        if (const void* wide = pick_wide_reduce_kernel(a.W, &wide_threads)) {
            kernel = wide;
            threads = wide_threads;
        }
    }
    int device = 0;
    const int sms = current_sm_count(&device);
    if (sms <= 0)
        return cudaErrorNoDevice;
    // One CTA per token row by default, scheduled by the hardware: on B200
    // that measured 1-11 % faster than persistent grid-stride launches, whose
    // lockstep sweep over the rows resonated with the DRAM mapping at some
    // grid sizes.  ctas_per_sm > 0 caps the grid (grid-stride).
    int64_t grid = ctas_per_sm > 0 ? int64_t(sms) * ctas_per_sm : int64_t(a.T);
    if (grid > a.T)
        grid = a.T;
    if (grid < 1)
        grid = 1;
    if (shape) {
        shape->grid = int(grid);
        shape->block = threads;
        shape->variant = H3_VARIANT_REDUCE;
    }
    void* params[] = {const_cast<ReduceArgs*>(&a)};
    return launch_kernel(kernel, grid, threads, 0, stream, params, programmatic);
}

}  // namespace h3rr
