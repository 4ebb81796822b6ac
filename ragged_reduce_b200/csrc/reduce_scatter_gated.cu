// Reduce-scatter fused with residual gating for sm_100a ("Distributed H3
// Execution", "Partition Contract": segment boundaries clipped to each rank's
// token interval and rebased before AdaLN modulation and residual gating).  Per
// element: y = the reduce-scatter output (rounded to BF16, exactly as the
// plain kernel writes it), then out = bf16_rne(x + gate[seg(t)] * y) in
// binary32.  The product of two BF16 values is exact in binary32, so only the
// add rounds; fusing changes no bits against running the two steps in turn and
// saves writing and re-reading y.  seg(t) is found by binary search over the
// packed segment bounds (the rank's clipped pieces name the same segments).
// x may be the output buffer itself (in place): each element is read by the
// thread that then writes it, with plain (coherent) loads.
#include "bf16_sum.cuh"
#include "h3rr_internal.h"

namespace h3rr {
namespace {

constexpr int kThreads = kReduceThreads;

template <int kW>
__global__ void __launch_bounds__(kThreads) reduce_scatter_gated_kernel(const __grid_constant__ GatedArgs g)
{
    const ReduceArgs& a = g.r;
    constexpr int kBatch = kW > 0 ? kW : 8;
    // Programmatic launch: the previous kernel in the stream completes before
    // the first memory access.
    pdl_wait_prerequisites();
    pdl_allow_dependents();
    for (int64_t t64 = blockIdx.x; t64 < a.T; t64 += gridDim.x) {
        const int32_t t = int32_t(t64);
        const int32_t s = split_owner(t, a.tq, a.tm);
        const int32_t tl = t - split_start(s, a.tq, a.tm);
        int32_t lo = 0, hi = g.n_segs;  // largest k with bounds[k] <= t
        while (hi - lo > 1) {
            const int32_t mid = (lo + hi) >> 1;
            if (g.seg_bounds[mid] <= t)
                lo = mid;
            else
                hi = mid;
        }
        const char* grow = g.gate + int64_t(lo) * a.row_bytes;
        const char* xrow = g.x[s] + int64_t(tl) * a.row_bytes;
        char* orow = a.out[s] + int64_t(tl) * a.row_bytes;
        const int64_t in_off = int64_t(t) * a.row_bytes;
        for (int32_t c = threadIdx.x; c < a.row_vecs; c += kThreads) {
            const int64_t off = int64_t(c) * kVecBytes;
            float acc[8];
            const int W = kW > 0 ? kW : a.W;
            for (int w0 = 0; w0 < W; w0 += kBatch) {
                Vec<16> xv[kBatch];
#pragma unroll
                for (int b = 0; b < kBatch; ++b)
                    if (w0 + b < W)
                        ld_stream(xv[b], a.part[w0 + b] + in_off + off);
#pragma unroll
                for (int b = 0; b < kBatch; ++b) {
                    if (w0 + b >= W)
                        break;
                    if (w0 + b == 0)
                        widen(xv[b], acc);
                    else
                        add_widened(xv[b], acc);
                }
            }
            if (a.bias != nullptr) {
                Vec<16> bv;
                ld_cached(bv, a.bias + off);
                add_widened(bv, acc);
            }
            float y[8], gt[8], xr[8];
            widen(narrow_rne<16>(acc), y);  // the reduce-scatter output, as BF16
            Vec<16> gv, xv2;
            ld_cached(gv, grow + off);
            ld_plain(xv2, xrow + off);
            widen(gv, gt);
            widen(xv2, xr);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                acc[e] = __fadd_rn(xr[e], __fmul_rn(gt[e], y[e]));
            st_stream(orow + off, narrow_rne<16>(acc));
        }
    }
}

// The gated kernel with 32-byte vectors, U per thread at once (as
// reduce_scatter_wide_kernel); same arithmetic per element.
template <int kW, int U, int NT>
__global__ void __launch_bounds__(NT) reduce_scatter_gated_wide_kernel(const __grid_constant__ GatedArgs g)
{
    const ReduceArgs& a = g.r;
    const int32_t row_v = a.row_vecs / 2;
    pdl_wait_prerequisites();
    pdl_allow_dependents();
    for (int64_t t64 = blockIdx.x; t64 < a.T; t64 += gridDim.x) {
        const int32_t t = int32_t(t64);
        const int32_t s = split_owner(t, a.tq, a.tm);
        const int32_t tl = t - split_start(s, a.tq, a.tm);
        int32_t lo = 0, hi = g.n_segs;  // largest k with bounds[k] <= t
        while (hi - lo > 1) {
            const int32_t mid = (lo + hi) >> 1;
            if (g.seg_bounds[mid] <= t)
                lo = mid;
            else
                hi = mid;
        }
        const char* grow = g.gate + int64_t(lo) * a.row_bytes;
        const char* xrow = g.x[s] + int64_t(tl) * a.row_bytes;
        char* orow = a.out[s] + int64_t(tl) * a.row_bytes;
        const int64_t in_off = int64_t(t) * a.row_bytes;
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
                const int64_t off = int64_t(c0 + u * NT) * 32;
                float acc[16];
                widen(x[u][0], acc);
#pragma unroll
                for (int b = 1; b < kW; ++b)
                    add_widened(x[u][b], acc);
                if (a.bias != nullptr) {
                    Vec<32> bv;
                    ld_cached(bv, a.bias + off);
                    add_widened(bv, acc);
                }
                float y[16], gt[16], xr[16];
                widen(narrow_rne<32>(acc), y);  // the reduce-scatter output, as BF16
                Vec<32> gv, xv;
                ld_cached(gv, grow + off);
                ld_plain(xv, xrow + off);
                widen(gv, gt);
                widen(xv, xr);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    acc[e] = __fadd_rn(xr[e], __fmul_rn(gt[e], y[e]));
                st_stream(orow + off, narrow_rne<32>(acc));
            }
        }
    }
}

// One vector per thread: the gated kernel also loads the gate row and the
// residual, and measured 2-3 % faster with U = 1 (256 threads for W <= 6, 64
// for W = 7, 8) than with the plain kernel's two vectors per thread.
const void* pick_wide_gated_kernel(int W, int* threads)
{
    *threads = W <= 6 ? 256 : 64;
    switch (W) {
        case 1: return (const void*)reduce_scatter_gated_wide_kernel<1, 1, 256>;
        case 2: return (const void*)reduce_scatter_gated_wide_kernel<2, 1, 256>;
        case 3: return (const void*)reduce_scatter_gated_wide_kernel<3, 1, 256>;
        case 4: return (const void*)reduce_scatter_gated_wide_kernel<4, 1, 256>;
        case 5: return (const void*)reduce_scatter_gated_wide_kernel<5, 1, 256>;
        case 6: return (const void*)reduce_scatter_gated_wide_kernel<6, 1, 256>;
        case 7: return (const void*)reduce_scatter_gated_wide_kernel<7, 1, 64>;
        case 8: return (const void*)reduce_scatter_gated_wide_kernel<8, 1, 64>;
        default: return nullptr;
    }
}

const void* pick_gated_kernel(int W)
{
    switch (W) {
        case 1: return (const void*)reduce_scatter_gated_kernel<1>;
        case 2: return (const void*)reduce_scatter_gated_kernel<2>;
        case 3: return (const void*)reduce_scatter_gated_kernel<3>;
        case 4: return (const void*)reduce_scatter_gated_kernel<4>;
        case 5: return (const void*)reduce_scatter_gated_kernel<5>;
        case 6: return (const void*)reduce_scatter_gated_kernel<6>;
        case 7: return (const void*)reduce_scatter_gated_kernel<7>;
        case 8: return (const void*)reduce_scatter_gated_kernel<8>;
        default: return (const void*)reduce_scatter_gated_kernel<0>;
    }
}

}  // namespace

cudaError_t launch_reduce_scatter_gated(const GatedArgs& a, cudaStream_t stream, LaunchShape* shape,
                                        bool programmatic)
{
    const void* kernel = pick_gated_kernel(a.r.W);
    int threads = kThreads;
    bool wide = wide_rows_ok(a.r) && (reinterpret_cast<uintptr_t>(a.gate) & 31u) == 0;
    for (int r = 0; wide && r < a.r.W; ++r)
        wide = (reinterpret_cast<uintptr_t>(a.x[r]) & 31u) == 0;
    if (wide) {
        int wide_threads = 0;
        if (const void* k = pick_wide_gated_kernel(a.r.W, &wide_threads)) {
            kernel = k;
            threads = wide_threads;
        }
    }
    int device = 0;
    const int sms = current_sm_count(&device);
    if (sms <= 0)
        return cudaErrorNoDevice;
    int64_t grid = a.r.T;  // one CTA per token row (see launch_reduce_scatter)
    if (grid < 1)
        grid = 1;
    if (shape) {
        shape->grid = int(grid);
        shape->block = threads;
        shape->variant = H3_VARIANT_REDUCE_GATED;
    }
    void* params[] = {const_cast<GatedArgs*>(&a)};
    return launch_kernel(kernel, grid, threads, 0, stream, params, programmatic);
}

}  // namespace h3rr
