// Tensor-mode ragged reduce-scatter kernel for sm_100a.
//
// "Distributed H3 Execution", "Partition Contract": each rank computes a
// partial output, a ragged reduce-scatter sums the partials and assigns token
// rows, and the projection bias, left out of the partials, is added exactly
// once after the reduction.  Token rows go to ranks by the quotient/remainder
// split.
//
// Per output element: widen the W BF16 partials exactly to binary32, add them
// in rank order 0..W-1 starting from partial 0, add the bias once, round to
// BF16 to nearest even.  The library is compiled without FMA contraction or
// flush-to-zero, so the result is the same bit pattern the sequential CPU
// definition gives.
//
// Layout of the work: a CTA of 128 threads takes one token row at a time;
// each thread owns 16-byte column vectors tid, tid+128, ... of the row and,
// for U of them at once, issues all W partial loads before the first add, so
// U*W 16-byte loads per thread are in flight.  The row's owner rank is
// computed once per row.  (128 threads with one vector per thread measured
// fastest on B200 at W = 6 and 8.)
#include <cuda_bf16.h>

#include "h3rr_internal.h"

namespace h3rr {
namespace {

constexpr int kThreads = 128;

__device__ __forceinline__ uint4 ld_stream(const char* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ld_cached(const char* p)
{
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_stream(char* p, const uint4& v)
{
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ int32_t split_owner(int32_t x, int32_t q, int32_t m)
{
    const int32_t big = m * (q + 1);
    return x < big ? x / (q + 1) : m + (x - big) / q;
}

__device__ __forceinline__ int32_t split_start(int32_t i, int32_t q, int32_t m)
{
    return i * q + (i < m ? i : m);
}

// BF16 -> binary32 is exact: the 16 bits become the top half of the word.
__device__ __forceinline__ void widen(const uint4& v, float* f)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void add_widened(const uint4& v, float* acc)
{
    float f[8];
    widen(v, f);
#pragma unroll
    for (int e = 0; e < 8; ++e)
        acc[e] = __fadd_rn(acc[e], f[e]);
}

__device__ __forceinline__ uint4 narrow_rne(const float* acc)
{
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
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
                uint4 x[U][kBatch];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int64_t off = in_off + int64_t(c0 + u * kThreads) * kVecBytes;
#pragma unroll
                    for (int b = 0; b < kBatch; ++b)
                        if (live[u] && w0 + b < W)
                            x[u][b] = ld_stream(a.part[w0 + b] + off);
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
                for (int u = 0; u < U; ++u)
                    if (live[u])
                        add_widened(ld_cached(a.bias + int64_t(c0 + u * kThreads) * kVecBytes),
                                    acc[u]);
            }
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (live[u])
                    st_stream(orow + int64_t(c0 + u * kThreads) * kVecBytes, narrow_rne(acc[u]));
        }
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

// ---------------------------------------------------------------------------
// Reduce-scatter fused with residual gating ("Distributed H3 Execution",
// "Partition Contract": segment boundaries clipped to each rank's token
// interval and rebased before AdaLN modulation and residual gating).  Per
// element: y = the reduce-scatter output (rounded to BF16, exactly as the
// plain kernel writes it), then out = bf16_rne(x + gate[seg(t)] * y) in
// binary32.  The product of two BF16 values is exact in binary32, so only the
// add rounds; fusing changes no bits against running the two steps in turn and
// saves writing and re-reading y.  seg(t) is found by binary search over the
// packed segment bounds (the rank's clipped pieces name the same segments).
// x may be the output buffer itself (in place): each element is read by the
// thread that then writes it, with plain (coherent) loads.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 ld_plain(const char* p)
{
    uint4 v;
    asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

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
                uint4 xv[kBatch];
#pragma unroll
                for (int b = 0; b < kBatch; ++b)
                    if (w0 + b < W)
                        xv[b] = ld_stream(a.part[w0 + b] + in_off + off);
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
            if (a.bias != nullptr)
                add_widened(ld_cached(a.bias + off), acc);
            float y[8], gt[8], xr[8];
            widen(narrow_rne(acc), y);          // the reduce-scatter output, as BF16
            widen(ld_cached(grow + off), gt);
            widen(ld_plain(xrow + off), xr);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                acc[e] = __fadd_rn(xr[e], __fmul_rn(gt[e], y[e]));
            st_stream(orow + off, narrow_rne(acc));
        }
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
    int device = 0;
    const int sms = current_sm_count(&device);
    if (sms <= 0)
        return cudaErrorNoDevice;
    int64_t grid = a.r.T;  // one CTA per token row (see launch_reduce_scatter)
    if (grid < 1)
        grid = 1;
    if (shape) {
        shape->grid = int(grid);
        shape->block = kThreads;
        shape->variant = H3_VARIANT_REDUCE_GATED;
    }
    void* params[] = {const_cast<GatedArgs*>(&a)};
    return launch_kernel(kernel, grid, kThreads, 0, stream, params, programmatic);
}

cudaError_t launch_reduce_scatter(const ReduceArgs& a, int ctas_per_sm, cudaStream_t stream,
                                  LaunchShape* shape, bool programmatic)
{
    const void* kernel = pick_reduce_kernel(a.W);
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
        shape->block = kThreads;
        shape->variant = H3_VARIANT_REDUCE;
    }
    void* params[] = {const_cast<ReduceArgs*>(&a)};
    return launch_kernel(kernel, grid, kThreads, 0, stream, params, programmatic);
}

}  // namespace h3rr
