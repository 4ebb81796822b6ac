// The binary32 arithmetic of the reduce-scatters (plain and gated), and the
// alignment test that selects their 32-byte kernels.
//
// "Distributed H3 Execution", "Partition Contract": the partial outputs are
// summed and the bias, left out of the partials, is added once after the
// reduction.  Every BF16 term is widened exactly to binary32, the partials
// are added in rank order 0..W-1 starting from partial 0, the bias is added
// once, and the sum is rounded to BF16 to nearest even.  The library is built
// without FMA contraction or flush-to-zero, so the bits are those of the
// sequential CPU definition.
#pragma once

#include <cuda_bf16.h>

#include "device_access.cuh"
#include "kernel_args.h"

namespace h3rr {

constexpr int kReduceThreads = 128;  // block size of the 16-byte kernels

// Exact widening of a vector of BF16 values to binary32 (the 16 bits become
// the top half of the word), the rank-ordered binary32 add, and rounding
// back to BF16 to nearest even.
template <int VW>
__device__ __forceinline__ void widen(const Vec<VW>& v, float* f)
{
#pragma unroll
    for (int i = 0; i < VW / 4; ++i) {
        f[2 * i] = __uint_as_float(v.r[i] << 16);
        f[2 * i + 1] = __uint_as_float(v.r[i] & 0xFFFF0000u);
    }
}

template <int VW>
__device__ __forceinline__ void add_widened(const Vec<VW>& v, float* acc)
{
#pragma unroll
    for (int i = 0; i < VW / 4; ++i) {
        acc[2 * i] = __fadd_rn(acc[2 * i], __uint_as_float(v.r[i] << 16));
        acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __uint_as_float(v.r[i] & 0xFFFF0000u));
    }
}

template <int VW>
__device__ __forceinline__ Vec<VW> narrow_rne(const float* acc)
{
    Vec<VW> o;
#pragma unroll
    for (int i = 0; i < VW / 4; ++i) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        o.r[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    return o;
}

// Every row start and buffer 32-byte aligned (the 32-byte kernels' condition).
inline bool wide_rows_ok(const ReduceArgs& a)
{
    if ((a.row_bytes % 32) != 0 || (reinterpret_cast<uintptr_t>(a.bias) & 31u))
        return false;
    for (int r = 0; r < a.W; ++r)
        if ((reinterpret_cast<uintptr_t>(a.part[r]) & 31u) || (reinterpret_cast<uintptr_t>(a.out[r]) & 31u))
            return false;
    return true;
}

}  // namespace h3rr
