// Ragged all-gather of token rows for sm_100a.
//
// "Distributed H3 Execution", intro: ragged row gathering (its temporary
// collective padding is removed before model operations); "Validation":
// ragged gather and reduce-scatter behaviour.  Rank r holds rows
// ts_r .. te_r-1 of a [T, C] activation as a [T_r, C] block; after the gather
// every rank holds all T rows.  With every virtual rank in one GPU's memory
// there is nothing to pad: each row is read once from its owner's block and
// written to each of the W outputs.
//
// A CTA of NT threads takes one token row per iteration (grid-stride); thread
// i owns the row's vectors i, i+NT, ... (32 bytes when every pointer and the
// row allow it, else 16), loads all of them, then stores each to the W
// outputs.  Non-coherent streaming loads (inputs never overlap outputs; the
// host checks this), streaming stores.
#include "h3rr_internal.h"

namespace h3rr {
namespace {

template <int VW>
struct Vec {
    uint32_t r[VW / 4];
};

__device__ __forceinline__ void ld_stream(Vec<16>& v, const char* p)
{
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.r[0]), "=r"(v.r[1]), "=r"(v.r[2]), "=r"(v.r[3])
                 : "l"(p));
}

__device__ __forceinline__ void ld_stream(Vec<32>& v, const char* p)
{
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v.r[0]), "=r"(v.r[1]), "=r"(v.r[2]), "=r"(v.r[3]), "=r"(v.r[4]),
                   "=r"(v.r[5]), "=r"(v.r[6]), "=r"(v.r[7])
                 : "l"(p));
}

__device__ __forceinline__ void st_stream(char* p, const Vec<16>& v)
{
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.r[0]), "r"(v.r[1]),
                 "r"(v.r[2]), "r"(v.r[3])
                 : "memory");
}

__device__ __forceinline__ void st_stream(char* p, const Vec<32>& v)
{
    asm volatile("st.global.cs.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p),
                 "r"(v.r[0]), "r"(v.r[1]), "r"(v.r[2]), "r"(v.r[3]), "r"(v.r[4]), "r"(v.r[5]),
                 "r"(v.r[6]), "r"(v.r[7])
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

template <int VW, int NT, int VPT>
__global__ void __launch_bounds__(NT) all_gather_vec_kernel(const __grid_constant__ GatherArgs a)
{
    constexpr int kUnits = VW / kVecBytes;
    const int32_t row_v = a.row_vecs / kUnits;
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

struct GatherChoice {
    const void* fn = nullptr;
    int threads = 0;
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
    for (int r = 0; r < a.W; ++r)
        if ((reinterpret_cast<uintptr_t>(a.in[r]) & 31u) || (reinterpret_cast<uintptr_t>(a.out[r]) & 31u))
            return false;
    return true;
}

}  // namespace

cudaError_t launch_all_gather(const GatherArgs& a, int ctas_per_sm, cudaStream_t stream, LaunchShape* shape)
{
    int device = 0;
    const int sms = current_sm_count(&device);
    if (sms <= 0)
        return cudaErrorNoDevice;
    GatherChoice gc;
    bool ok = false;
    if (wide_ok(a))
        ok = pick<32, 64>((a.row_vecs / 2 + 63) / 64, &gc);
    if (!ok)
        ok = pick<16, 128>((a.row_vecs + 127) / 128, &gc);
    if (!ok) {
        gc.fn = (const void*)all_gather_generic_kernel;
        gc.threads = kGenericThreads;
    }
    const int per_sm = ctas_per_sm > 0 ? ctas_per_sm : resident_ctas(gc.fn, gc.threads, 0, device);
    int64_t grid = int64_t(sms) * per_sm;
    if (grid > a.T)
        grid = a.T;
    if (grid < 1)
        grid = 1;
    if (shape) {
        shape->grid = int(grid);
        shape->block = gc.threads;
        shape->variant = H3_VARIANT_GATHER;
    }
    void* params[] = {const_cast<GatherArgs*>(&a)};
    return cudaLaunchKernel(gc.fn, dim3(unsigned(grid)), dim3(gc.threads), params, 0, stream);
}

}  // namespace h3rr
