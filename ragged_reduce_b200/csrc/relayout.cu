// Ulysses relayout kernels for sm_100a: sequence->head and head->sequence.
//
// "Distributed H3 Execution", intro: the ulysses mode runs a QKV
// sequence-to-head all-to-all and the inverse head-to-sequence all-to-all
// around attention; "Partition Contract": 56 heads of width 128, balanced
// and ragged over the ranks.  With every virtual rank in one GPU's memory the
// all-to-all is a pure byte relayout: each (token, plane) row of the
// sequence side (H*D BF16 values, 14,336 bytes for H3) is cut into W
// contiguous runs of H_j*D values, one per head-side rank, and each run lands
// contiguously in that rank's [T, P, H_j, D] buffer.  Every byte is read once
// and written once; nothing is padded.
//
// The vector variant gives each 128-thread CTA one row at a time (or two):
// thread i owns the row's 16-byte vectors i, i+128, i+256, ..., so a warp
// touches 512 contiguous bytes on both sides.  The head-side rank, its base
// pointer and its row stride for each of a thread's vectors depend only on
// the column, so they are computed once per thread before the row loop.
// Sources are read with non-coherent streaming loads (inputs never overlap
// outputs; the host checks this), outputs are written with streaming stores.
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

__device__ __forceinline__ void st_stream(char* p, const uint4& v)
{
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// Owner rank and start of item x under the (q, m) split.
__device__ __forceinline__ int32_t split_owner(int32_t x, int32_t q, int32_t m)
{
    const int32_t big = m * (q + 1);
    return x < big ? x / (q + 1) : m + (x - big) / q;
}

__device__ __forceinline__ int32_t split_start(int32_t i, int32_t q, int32_t m)
{
    return i * q + (i < m ? i : m);
}

template <bool kSeqToHead, int VPT, int ROWS>
__global__ void __launch_bounds__(kThreads) relayout_vec_kernel(const __grid_constant__ RelayoutArgs a)
{
    // Head-side placement of this thread's columns (same for every row).
    char* hbase[VPT];
    int64_t hstride[VPT];
    bool live[VPT];
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        const int32_t c = threadIdx.x + k * kThreads;
        live[k] = c < a.row_vecs;
        const int32_t cc = live[k] ? c : 0;
        const int32_t h = cc / a.head_vecs;
        const int32_t within = cc - h * a.head_vecs;
        const int32_t j = split_owner(h, a.hq, a.hm);
        const int32_t hj = a.hq + (j < a.hm ? 1 : 0);
        const int32_t hl = h - split_start(j, a.hq, a.hm);
        hbase[k] = a.head[j] + (int64_t(hl) * a.head_vecs + within) * kVecBytes;
        hstride[k] = int64_t(hj) * a.head_vecs * kVecBytes;
    }
    const int64_t seq_row_bytes = int64_t(a.row_vecs) * kVecBytes;

    for (int64_t i0 = int64_t(blockIdx.x) * ROWS; i0 < a.rows; i0 += int64_t(gridDim.x) * ROWS) {
        char* sptr[ROWS];
        int64_t g[ROWS];
        bool rv[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            rv[r] = i0 + r < a.rows;
            const int32_t ii = int32_t(rv[r] ? i0 + r : i0);
            const int32_t t = ii / a.nplanes;
            const int32_t p = a.plane0 + (ii - t * a.nplanes);
            const int32_t s = split_owner(t, a.tq, a.tm);
            const int32_t tl = t - split_start(s, a.tq, a.tm);
            g[r] = int64_t(t) * a.P + p;
            sptr[r] = a.seq[s] + (int64_t(tl) * a.P + p) * seq_row_bytes +
                      int64_t(threadIdx.x) * kVecBytes;
        }
        uint4 v[ROWS][VPT];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                if (rv[r] && live[k]) {
                    const char* src = kSeqToHead ? sptr[r] + k * kThreads * kVecBytes
                                                 : hbase[k] + g[r] * hstride[k];
                    v[r][k] = ld_stream(src);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                if (rv[r] && live[k]) {
                    char* dst = kSeqToHead ? hbase[k] + g[r] * hstride[k]
                                           : sptr[r] + k * kThreads * kVecBytes;
                    st_stream(dst, v[r][k]);
                }
            }
        }
    }
}

// Any row width: one row per CTA iteration, head-side placement per vector.
template <bool kSeqToHead>
__global__ void __launch_bounds__(kThreads) relayout_generic_kernel(const __grid_constant__ RelayoutArgs a)
{
    const int64_t seq_row_bytes = int64_t(a.row_vecs) * kVecBytes;
    for (int64_t i64 = blockIdx.x; i64 < a.rows; i64 += gridDim.x) {
        const int32_t i = int32_t(i64);
        const int32_t t = i / a.nplanes;
        const int32_t p = a.plane0 + (i - t * a.nplanes);
        const int32_t s = split_owner(t, a.tq, a.tm);
        const int32_t tl = t - split_start(s, a.tq, a.tm);
        const int64_t g = int64_t(t) * a.P + p;
        char* srow = a.seq[s] + (int64_t(tl) * a.P + p) * seq_row_bytes;
        for (int32_t c = threadIdx.x; c < a.row_vecs; c += kThreads) {
            const int32_t h = c / a.head_vecs;
            const int32_t within = c - h * a.head_vecs;
            const int32_t j = split_owner(h, a.hq, a.hm);
            const int32_t hj = a.hq + (j < a.hm ? 1 : 0);
            const int32_t hl = h - split_start(j, a.hq, a.hm);
            char* hp = a.head[j] + ((g * hj + hl) * a.head_vecs + within) * kVecBytes;
            char* sp = srow + int64_t(c) * kVecBytes;
            if (kSeqToHead)
                st_stream(hp, ld_stream(sp));
            else
                st_stream(sp, ld_stream(hp));
        }
    }
}

template <bool kSeqToHead>
const void* pick_vec_kernel(int vpt, int* rows_per_iter)
{
    // Two rows per iteration keeps at least 8 vectors per thread in flight
    // when a row is narrow.
#define H3RR_VEC_CASE(V, R)                                             \
    case V:                                                             \
        *rows_per_iter = R;                                             \
        return (const void*)relayout_vec_kernel<kSeqToHead, V, R>;
    switch (vpt) {
        H3RR_VEC_CASE(1, 2)
        H3RR_VEC_CASE(2, 2)
        H3RR_VEC_CASE(3, 2)
        H3RR_VEC_CASE(4, 2)
        H3RR_VEC_CASE(5, 1)
        H3RR_VEC_CASE(6, 1)
        H3RR_VEC_CASE(7, 1)
        H3RR_VEC_CASE(8, 1)
        default:
            break;
    }
#undef H3RR_VEC_CASE
    *rows_per_iter = 1;
    return (const void*)relayout_generic_kernel<kSeqToHead>;
}

}  // namespace

cudaError_t launch_relayout(bool seq_to_head, const RelayoutArgs& a, int variant,
                            int ctas_per_sm, cudaStream_t stream, LaunchShape* shape)
{
    (void)variant;  // only the vector variant exists so far
    const int vpt = (a.row_vecs + kThreads - 1) / kThreads;
    int rows_per_iter = 1;
    const void* kernel = seq_to_head ? pick_vec_kernel<true>(vpt, &rows_per_iter)
                                     : pick_vec_kernel<false>(vpt, &rows_per_iter);
    int device = 0;
    const int sms = current_sm_count(&device);
    if (sms <= 0)
        return cudaErrorNoDevice;
    const int per_sm = ctas_per_sm > 0 ? ctas_per_sm : resident_ctas(kernel, kThreads, 0, device);
    const int64_t needed = (int64_t(a.rows) + rows_per_iter - 1) / rows_per_iter;
    int64_t grid = int64_t(sms) * per_sm;
    if (grid > needed)
        grid = needed;
    if (grid < 1)
        grid = 1;
    if (shape) {
        shape->grid = int(grid);
        shape->block = kThreads;
        shape->variant = H3_VARIANT_VECTOR;
    }
    void* params[] = {const_cast<RelayoutArgs*>(&a)};
    return cudaLaunchKernel(kernel, dim3(unsigned(grid)), dim3(kThreads), params, 0, stream);
}

}  // namespace h3rr
