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
// Two kernel families move the same bytes:
//
// * Vector kernels: a CTA of NT threads takes ROWS rows at a time; thread i
//   owns the row's vectors i, i+NT, i+2NT, ... (VW = 16 or 32 bytes, 32 when
//   every pointer and run allows it), so a warp touches 512 or 1024
//   contiguous bytes on both sides.  The head-side rank, base pointer and
//   row stride of each of a thread's vectors depend only on the column, so
//   they are computed once per thread before the row loop.  All loads of an
//   iteration are issued before its first store.  Sources use non-coherent
//   streaming loads (inputs never overlap outputs; the host checks this),
//   outputs streaming stores.
//
// * Bulk kernel: the tensor memory accelerator's 1-D bulk copies move each
//   row through shared memory.  A CTA is one warp; each of its first few
//   lanes owns one row, one shared-memory stage and one mbarrier that counts
//   the row's load bytes, and stores the stage once the load has landed.  No
//   multicast is used.  Every mbarrier wait is bounded: on expiry the kernel
//   counts the event in a device word (read with h3_bulk_wait_timeouts),
//   waits once more for what it issued and returns.
#include "bulk_copy.cuh"
#include "device_access.cuh"
#include "h3rr_internal.h"

namespace h3rr {

// Count of bounded waits that expired in the bulk kernel (per device).
__device__ unsigned int g_bulk_wait_timeouts = 0;

namespace {

// ---------------------------------------------------------------------------
// vector kernels
// ---------------------------------------------------------------------------
template <bool kSeqToHead, int VW, int NT, int VPT, int ROWS, bool kLayout = false>
__global__ void __launch_bounds__(NT) relayout_vec_kernel(const __grid_constant__ RelayoutArgs a)
{
    constexpr int kUnits = VW / kVecBytes;  // 16-byte units per vector
    const int32_t row_v = a.row_vecs / kUnits;
    const int32_t head_v = a.head_vecs / kUnits;
    // Head-side placement of this thread's columns (same for every row).
    char* hbase[VPT];
    int32_t hstride[VPT];
    bool live[VPT];
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        const int32_t c = threadIdx.x + k * NT;
        live[k] = c < row_v;
        const int32_t cc = live[k] ? c : 0;
        const int32_t h = cc / head_v;
        const int32_t within = cc - h * head_v;
        const int32_t j = split_owner(h, a.hq, a.hm);
        const int32_t hj = a.hq + (j < a.hm ? 1 : 0);
        const int32_t hl = h - split_start(j, a.hq, a.hm);
        hbase[k] = a.head[j] + (int64_t(hl) * head_v + within) * VW;
        hstride[k] = hj * head_v * VW;
    }
    const int64_t seq_row_bytes = int64_t(row_v) * VW;
    // Programmatic launch: the previous kernel in the stream must be complete
    // before the first memory access, unless this launch is independent of
    // it (a later plane of a chunked call), which waits at its end instead.
    if (!a.wait_late)
        pdl_wait_prerequisites();
    pdl_allow_dependents();

    for (int64_t i0 = int64_t(blockIdx.x) * ROWS; i0 < a.rows; i0 += int64_t(gridDim.x) * ROWS) {
        char* sptr[ROWS];
        int64_t g[ROWS];
        bool rv[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            rv[r] = i0 + r < a.rows;
            const int32_t ii = int32_t(rv[r] ? i0 + r : i0);
            const int32_t u = ii / a.nplanes;  // token unit of the launch
            const int32_t p = a.plane0 + (ii - u * a.nplanes);
            const ChunkToken k = chunk_token(u, a.cq, a.cm, a.t0, a.tq, a.tm);
            const int32_t s = k.s, tl = k.tl, t = k.t;
            if constexpr (kLayout) {
                // plane-major sides: plane p is a contiguous block of T (or T_s) rows
                const int32_t ts_len = a.tq + (s < a.tm ? 1 : 0);
                g[r] = a.head_pm ? int64_t(p) * a.T + t : int64_t(t) * a.P + p;
                const int64_t srow = a.seq_pm ? int64_t(p) * ts_len + tl : int64_t(tl) * a.P + p;
                sptr[r] = a.seq[s] + srow * seq_row_bytes + int64_t(threadIdx.x) * VW;
            } else {
                g[r] = int64_t(t) * a.P + p;
                sptr[r] = a.seq[s] + (int64_t(tl) * a.P + p) * seq_row_bytes + int64_t(threadIdx.x) * VW;
            }
        }
        Vec<VW> v[ROWS][VPT];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                if (rv[r] && live[k]) {
                    const char* src = kSeqToHead ? sptr[r] + k * NT * VW : hbase[k] + g[r] * hstride[k];
                    ld_stream(v[r][k], src);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                if (rv[r] && live[k]) {
                    char* dst = kSeqToHead ? hbase[k] + g[r] * hstride[k] : sptr[r] + k * NT * VW;
                    st_stream(dst, v[r][k]);
                }
            }
        }
    }
    pdl_wait_at_end(a.wait_late);
}

// Any row width: one row per CTA iteration, head-side placement per vector.
constexpr int kGenericThreads = 128;

template <bool kSeqToHead, bool kLayout = false>
__global__ void __launch_bounds__(kGenericThreads) relayout_generic_kernel(const __grid_constant__ RelayoutArgs a)
{
    const int64_t seq_row_bytes = int64_t(a.row_vecs) * kVecBytes;
    if (!a.wait_late)
        pdl_wait_prerequisites();
    pdl_allow_dependents();
    for (int64_t i64 = blockIdx.x; i64 < a.rows; i64 += gridDim.x) {
        const int32_t i = int32_t(i64);
        const int32_t u = i / a.nplanes;  // token unit of the launch
        const int32_t p = a.plane0 + (i - u * a.nplanes);
        const ChunkToken k = chunk_token(u, a.cq, a.cm, a.t0, a.tq, a.tm);
        const int32_t s = k.s, tl = k.tl, t = k.t;
        int64_t g = int64_t(t) * a.P + p;
        int64_t srow_index = int64_t(tl) * a.P + p;
        if constexpr (kLayout) {
            const int32_t ts_len = a.tq + (s < a.tm ? 1 : 0);
            if (a.head_pm)
                g = int64_t(p) * a.T + t;
            if (a.seq_pm)
                srow_index = int64_t(p) * ts_len + tl;
        }
        char* srow = a.seq[s] + srow_index * seq_row_bytes;
        for (int32_t c = threadIdx.x; c < a.row_vecs; c += kGenericThreads) {
            const int32_t h = c / a.head_vecs;
            const int32_t within = c - h * a.head_vecs;
            const int32_t j = split_owner(h, a.hq, a.hm);
            const int32_t hj = a.hq + (j < a.hm ? 1 : 0);
            const int32_t hl = h - split_start(j, a.hq, a.hm);
            char* hp = a.head[j] + ((g * hj + hl) * a.head_vecs + within) * kVecBytes;
            char* sp = srow + int64_t(c) * kVecBytes;
            Vec<16> v;
            if (kSeqToHead) {
                ld_stream(v, sp);
                st_stream(hp, v);
            } else {
                ld_stream(v, hp);
                st_stream(sp, v);
            }
        }
    }
    pdl_wait_at_end(a.wait_late);
}

// ---------------------------------------------------------------------------
// bulk kernel (tensor memory accelerator, 1-D bulk copies, no multicast)
// ---------------------------------------------------------------------------
// A CTA is one warp and moves kBulkRows consecutive rows; lane r drives row
// r on its own: bulk loads into its shared-memory stage (the whole sequence-
// side row, or the row's W head-side runs), a wait on its own mbarrier, bulk
// stores out of the stage.  CTAs are not persistent: one per kBulkRows rows,
// handed out by the block scheduler as SMs free up.  On B200 a persistent
// ring (one thread per CTA streaming rows through 4-14 stages, grid = the
// SM count times the CTAs that fit) ran 9-13 % slower on every full-size
// workload, the same lockstep effect that made the vector kernels one CTA
// per row; 1-8 rows per CTA measured within 1.5 % of each other, 4 best.
// The copies carry no L2 cache hint: evict-first loads cost 1-2 %.
constexpr int kBulkRows = 4;
constexpr int kBulkBarrierBytes = 128;  // the lanes' mbarriers, padded to keep stages aligned

template <bool kSeqToHead>
__global__ void __launch_bounds__(32) relayout_bulk_kernel(const __grid_constant__ RelayoutArgs a)
{
    static_assert(kBulkRows <= 32 && kBulkRows * 8 <= kBulkBarrierBytes, "bulk CTA shape");
    extern __shared__ __align__(128) unsigned char smem[];
    const int lane = int(threadIdx.x);
    const bool driver = lane < kBulkRows;
    const uint32_t row_bytes = uint32_t(a.row_vecs) * kVecBytes;
    const uint32_t head_bytes = uint32_t(a.head_vecs) * kVecBytes;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem) + (driver ? lane : 0);
    unsigned char* stage = smem + kBulkBarrierBytes + size_t(driver ? lane : 0) * row_bytes;
    if (driver) {
        mbar_init(bar, 1);
        mbar_fence_init();
    }
    // Programmatic launch, as in the vector kernels: wait for the previous
    // kernel before the first global access unless this launch is a later,
    // independent plane of a chunked call, which waits at its end instead.
    if (!a.wait_late)
        pdl_wait_prerequisites();
    pdl_allow_dependents();

    if (driver) {
        const int64_t stride = int64_t(gridDim.x) * kBulkRows;
        uint32_t parity = 0;
        for (int64_t i = int64_t(blockIdx.x) * kBulkRows + lane; i < a.rows; i += stride) {
            if (i >= stride)
                bulk_wait_read<0>();  // a later row: the stage's previous stores have read it
            const int32_t u = int32_t(i / a.nplanes);  // token unit of the launch
            const int32_t p = a.plane0 + int32_t(i - int64_t(u) * a.nplanes);
            const ChunkToken k = chunk_token(u, a.cq, a.cm, a.t0, a.tq, a.tm);
            char* seq_row = a.seq[k.s] + (int64_t(k.tl) * a.P + p) * row_bytes;
            const int64_t g = int64_t(k.t) * a.P + p;  // head-side row
            mbar_arrive_expect_tx(bar, row_bytes);
            if (kSeqToHead) {
                bulk_load(stage, seq_row, row_bytes, bar);
            } else {
                uint32_t off = 0;
                for (int j = 0; j < a.W; ++j) {
                    const uint32_t run = uint32_t(a.hq + (j < a.hm ? 1 : 0)) * head_bytes;
                    bulk_load(stage + off, a.head[j] + g * run, run, bar);
                    off += run;
                }
            }
            if (!mbar_wait(bar, parity)) {
                atomicAdd(&g_bulk_wait_timeouts, 1u);
                mbar_wait(bar, parity);  // give the copies in flight one more bounded wait
                break;
            }
            parity ^= 1u;
            if (kSeqToHead) {
                uint32_t off = 0;
                for (int j = 0; j < a.W; ++j) {
                    const uint32_t run = uint32_t(a.hq + (j < a.hm ? 1 : 0)) * head_bytes;
                    bulk_store(a.head[j] + g * run, stage + off, run);
                    off += run;
                }
            } else {
                bulk_store(seq_row, stage, row_bytes);
            }
            bulk_commit();
        }
        bulk_wait_all();
    }
    pdl_wait_at_end(a.wait_late);
}

// ---------------------------------------------------------------------------
// one rank's share of sequence->head (one rank per GPU)
// ---------------------------------------------------------------------------
// Row (t, p) of this rank's head-side buffer is one contiguous run of H_k
// heads cut from the sequence-side row (t, p) of token t's rank, which may
// live on another GPU.  A run is short (2.5 KB for 10 heads of 128), and one
// CTA per run left the kernel bound by the rate at which the GPU starts
// CTAs, so a CTA takes ROWS consecutive runs laid end to end: thread i owns
// vectors i, i+NT, ... of the group (a fixed run and column per slot), the
// group's row addresses sit in shared memory, and all loads precede the
// stores.  Needs ROWS * run <= NT * MAXV vectors.
template <int VW, int NT, int ROWS, int MAXV>
__global__ void __launch_bounds__(NT) pull_seq_to_head_kernel(const __grid_constant__ PullArgs a)
{
    constexpr int kUnits = VW / kVecBytes;
    const int32_t run_v = a.run_vecs / kUnits;
    __shared__ const char* s_src[ROWS];
    __shared__ char* s_dst[ROWS];
    int32_t slot_row[MAXV];
    int32_t slot_col[MAXV];
#pragma unroll
    for (int k = 0; k < MAXV; ++k) {
        const int32_t c = int32_t(threadIdx.x) + k * NT;
        slot_row[k] = c / run_v;  // >= ROWS: no vector in this slot
        slot_col[k] = c - slot_row[k] * run_v;
    }
    if (!a.wait_late)
        pdl_wait_prerequisites();
    pdl_allow_dependents();
    for (int64_t i0 = int64_t(blockIdx.x) * ROWS; i0 < a.rows; i0 += int64_t(gridDim.x) * ROWS) {
        if (threadIdx.x < ROWS) {
            const int64_t i64 = i0 + threadIdx.x;
            const char* src = nullptr;
            char* dst = nullptr;
            if (i64 < a.rows) {
                const int32_t i = int32_t(i64);
                const int32_t u = i / a.nplanes;  // token unit of the launch
                const int32_t p = a.plane0 + (i - u * a.nplanes);
                const ChunkToken k = chunk_token(u, a.cq, a.cm, a.t0, a.tq, a.tm);
                src = a.src[k.s] + ((int64_t(k.tl) * a.P + p) * a.row_vecs + a.col0_vecs) * kVecBytes;
                dst = a.dst + (int64_t(k.t) * a.P + p) * a.run_vecs * kVecBytes;
            }
            s_src[threadIdx.x] = src;
            s_dst[threadIdx.x] = dst;
        }
        __syncthreads();
        Vec<VW> v[MAXV];
#pragma unroll
        for (int k = 0; k < MAXV; ++k) {
            if (slot_row[k] < ROWS) {
                const char* src = s_src[slot_row[k]];
                if (src)
                    ld_stream(v[k], src + int64_t(slot_col[k]) * VW);
            }
        }
#pragma unroll
        for (int k = 0; k < MAXV; ++k) {
            if (slot_row[k] < ROWS) {
                char* dst = s_dst[slot_row[k]];
                if (dst)
                    st_stream(dst + int64_t(slot_col[k]) * VW, v[k]);
            }
        }
        __syncthreads();  // the next group overwrites the row table
    }
    pdl_wait_at_end(a.wait_late);
}

// Runs longer than one CTA's slots (NT * MAXV vectors): one run per CTA
// iteration, in passes of NT * MAXV vectors.
template <int VW, int NT, int MAXV>
__global__ void __launch_bounds__(NT) pull_seq_to_head_long_kernel(const __grid_constant__ PullArgs a)
{
    constexpr int kUnits = VW / kVecBytes;
    const int32_t run_v = a.run_vecs / kUnits;
    if (!a.wait_late)
        pdl_wait_prerequisites();
    pdl_allow_dependents();
    for (int64_t i64 = blockIdx.x; i64 < a.rows; i64 += gridDim.x) {
        const int32_t i = int32_t(i64);
        const int32_t u = i / a.nplanes;  // token unit of the launch
        const int32_t p = a.plane0 + (i - u * a.nplanes);
        const ChunkToken k = chunk_token(u, a.cq, a.cm, a.t0, a.tq, a.tm);
        const char* src = a.src[k.s] + ((int64_t(k.tl) * a.P + p) * a.row_vecs + a.col0_vecs) * kVecBytes;
        char* dst = a.dst + (int64_t(k.t) * a.P + p) * a.run_vecs * kVecBytes;
        for (int32_t c0 = 0; c0 < run_v; c0 += MAXV * NT) {
            Vec<VW> v[MAXV];
#pragma unroll
            for (int k = 0; k < MAXV; ++k) {
                const int32_t c = c0 + int32_t(threadIdx.x) + k * NT;
                if (c < run_v)
                    ld_stream(v[k], src + int64_t(c) * VW);
            }
#pragma unroll
            for (int k = 0; k < MAXV; ++k) {
                const int32_t c = c0 + int32_t(threadIdx.x) + k * NT;
                if (c < run_v)
                    st_stream(dst + int64_t(c) * VW, v[k]);
            }
        }
    }
    pdl_wait_at_end(a.wait_late);
}

// ---------------------------------------------------------------------------
// dispatch
// ---------------------------------------------------------------------------
struct KernelChoice {
    const void* fn = nullptr;
    int threads = 0;
    int rows_per_cta_iter = 1;
    size_t smem = 0;
    int variant = H3_VARIANT_NONE;
};

// Smallest instantiated vectors-per-thread count (at most MAXV) covering `need`.
template <bool S2H, int VW, int NT, int ROWS, int MAXV, bool LAYOUT = false>
bool pick_vec(int need, KernelChoice* kc)
{
#define H3RR_VPT(V)                                                              \
    if constexpr (V <= MAXV) {                                                   \
        if (need <= V) {                                                         \
            kc->fn = (const void*)relayout_vec_kernel<S2H, VW, NT, V, ROWS, LAYOUT>; \
            kc->threads = NT;                                                    \
            kc->rows_per_cta_iter = ROWS;                                        \
            kc->variant = H3_VARIANT_VECTOR;                                     \
            return true;                                                         \
        }                                                                        \
    }
    H3RR_VPT(1)
    H3RR_VPT(2)
    H3RR_VPT(4)
    H3RR_VPT(7)
    H3RR_VPT(8)
    H3RR_VPT(14)
    H3RR_VPT(16)
#undef H3RR_VPT
    return false;
}

// Vector kernel shapes measured fastest on B200 for H3 rows (14,336 bytes =
// 448 vectors of 32 bytes) with one CTA per row unit: 128 threads, 32-byte
// vectors, 4 per thread, two rows per CTA for sequence->head (120 registers)
// and one for head->sequence (72 registers).  They beat 64 threads x 7 x 2
// rows (seq->head) and one warp x 14 (head->seq) by 1-2 % on every workload;
// those had won under persistent grids.  Rows wider than 16 KB fall back to
// 16-byte vectors with 128 threads, then to the generic kernel.
template <bool S2H, bool LAYOUT = false>
void choose_vec(const RelayoutArgs& a, bool wide_ok, KernelChoice* kc)
{
    if (wide_ok) {
        const int row32 = a.row_vecs / 2;
        const bool ok = S2H ? pick_vec<true, 32, 128, 2, 4, LAYOUT>((row32 + 127) / 128, kc)
                            : pick_vec<false, 32, 128, 1, 4, LAYOUT>((row32 + 127) / 128, kc);
        if (ok)
            return;
    }
    if (pick_vec<S2H, 16, 128, 1, 16, LAYOUT>((a.row_vecs + 127) / 128, kc))
        return;
    kc->fn = (const void*)relayout_generic_kernel<S2H, LAYOUT>;
    kc->threads = kGenericThreads;
    kc->rows_per_cta_iter = 1;
    kc->variant = H3_VARIANT_VECTOR;
}

bool choose_bulk(bool s2h, const RelayoutArgs& a, int device, KernelChoice* kc)
{
    const size_t row_bytes = size_t(a.row_vecs) * kVecBytes;
    const size_t smem = kBulkBarrierBytes + kBulkRows * row_bytes;
    int max_smem = 0;
    if (cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) != cudaSuccess)
        return false;
    if (smem > size_t(max_smem))
        return false;
    kc->fn = s2h ? (const void*)relayout_bulk_kernel<true> : (const void*)relayout_bulk_kernel<false>;
    kc->threads = 32;
    kc->rows_per_cta_iter = kBulkRows;
    kc->smem = smem;
    kc->variant = H3_VARIANT_BULK;
    return true;
}

bool wide_vectors_ok(const RelayoutArgs& a)
{
    if ((a.head_vecs % 2) != 0)
        return false;
    for (int r = 0; r < a.W; ++r)
        if ((reinterpret_cast<uintptr_t>(a.seq[r]) & 31u) || (reinterpret_cast<uintptr_t>(a.head[r]) & 31u))
            return false;
    return true;
}

}  // namespace

bool relayout_bulk_fits(const RelayoutArgs& a, int device)
{
    KernelChoice kc;
    return choose_bulk(true, a, device, &kc);
}

cudaError_t launch_relayout(bool seq_to_head, const RelayoutArgs& a, int variant, int ctas_per_sm,
                            cudaStream_t stream, LaunchShape* shape, bool layout, bool programmatic)
{
    int device = 0;
    const int sms = current_sm_count(&device);
    if (sms <= 0)
        return cudaErrorNoDevice;
    KernelChoice kc;
    // Default: the vector kernels; the bulk kernel only when asked for.
    const bool want_bulk = variant == H3_VARIANT_BULK;
    bool bulk = false;
    if (want_bulk)
        bulk = choose_bulk(seq_to_head, a, device, &kc);
    if (variant == H3_VARIANT_BULK && !bulk)
        return cudaErrorInvalidConfiguration;
    if (bulk && layout)
        return cudaErrorInvalidConfiguration;  // the bulk kernel moves token-major rows only
    if (!bulk) {
        if (layout) {
            if (seq_to_head)
                choose_vec<true, true>(a, wide_vectors_ok(a), &kc);
            else
                choose_vec<false, true>(a, wide_vectors_ok(a), &kc);
        } else if (seq_to_head) {
            choose_vec<true>(a, wide_vectors_ok(a), &kc);
        } else {
            choose_vec<false>(a, wide_vectors_ok(a), &kc);
        }
    } else {
        const cudaError_t err = allow_dynamic_smem(kc.fn, kc.smem, device);
        if (err != cudaSuccess)
            return err;
    }
    // Grid: every kernel launches one CTA per row, row pair or row group by
    // default and lets the hardware schedule them.  On B200 that measured
    // 2-13 % faster than any persistent grid-stride launch (a multiple of the
    // SM count): CTAs marching through the rows in lockstep resonated with the
    // DRAM mapping at some grid sizes.  ctas_per_sm > 0 caps the grid at that
    // many CTAs per SM (grid-stride).
    const int64_t needed = (int64_t(a.rows) + kc.rows_per_cta_iter - 1) / kc.rows_per_cta_iter;
    int64_t grid = needed;
    if (ctas_per_sm > 0)
        grid = int64_t(sms) * ctas_per_sm;
    if (grid > needed)
        grid = needed;
    if (grid < 1)
        grid = 1;
    if (shape) {
        shape->grid = int(grid);
        shape->block = kc.threads;
        shape->variant = kc.variant;
    }
    // Every relayout kernel follows the griddepcontrol protocol.
    void* params[] = {const_cast<RelayoutArgs*>(&a)};
    return launch_kernel(kc.fn, grid, kc.threads, kc.smem, stream, params, programmatic);
}

namespace {

constexpr int kPullThreads = 128;
constexpr int kPullSlots = 8;  // vectors per thread per group

// The pull kernel for `rows_per_cta` runs per CTA (2, 4 or 8; one run per
// CTA goes to the long-run kernel).
template <int VW>
const void* pull_kernel(int rows_per_cta)
{
    switch (rows_per_cta) {
        case 8: return (const void*)pull_seq_to_head_kernel<VW, kPullThreads, 8, kPullSlots>;
        case 4: return (const void*)pull_seq_to_head_kernel<VW, kPullThreads, 4, kPullSlots>;
        default: return (const void*)pull_seq_to_head_kernel<VW, kPullThreads, 2, kPullSlots>;
    }
}

}  // namespace

cudaError_t launch_pull_seq_to_head(const PullArgs& a, int ctas_per_sm, cudaStream_t stream,
                                    LaunchShape* shape, bool programmatic)
{
    int device = 0;
    const int sms = current_sm_count(&device);
    if (sms <= 0)
        return cudaErrorNoDevice;
    // 32-byte vectors when the run, its start and every buffer allow them.
    bool wide = (a.row_vecs % 2) == 0 && (a.run_vecs % 2) == 0 && (a.col0_vecs % 2) == 0 &&
                (reinterpret_cast<uintptr_t>(a.dst) & 31u) == 0;
    for (int r = 0; wide && r < a.W; ++r)
        wide = (reinterpret_cast<uintptr_t>(a.src[r]) & 31u) == 0;
    const int64_t run_v = wide ? a.run_vecs / 2 : a.run_vecs;
    const int64_t slots = int64_t(kPullThreads) * kPullSlots;
    // As many runs per CTA (up to 8) as fill the CTA's slots.
    int rows_per_cta = 8;
    while (rows_per_cta > 1 && rows_per_cta * run_v > slots)
        rows_per_cta /= 2;
    if (run_v > slots)
        rows_per_cta = 1;
    const void* fn;
    if (rows_per_cta == 1)
        fn = wide ? (const void*)pull_seq_to_head_long_kernel<32, kPullThreads, kPullSlots>
                  : (const void*)pull_seq_to_head_long_kernel<16, kPullThreads, kPullSlots>;
    else
        fn = wide ? pull_kernel<32>(rows_per_cta) : pull_kernel<16>(rows_per_cta);
    // One CTA per group of runs, as the other register kernels.
    int64_t grid = (int64_t(a.rows) + rows_per_cta - 1) / rows_per_cta;
    if (ctas_per_sm > 0 && int64_t(sms) * ctas_per_sm < grid)
        grid = int64_t(sms) * ctas_per_sm;
    if (grid < 1)
        grid = 1;
    if (shape) {
        shape->grid = int(grid);
        shape->block = kPullThreads;
        shape->variant = H3_VARIANT_VECTOR;
    }
    void* params[] = {const_cast<PullArgs*>(&a)};
    return launch_kernel(fn, grid, kPullThreads, 0, stream, params, programmatic);
}

cudaError_t read_bulk_wait_timeouts(unsigned int* count, bool reset, cudaStream_t stream)
{
    cudaError_t err = cudaMemcpyFromSymbolAsync(count, g_bulk_wait_timeouts, sizeof(unsigned int), 0,
                                                cudaMemcpyDeviceToHost, stream);
    if (err == cudaSuccess)
        err = cudaStreamSynchronize(stream);
    if (err == cudaSuccess && reset) {
        static const unsigned int zero = 0;
        err = cudaMemcpyToSymbolAsync(g_bulk_wait_timeouts, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice,
                                      stream);
        if (err == cudaSuccess)
            err = cudaStreamSynchronize(stream);
    }
    return err;
}

}  // namespace h3rr
