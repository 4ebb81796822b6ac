// Staged ("registered window") relayouts for sm_100a.
//
// FastVideo PR #1807, "Problem and behavior": the GB200 transport moves one
// batch plane at a time through a registered window of at most 896,000,000
// bytes instead of exceeding a 1 GiB cap.  This mode reproduces that data
// path on one GPU: every chunk (one plane, a run of tokens) is first packed
// into a caller-provided window buffer, laid out head-rank-major, and then
// unpacked into the destination buffers.  Each byte therefore crosses HBM
// twice; the mode exists for callers that must stage through a bounded buffer
// (and to split planes larger than the window into token chunks), not for
// speed.
//
// Window layout of a chunk of n tokens [t0, t0 + n) of plane p: head-side
// rank j's block [n, H_j, D] at byte offset n * hs_j * D * 2, blocks in rank
// order, n * H * D * 2 bytes in all.
//
// Kernels, two launches per chunk:
//   row kernel     sequence-side rows <-> window blocks (the relayout proper):
//                  one CTA per token row; each thread owns fixed columns of
//                  the row whose window placement it computes once.
//   block kernel   window blocks <-> head-side rows of plane p (a strided copy
//                  per rank): up to 8 head runs per CTA, their addresses in
//                  shared memory (one 2.5 KB run per CTA was bound by the rate
//                  at which CTAs start).
// Both move 32-byte vectors when every buffer and run allows, else 16-byte
// ones; rows or runs too wide for those shapes take the plain per-vector
// kernels (staged_row_kernel, window_block_kernel).
// seq->head = row kernel then block kernel; head->seq = block then row.
//
// Every launch uses programmatic dependent launch: its CTAs may be scheduled
// while the previous launch drains, and each waits for that launch to
// complete (griddepcontrol.wait) before its first memory access.  Each
// launch reads what the previous one wrote, or overwrites the window it
// read, so nothing runs early; what is saved is the launch latency between
// chunks, which bounds small windows.
#include "device_access.cuh"
#include "h3rr_internal.h"

namespace h3rr {
namespace {

constexpr int kThreads = 128;
constexpr int64_t kMaxGrid = (int64_t(1) << 31) - 1;

// Sequence-side rows t0..t0+n-1 of plane p <-> the chunk's window blocks.
template <bool kToWindow>
__global__ void __launch_bounds__(kThreads) staged_row_kernel(const __grid_constant__ StagedArgs a)
{
    pdl_wait_prerequisites();
    pdl_allow_dependents();
    const int64_t row_bytes = int64_t(a.row_vecs) * kVecBytes;
    for (int64_t i = blockIdx.x; i < a.n; i += gridDim.x) {
        const int32_t t = a.t0 + int32_t(i);
        const int32_t s = split_owner(t, a.tq, a.tm);
        const int32_t tl = t - split_start(s, a.tq, a.tm);
        char* srow = a.seq[s] + (int64_t(tl) * a.P + a.p) * row_bytes;
        for (int32_t c = threadIdx.x; c < a.row_vecs; c += kThreads) {
            const int32_t h = c / a.head_vecs;
            const int32_t within = c - h * a.head_vecs;
            const int32_t j = split_owner(h, a.hq, a.hm);
            const int32_t hs = split_start(j, a.hq, a.hm);
            const int32_t hj = a.hq + (j < a.hm ? 1 : 0);
            // block j starts at n * hs_j heads; token i of the chunk, head h - hs_j
            char* wp = a.window +
                       ((int64_t(a.n) * hs + i * hj + (h - hs)) * a.head_vecs + within) * kVecBytes;
            char* sp = srow + int64_t(c) * kVecBytes;
            Vec<16> v;
            if (kToWindow) {
                ld_stream(v, sp);
                st_plain(wp, v);
            } else {
                // The window is written and read back within one call: coherent loads.
                ld_plain(v, wp);
                st_plain(sp, v);
            }
        }
    }
}

// Window block rows <-> head-side rows (t, p), one (rank, token) run per CTA iteration.
template <bool kToHead>
__global__ void __launch_bounds__(kThreads) window_block_kernel(const __grid_constant__ StagedArgs a)
{
    pdl_wait_prerequisites();
    pdl_allow_dependents();
    const int64_t runs = int64_t(a.W) * a.n;
    for (int64_t r = blockIdx.x; r < runs; r += gridDim.x) {
        const int32_t j = int32_t(r / a.n);
        const int64_t i = r - int64_t(j) * a.n;
        const int32_t hs = split_start(j, a.hq, a.hm);
        const int32_t hj = a.hq + (j < a.hm ? 1 : 0);
        const int32_t run_vecs = hj * a.head_vecs;
        char* wrow = a.window + (int64_t(a.n) * hs + i * hj) * a.head_vecs * kVecBytes;
        char* hrow = a.head[j] + ((int64_t(a.t0) + i) * a.P + a.p) * run_vecs * kVecBytes;
        for (int32_t c = threadIdx.x; c < run_vecs; c += kThreads) {
            Vec<16> v;
            if (kToHead) {
                ld_plain(v, wrow + int64_t(c) * kVecBytes);
                st_plain(hrow + int64_t(c) * kVecBytes, v);
            } else {
                ld_stream(v, hrow + int64_t(c) * kVecBytes);
                st_plain(wrow + int64_t(c) * kVecBytes, v);
            }
        }
    }
}


// Row kernel with per-thread window placement: column c of the sequence-side
// row (head h, vector within) goes to rank j's block at n*hs_j heads, token
// i at i*H_j heads, head h - hs_j.  VPT vectors per thread, all loads of a
// row before its stores.
template <bool kToWindow, int VW, int NT, int VPT>
__global__ void __launch_bounds__(NT) staged_row_vec_kernel(const __grid_constant__ StagedArgs a)
{
    constexpr int kUnits = VW / kVecBytes;
    const int32_t row_v = a.row_vecs / kUnits;
    const int32_t head_v = a.head_vecs / kUnits;
    int64_t wbase[VPT];
    int64_t wstride[VPT];
    bool live[VPT];
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        const int32_t c = int32_t(threadIdx.x) + k * NT;
        live[k] = c < row_v;
        const int32_t cc = live[k] ? c : 0;
        const int32_t h = cc / head_v;
        const int32_t within = cc - h * head_v;
        const int32_t j = split_owner(h, a.hq, a.hm);
        const int32_t hs = split_start(j, a.hq, a.hm);
        const int32_t hj = a.hq + (j < a.hm ? 1 : 0);
        wbase[k] = ((int64_t(a.n) * hs + (h - hs)) * head_v + within) * VW;
        wstride[k] = int64_t(hj) * head_v * VW;
    }
    pdl_wait_prerequisites();
    pdl_allow_dependents();
    const int64_t row_bytes = int64_t(row_v) * VW;
    for (int64_t i = blockIdx.x; i < a.n; i += gridDim.x) {
        const int32_t t = a.t0 + int32_t(i);
        const int32_t s = split_owner(t, a.tq, a.tm);
        const int32_t tl = t - split_start(s, a.tq, a.tm);
        char* srow = a.seq[s] + (int64_t(tl) * a.P + a.p) * row_bytes + int64_t(threadIdx.x) * VW;
        Vec<VW> v[VPT];
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            if (!live[k])
                continue;
            if (kToWindow)
                ld_stream(v[k], srow + int64_t(k) * NT * VW);
            else  // the window was written earlier in this call: coherent loads
                ld_plain(v[k], a.window + wbase[k] + i * wstride[k]);
        }
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            if (!live[k])
                continue;
            if (kToWindow)
                st_plain(a.window + wbase[k] + i * wstride[k], v[k]);
            else
                st_stream(srow + int64_t(k) * NT * VW, v[k]);
        }
    }
}

// Block kernel: CTA (x, y) copies head runs of tokens [x*ROWS, x*ROWS+ROWS)
// of rank j = y between the window block and the head-side rows; thread i
// owns vectors i, i+NT, ... of the group's runs laid end to end.  Needs
// ROWS * run <= NT * MAXV vectors.
template <bool kToHead, int VW, int NT, int ROWS, int MAXV>
__global__ void __launch_bounds__(NT) window_block_vec_kernel(const __grid_constant__ StagedArgs a)
{
    constexpr int kUnits = VW / kVecBytes;
    const int32_t j = int32_t(blockIdx.y);
    const int32_t hs = split_start(j, a.hq, a.hm);
    const int32_t hj = a.hq + (j < a.hm ? 1 : 0);
    const int32_t run_v = hj * (a.head_vecs / kUnits);
    __shared__ char* s_win[ROWS];
    __shared__ char* s_head[ROWS];
    int32_t slot_row[MAXV];
    int32_t slot_col[MAXV];
#pragma unroll
    for (int k = 0; k < MAXV; ++k) {
        const int32_t c = int32_t(threadIdx.x) + k * NT;
        slot_row[k] = c / run_v;  // >= ROWS: no vector in this slot
        slot_col[k] = c - slot_row[k] * run_v;
    }
    pdl_wait_prerequisites();
    pdl_allow_dependents();
    for (int64_t i0 = int64_t(blockIdx.x) * ROWS; i0 < a.n; i0 += int64_t(gridDim.x) * ROWS) {
        if (threadIdx.x < ROWS) {
            const int64_t i = i0 + threadIdx.x;
            char* w = nullptr;
            char* h = nullptr;
            if (i < a.n) {
                w = a.window + (int64_t(a.n) * hs + i * hj) * a.head_vecs * kVecBytes;
                h = a.head[j] + ((int64_t(a.t0) + i) * a.P + a.p) * int64_t(run_v) * VW;
            }
            s_win[threadIdx.x] = w;
            s_head[threadIdx.x] = h;
        }
        __syncthreads();
        Vec<VW> v[MAXV];
#pragma unroll
        for (int k = 0; k < MAXV; ++k) {
            if (slot_row[k] >= ROWS || !s_win[slot_row[k]])
                continue;
            const int64_t off = int64_t(slot_col[k]) * VW;
            if (kToHead)
                ld_plain(v[k], s_win[slot_row[k]] + off);
            else
                ld_stream(v[k], s_head[slot_row[k]] + off);
        }
#pragma unroll
        for (int k = 0; k < MAXV; ++k) {
            if (slot_row[k] >= ROWS || !s_win[slot_row[k]])
                continue;
            const int64_t off = int64_t(slot_col[k]) * VW;
            if (kToHead)
                st_stream(s_head[slot_row[k]] + off, v[k]);
            else
                st_plain(s_win[slot_row[k]] + off, v[k]);
        }
        __syncthreads();  // the next group overwrites the row table
    }
}

}  // namespace

namespace {

constexpr int kVecThreads = 128;
constexpr int kBlockSlots = 8;  // vectors per thread per group in the block kernel

struct StagedKernel {
    const void* fn = nullptr;
    int64_t grid_x = 0;
    int grid_y = 1;
    int threads = kThreads;
};

// The row kernel for `need` vectors per thread (VPT 1, 2, 4, 8 or 16).
template <bool kToWindow, int VW>
const void* row_vec_kernel(int need)
{
    if (need <= 1) return (const void*)staged_row_vec_kernel<kToWindow, VW, kVecThreads, 1>;
    if (need <= 2) return (const void*)staged_row_vec_kernel<kToWindow, VW, kVecThreads, 2>;
    if (need <= 4) return (const void*)staged_row_vec_kernel<kToWindow, VW, kVecThreads, 4>;
    if (need <= 8) return (const void*)staged_row_vec_kernel<kToWindow, VW, kVecThreads, 8>;
    if (need <= 16) return (const void*)staged_row_vec_kernel<kToWindow, VW, kVecThreads, 16>;
    return nullptr;
}

template <bool kToHead, int VW>
const void* block_vec_kernel(int rows)
{
    switch (rows) {
        case 8: return (const void*)window_block_vec_kernel<kToHead, VW, kVecThreads, 8, kBlockSlots>;
        case 4: return (const void*)window_block_vec_kernel<kToHead, VW, kVecThreads, 4, kBlockSlots>;
        case 2: return (const void*)window_block_vec_kernel<kToHead, VW, kVecThreads, 2, kBlockSlots>;
        default: return (const void*)window_block_vec_kernel<kToHead, VW, kVecThreads, 1, kBlockSlots>;
    }
}

bool wide_ok(const StagedArgs& a)
{
    if ((a.head_vecs % 2) != 0 || (reinterpret_cast<uintptr_t>(a.window) & 31u))
        return false;
    for (int r = 0; r < a.W; ++r)
        if ((reinterpret_cast<uintptr_t>(a.seq[r]) & 31u) || (reinterpret_cast<uintptr_t>(a.head[r]) & 31u))
            return false;
    return true;
}

template <bool kToWindow>
StagedKernel pick_row(const StagedArgs& a, bool wide)
{
    StagedKernel k;
    const int units = wide ? 2 : 1;
    const int row_v = a.row_vecs / units;
    const int need = (row_v + kVecThreads - 1) / kVecThreads;
    k.fn = wide ? row_vec_kernel<kToWindow, 32>(need) : row_vec_kernel<kToWindow, 16>(need);
    k.threads = kVecThreads;
    if (!k.fn) {
        k.fn = (const void*)staged_row_kernel<kToWindow>;
        k.threads = kThreads;
    }
    k.grid_x = a.n;
    return k;
}

template <bool kToHead>
StagedKernel pick_block(const StagedArgs& a, bool wide)
{
    StagedKernel k;
    const int units = wide ? 2 : 1;
    const int64_t longest_run = int64_t(a.hq + (a.hm > 0 ? 1 : 0)) * (a.head_vecs / units);
    const int64_t slots = int64_t(kVecThreads) * kBlockSlots;
    if (longest_run > slots) {
        k.fn = (const void*)window_block_kernel<kToHead>;
        k.threads = kThreads;
        k.grid_x = int64_t(a.W) * a.n;
        return k;
    }
    int rows = 8;
    while (rows > 1 && rows * longest_run > slots)
        rows /= 2;
    k.fn = wide ? block_vec_kernel<kToHead, 32>(rows) : block_vec_kernel<kToHead, 16>(rows);
    k.threads = kVecThreads;
    k.grid_x = (int64_t(a.n) + rows - 1) / rows;
    k.grid_y = a.W;
    return k;
}

cudaError_t launch_staged(const StagedKernel& k, const StagedArgs& a, cudaStream_t stream,
                          int* grid_out)
{
    int64_t gx = k.grid_x < kMaxGrid ? k.grid_x : kMaxGrid;
    if (gx < 1)
        gx = 1;
    *grid_out = int(gx);
    void* params[] = {const_cast<StagedArgs*>(&a)};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(gx), unsigned(k.grid_y));
    cfg.blockDim = dim3(unsigned(k.threads));
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, k.fn, params);
}

}  // namespace

cudaError_t launch_staged_chunk(bool seq_to_head, const StagedArgs& a, cudaStream_t stream,
                                LaunchShape* shape)
{
    int device = 0;
    if (current_sm_count(&device) <= 0)
        return cudaErrorNoDevice;
    const bool wide = wide_ok(a);
    const StagedKernel first = seq_to_head ? pick_row<true>(a, wide) : pick_block<false>(a, wide);
    const StagedKernel second = seq_to_head ? pick_block<true>(a, wide) : pick_row<false>(a, wide);
    int grid1 = 0, grid2 = 0;
    cudaError_t err = launch_staged(first, a, stream, &grid1);
    if (err == cudaSuccess)
        err = launch_staged(second, a, stream, &grid2);
    if (shape) {
        shape->grid = grid1 > grid2 ? grid1 : grid2;
        shape->block = first.threads > second.threads ? first.threads : second.threads;
        shape->variant = H3_VARIANT_STAGED;
    }
    return err;
}

}  // namespace h3rr
