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
// Kernels (16-byte vectors, 128 threads, one row per CTA iteration):
//   staged_row_kernel<to_window>   sequence-side rows <-> window blocks
//                                  (the relayout proper)
//   window_block_kernel<to_head>   window blocks <-> head-side rows of plane p
//                                  (a strided copy per rank)
// seq->head = staged_row<true> then window_block<true>;
// head->seq = window_block<false> then staged_row<false>.
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

cudaError_t launch_one(const void* fn, int64_t work, const StagedArgs& a, cudaStream_t stream,
                       int* grid_out)
{
    int device = 0;
    const int sms = current_sm_count(&device);
    if (sms <= 0)
        return cudaErrorNoDevice;
    // One CTA per row / run, scheduled by the hardware (the kernels stride over
    // the rest if the work exceeds the grid limit).
    int64_t grid = work < kMaxGrid ? work : kMaxGrid;
    if (grid < 1)
        grid = 1;
    *grid_out = int(grid);
    void* params[] = {const_cast<StagedArgs*>(&a)};
    return cudaLaunchKernel(fn, dim3(unsigned(grid)), dim3(kThreads), params, 0, stream);
}

}  // namespace

cudaError_t launch_staged_chunk(bool seq_to_head, const StagedArgs& a, cudaStream_t stream,
                                LaunchShape* shape)
{
    int grid1 = 0, grid2 = 0;
    cudaError_t err;
    if (seq_to_head) {
        err = launch_one((const void*)staged_row_kernel<true>, a.n, a, stream, &grid1);
        if (err == cudaSuccess)
            err = launch_one((const void*)window_block_kernel<true>, int64_t(a.W) * a.n, a, stream, &grid2);
    } else {
        err = launch_one((const void*)window_block_kernel<false>, int64_t(a.W) * a.n, a, stream, &grid1);
        if (err == cudaSuccess)
            err = launch_one((const void*)staged_row_kernel<false>, a.n, a, stream, &grid2);
    }
    if (shape) {
        shape->grid = grid1 > grid2 ? grid1 : grid2;
        shape->block = kThreads;
        shape->variant = H3_VARIANT_STAGED;
    }
    return err;
}

}  // namespace h3rr
