// What the kernels see: sizes, the argument structures passed by value to
// every launch, and the device side of programmatic dependent launch.  Host
// planning, checks and launch declarations are in h3rr_internal.h.
#pragma once

#include <climits>
#include <cstdint>

#include "h3rr.h"

namespace h3rr {

constexpr int kMaxWorld = H3RR_MAX_WORLD;
constexpr int kVecBytes = 16;  // one 16-byte vector = 8 BF16 values
constexpr int64_t kMaxInt32 = INT32_MAX;
// Column loops step by up to 1024 vectors past the row end; keep that in int32.
constexpr int64_t kMaxRowVecs = int64_t(1) << 30;

// ---------------------------------------------------------------------------
// Kernel arguments (passed by value as __grid_constant__ parameters).
// ---------------------------------------------------------------------------

// One relayout launch moves planes [plane0, plane0 + nplanes) of every token.
// A "row" is one (token, plane) pair: row_vecs vectors on the sequence side,
// split into W runs of H_j * head_vecs vectors on the head side.
struct RelayoutArgs {
    char* seq[kMaxWorld];    // sequence-side rank buffers [T_r, P, H, D]
    char* head[kMaxWorld];   // head-side rank buffers [T, P, H_j, D]
    int32_t T;
    int32_t P;
    int32_t W;
    int32_t plane0;
    int32_t nplanes;
    int32_t rows;            // tokens of the launch * nplanes
    int32_t tq, tm;          // token split
    int32_t cq, cm, t0;      // the launch's tokens: cq + (r < cm) of rank r from local token t0
    int32_t hq, hm;          // head split
    int32_t row_vecs;        // H * D * 2 / 16
    int32_t head_vecs;       // D * 2 / 16
    int32_t seq_pm;          // sequence side plane-major [P, T_r, H, D] (layout kernels only)
    int32_t head_pm;         // head side plane-major [P, T, H_j, D] (layout kernels only)
    int32_t wait_late;       // 1: independent of the previous launch; wait for it at the end
};

struct ReduceArgs {
    const char* part[kMaxWorld];  // partials [T, C]
    char* out[kMaxWorld];         // outputs [T_r, C]
    const char* bias;             // [C] or nullptr
    int32_t T;
    int32_t W;
    int32_t tq, tm;
    int32_t row_vecs;             // C / 8
    int64_t row_bytes;            // C * 2
};

// One chunk of a staged relayout: tokens [t0, t0 + n) of plane p, packed into
// `window` head-rank-major (rank j's block [n, H_j, D] at n * hs_j heads).
struct StagedArgs {
    char* seq[kMaxWorld];
    char* head[kMaxWorld];
    char* window;
    int32_t T;
    int32_t P;
    int32_t W;
    int32_t p;
    int32_t t0;
    int32_t n;
    int32_t tq, tm;
    int32_t hq, hm;
    int32_t row_vecs;
    int32_t head_vecs;
};

// Ragged all-gather: rank r's rows [T_r, C] -> every rank's [T, C].
struct GatherArgs {
    const char* in[kMaxWorld];
    char* out[kMaxWorld];
    int32_t T;
    int32_t W;          // outputs written (every row goes to out[0..W-1])
    int32_t n_in;       // input blocks (the token split's ranks)
    int32_t tq, tm;
    int32_t row_vecs;   // C / 8
    int64_t row_bytes;  // C * 2
};

// One rank's share of sequence->head (one rank per GPU): for every (t, p) of
// the launch, the run of heads [hs, hs + H_k) of the sequence-side row held
// by token t's rank, copied to row (t, p) of this rank's head-side buffer.
struct PullArgs {
    const char* src[kMaxWorld];  // sequence-side buffers [T_r, P, H, D], any GPU
    char* dst;                   // this rank's head-side buffer [T, P, H_k, D]
    int32_t W;                   // ranks (entries of src)
    int32_t T;
    int32_t P;
    int32_t plane0;
    int32_t nplanes;
    int32_t rows;                // tokens of the launch * nplanes
    int32_t tq, tm;              // token split
    int32_t cq, cm, t0;          // the launch's tokens, as RelayoutArgs
    int32_t row_vecs;            // H * D * 2 / 16
    int32_t run_vecs;            // H_k * D * 2 / 16
    int32_t col0_vecs;           // hs * D * 2 / 16
    int32_t wait_late;           // as RelayoutArgs::wait_late
};

// Reduce-scatter fused with residual gating per packed segment.
constexpr int kMaxGateSegs = 256;
struct GatedArgs {
    ReduceArgs r;                       // partials, out (written), bias, sizes
    const char* x[kMaxWorld];           // residual rows [T_r, C] (may equal r.out[.])
    const char* gate;                   // [S, C]
    int32_t n_segs;
    int32_t seg_bounds[kMaxGateSegs + 1];  // 0 = b_0 < ... < b_S = T
};

#ifdef __CUDACC__
// Programmatic dependent launch, device side.  A kernel launched with
// programmatic stream serialization may start before the previous kernel in
// the stream has completed; griddepcontrol.wait blocks the calling thread
// until every prerequisite grid has completed and its writes are visible (a
// no-op for a plain launch).  launch_dependents lets the next such kernel be
// scheduled once every CTA of this grid has issued it (or exited).
__device__ __forceinline__ void pdl_wait_prerequisites()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void pdl_allow_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// End of a launch that is independent of the previous one (wait_late): it
// must not complete before the previous grid has.  One waiting thread is
// enough for that (a grid completes only when all its threads have exited),
// so only thread 0 of CTA 0 waits and every other CTA frees its slot at once.
__device__ __forceinline__ void pdl_wait_at_end(int32_t wait_late)
{
    if (wait_late && blockIdx.x == 0 && threadIdx.x == 0)
        pdl_wait_prerequisites();
}
#endif

}  // namespace h3rr
