// Internal host declarations shared by the entry points, the host plan and
// the launch code; what the kernels themselves see is in kernel_args.h.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

#include "h3rr.h"
#include "kernel_args.h"

namespace h3rr {

// ---------------------------------------------------------------------------
// Argument checks shared by the entry points (api.cpp, rank.cpp).
// ---------------------------------------------------------------------------
bool aligned16(const void* p);
void clear_info(h3_exec_info* info);
// Launch-config fields every entry point checks the same way; `flags` may
// hold only the bits in `allowed` (H3_LAUNCH_SERIAL everywhere, plus
// H3_LAUNCH_CHUNK_TOKENS for the relayouts).
bool config_ok(const h3_launch_config* cfg, int32_t allowed = H3_LAUNCH_SERIAL);
bool token_range_chunks(const h3_launch_config* cfg);
// Largest side of a relayout in bytes (64 PiB: far above any device), so
// that byte counts times the rank count stay within 64 bits.
constexpr uint64_t kMaxSideBytes = uint64_t(1) << 56;
// Sizes of a relayout (all entry points and the plan queries): positive
// sizes (H3_ERR_INVALID_ARG), head rows of whole 16-byte vectors
// (H3_ERR_MISALIGNED), T*P rows within int32, a row within kMaxRowVecs
// vectors and each side's T*P*H*D*2 bytes within kMaxSideBytes
// (H3_ERR_UNSUPPORTED).
h3_status check_relayout_sizes(int64_t n_tokens, int32_t planes, int32_t n_heads, int32_t head_dim);
// Row-based calls (reduce-scatters, all-gather) on [T, C] BF16 rows (C >= 1):
// true if T is beyond int32, a row beyond kMaxRowVecs vectors or T*C*2
// beyond kMaxSideBytes.
bool rows_beyond_limits(int64_t n_tokens, int64_t cols);
bool programmatic_launch(const h3_launch_config* cfg);
// Partition checks ("Distributed H3 Execution", intro: empty token or head
// partitions are rejected).
h3_status check_world(int64_t n_tokens, int64_t n_heads, int32_t world);
// Outputs may not overlap inputs or each other (FastVideo PR #1807, "Problem
// and behavior": outputs keep storage of their own).
h3_status check_no_overlap(const void* const* in, const uint64_t* in_bytes, int n_in,
                           void* const* out, const uint64_t* out_bytes, int n_out);

// ---------------------------------------------------------------------------
// Quotient/remainder partition ("Distributed H3 Execution", "Partition
// Contract"): n items over w ranks, q = n / w, m = n % w; rank i owns q + (i < m)
// items starting at i*q + min(i, m).  Host side; the kernels carry (q, m).
// ---------------------------------------------------------------------------
struct Split {
    int64_t q = 0;
    int64_t m = 0;
    int32_t w = 0;
    int64_t start(int32_t i) const { return i * q + (i < m ? i : m); }
    int64_t size(int32_t i) const { return q + (i < m ? 1 : 0); }
    int64_t largest() const { return q + (m > 0 ? 1 : 0); }
};

Split make_split(int64_t n, int32_t w);

// The launches of a relayout call: plane_groups x per_group launches, each
// moving per_launch planes of a range of local tokens of every rank:
// range c of a group covers [c*tokens, c*tokens + tokens) (fewer in the
// last one), so that every launch is one all-to-all over all ranks.
//   unchunked (window 0):   1 group of all P planes, one range;
//   one plane per launch:   P groups of one plane (FastVideo PR #1807,
//                           "Problem and behavior": one batch plane at a
//                           time through a byte window), split by tokens
//                           when a plane does not fit;
//   token ranges (H3_LAUNCH_CHUNK_TOKENS): 1 group of all P planes, split
//                           by tokens so that every launch fits the window.
struct RelayoutChunks {
    int64_t per_group = 1;  // token ranges per plane group
    int64_t tokens = 0;     // local tokens of each rank per full range
    int32_t plane_groups = 1;
    int32_t per_launch = 1;  // planes per launch
};

// The plan of a relayout of `planes` planes over `window_bytes` (0 = one
// launch).  A window must hold each rank's send slice (L tokens of
// row_bytes per plane moved) and receive slice (L tokens of W ranks, of the
// widest head rank, per plane moved); the fewest ranges of equal length L
// that fit are used, or one per plane group when its whole slices fit.
// H3_ERR_WINDOW if not even one token fits.
h3_status plan_relayout(const Split& ts, const Split& hs, int64_t n_tokens, int32_t planes,
                        uint64_t row_bytes, uint64_t head_bytes, int64_t window_bytes,
                        bool token_ranges, RelayoutChunks* out);

// Token split of range c of a plane group: rank r holds cq + (r < cm) tokens
// of the range, local tokens t0 .. of its own range.  Full ranges are
// (tokens, 0); the last is what remains of the quotient/remainder split,
// (q - t0, m).
void chunk_split(const Split& ts, const RelayoutChunks& ch, int64_t c, int64_t* cq, int64_t* cm,
                 int64_t* t0);

// Clip packed segments to [ts, te) and rebase; returns the piece count.
int32_t clip_segments(const int64_t* bounds, int32_t n_segs, int64_t ts, int64_t te,
                      int64_t* local_bounds, int32_t* seg_ids);

// [a, a+na) and [b, b+nb) share a byte.
bool ranges_overlap(uintptr_t a, uint64_t na, uintptr_t b, uint64_t nb);

struct LaunchShape {
    int grid = 0;
    int block = 0;
    int variant = H3_VARIANT_NONE;
};

// Enqueue one relayout launch.  seq_to_head selects the direction; layout
// selects the kernels that read a.seq_pm / a.head_pm (plane-major buffers).
cudaError_t launch_relayout(bool seq_to_head, const RelayoutArgs& a, int variant,
                            int ctas_per_sm, cudaStream_t stream, LaunchShape* shape,
                            bool layout = false, bool programmatic = false);

// Whether the bulk kernel's shared-memory stages fit the rows of these args.
bool relayout_bulk_fits(const RelayoutArgs& a, int device);

// Copy (and optionally clear) the per-device count of expired bulk waits.
cudaError_t read_bulk_wait_timeouts(unsigned int* count, bool reset, cudaStream_t stream);

// Enqueue the two launches (pack, unpack) of one staged chunk.
cudaError_t launch_staged_chunk(bool seq_to_head, const StagedArgs& a, cudaStream_t stream,
                                LaunchShape* shape);

// The staged relayout on a given window (checks, plan and launches).
h3_status staged_relayout_with_window(bool seq_to_head, const void* const* send, void* const* recv,
                                      int64_t n_tokens, int32_t planes, int32_t n_heads,
                                      int32_t head_dim, int32_t world, void* window,
                                      int64_t window_bytes, void* stream, h3_exec_info* info);

// Record `err` as the calling thread's last CUDA error; returns H3_ERR_CUDA.
h3_status record_cuda_failure(cudaError_t err);

// Enqueue one launch of a rank's share of sequence->head.
cudaError_t launch_pull_seq_to_head(const PullArgs& a, int ctas_per_sm, cudaStream_t stream,
                                    LaunchShape* shape, bool programmatic);

// Enqueue the all-gather launch (variant 0 / H3_VARIANT_VECTOR or H3_VARIANT_BULK).
cudaError_t launch_all_gather(const GatherArgs& a, int variant, int ctas_per_sm, cudaStream_t stream,
                              LaunchShape* shape, bool programmatic);
bool all_gather_bulk_fits(const GatherArgs& a, int device);
cudaError_t read_gather_wait_timeouts(unsigned int* count, bool reset, cudaStream_t stream);

// Enqueue the gated reduce-scatter launch.
cudaError_t launch_reduce_scatter_gated(const GatedArgs& a, cudaStream_t stream, LaunchShape* shape,
                                        bool programmatic);

// Enqueue the reduce-scatter launch.
cudaError_t launch_reduce_scatter(const ReduceArgs& a, int ctas_per_sm, cudaStream_t stream,
                                  LaunchShape* shape, bool programmatic);

// SM count of the current device (cached per device).
int current_sm_count(int* device);

// Opt a kernel in to `smem` bytes of dynamic shared memory on the current
// device (once per kernel, device and size).
cudaError_t allow_dynamic_smem(const void* kernel, size_t smem, int device);

// Launch `kernel` on a 1-D grid; `programmatic` sets programmatic stream
// serialization (the kernel must follow the griddepcontrol protocol below).
cudaError_t launch_kernel(const void* kernel, int64_t grid, int block, size_t smem,
                          cudaStream_t stream, void** params, bool programmatic);
}  // namespace h3rr
