/*
 * h3rr.h - C ABI of the B200 (sm_100a) library for the data-parallel hot path
 * of the distributed H3 denoiser: the Ulysses sequence->head relayout of
 * packed BF16 QKV/QKVG, its inverse head->sequence relayout, and the
 * tensor-mode ragged reduce-scatter.
 *
 * All W "virtual ranks" live in one GPU's memory: rank r's send and receive
 * buffers are ordinary device buffers, and the library moves bytes between
 * them with its own kernels.  No collective library is involved.
 *
 * Sources (page title, section):
 *   "Distributed H3 Execution" (h3-blackwell-runtime DISTRIBUTED.md)
 *      - intro: the "ulysses" mode's sequence-to-head all-to-all on QKV and
 *        the inverse head-to-sequence all-to-all around attention; the packed
 *        sequence is kept, empty token or head partitions are rejected, no
 *        padding is added.
 *      - "Partition Contract": 56 heads of width 128, balanced and possibly
 *        ragged (table: W=6 -> 10,10,9,9,9,9); tokens split the same way;
 *        segment boundaries clipped to each rank's interval and rebased;
 *        tensor mode's ragged reduce-scatter sums the rank partials and
 *        assigns token rows; the bias is added exactly once after reduction.
 *   FastVideo PR #1807 "[perf] Harden Ulysses agreement and tune bounded H3
 *        transfers", "Problem and behavior": one batch plane transferred at a
 *        time under an 896,000,000-byte window; outputs keep storage of their
 *        own.
 *
 * Conventions shared by every call
 *   - Partition of n items over W ranks: q = n / W, m = n % W; rank i owns
 *     q + (i < m) items starting at i*q + min(i, m).
 *   - BF16 buffers are dense row-major arrays of 16-bit patterns.
 *     Sequence side, rank r:  [T_r, P, H, D]  (tokens ts_r .. te_r-1, all heads)
 *     Head side, rank j:      [T, P, H_j, D]  (all tokens, heads hs_j .. he_j-1)
 *     Sequence-side buffers may be views into one [T, P, H, D] tensor at
 *     token offsets ts_r; head-side buffers may be views into one tensor.
 *   - Pointer arrays (send[], recv[], partials[], out[]) are HOST arrays of
 *     `world` DEVICE pointers; they are read during the call only.  The
 *     library allocates no device memory and keeps no caller pointer after
 *     return.  (One file-scope 16 MiB window aside: the first
 *     h3_seq_to_head_staged_noalloc call in a context loads it.)
 *   - The caller owns every buffer.  Outputs must not overlap any input or
 *     any other output (outputs keep storage of their own); overlap is
 *     detected and rejected.
 *   - Every device pointer must be 16-byte aligned and every contiguous run
 *     a multiple of 16 bytes (head_dim*2 % 16 == 0, cols % 8 == 0).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work
 *     is enqueued on it and the call returns without synchronising; results
 *     are visible to later work on that stream.
 *   - Arguments are checked before anything is launched; on any error
 *     nothing is launched and the returned status says why.
 *   - `info` (nullable) receives what actually ran: launches, chunks, grid,
 *     block and kernel variant.
 *   - Sizes: a relayout's T and T*P below 2^31, a row (H*D*2 bytes) of at
 *     most 2^30 16-byte vectors and each side (T*P*H*D*2 bytes) at most 2^56
 *     bytes; the row calls' T below 2^31, C/8 at most 2^30 and T*C*2 at most
 *     2^56 bytes; beyond them H3_ERR_UNSUPPORTED.
 *   - Thread-safe, and no environment variables are read.  State kept across
 *     calls: per-device caches (SM count),
 *     per-context state (the bulk kernels' shared-memory opt-in, the static
 *     window's address, the peer mappings h3_ipc_open holds until
 *     h3_ipc_close; after cudaDeviceReset the device's next context sets them
 *     up again), each thread's last CUDA error, and the device-side counters
 *     of expired bounded waits.
 */
#ifndef H3RR_H
#define H3RR_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define H3RR_API __attribute__((visibility("default")))
#else
#define H3RR_API
#endif

#define H3RR_ABI_VERSION 3
#define H3RR_MAX_WORLD 64

typedef enum h3_status {
    H3_OK = 0,
    H3_ERR_INVALID_ARG = 1,      /* NULL pointer, negative size, overlapping outputs, bad segments */
    H3_ERR_EMPTY_PARTITION = 2,  /* world > tokens or world > heads: some rank would own nothing */
    H3_ERR_MISALIGNED = 3,       /* a pointer or a contiguous run is not 16-byte aligned */
    H3_ERR_WINDOW = 4,           /* window_bytes cannot hold the data of one token */
    H3_ERR_UNSUPPORTED = 5,      /* world > H3RR_MAX_WORLD, or a size beyond the kernels' index range */
    H3_ERR_CUDA = 6              /* the CUDA runtime reported an error while launching */
} h3_status;

/* Kernel variants reported in h3_exec_info.variant. */
#define H3_VARIANT_NONE 0
#define H3_VARIANT_VECTOR 1      /* 16- or 32-byte vector loads/stores through registers */
#define H3_VARIANT_BULK 2        /* bulk async copies through shared memory */
#define H3_VARIANT_REDUCE 3      /* binary32 reduce-scatter through registers */
#define H3_VARIANT_STAGED 4      /* pack into a window buffer, then unpack */
#define H3_VARIANT_GATHER 5      /* ragged all-gather */
#define H3_VARIANT_REDUCE_GATED 6 /* reduce-scatter fused with residual gating */

typedef struct h3_exec_info {
    int32_t launches;            /* kernel launches enqueued by the call */
    int32_t chunks;              /* chunks of the plan: 1 unchunked, P * (token chunks per plane) one
                                    plane per launch, the token ranges with H3_LAUNCH_CHUNK_TOKENS */
    int32_t grid;                /* CTAs per launch */
    int32_t block;               /* threads per CTA */
    int32_t variant;             /* H3_VARIANT_* */
    int32_t planes_per_launch;   /* planes moved by one launch */
} h3_exec_info;

/*
 * Launch order.  By default every kernel the library launches (both
 * relayout and all-gather variants, the reduce-scatters, the staged and rank
 * calls' kernels) uses programmatic dependent launch (sm_90 and later): a
 * kernel may be scheduled while the previous kernel in the stream is
 * draining, and it waits for that kernel to complete
 * (griddepcontrol.wait) before its first global-memory access, so results are
 * those of plain stream order.  Within one chunked relayout call, the launch
 * of plane p+1 touches memory disjoint from plane p's and runs alongside
 * plane p's tail; it waits for plane p at its end instead, so that the call's
 * completion still implies every plane's.  The staged calls' kernels are
 * launched the same way and always wait at their start (each chunk depends on
 * the previous launch; only the launch latency is hidden).  A kernel that
 * follows in the stream and was itself launched with programmatic
 * serialization must wait (cudaGridDependencySynchronize) before reading
 * these calls' outputs.
 */
#define H3_LAUNCH_SERIAL 1       /* launch every kernel in plain stream order */
/*
 * H3_LAUNCH_CHUNK_TOKENS (relayout calls only; H3_ERR_INVALID_ARG elsewhere):
 * a chunked relayout (window_bytes > 0) cuts its work into token ranges that
 * cover every plane instead of one batch plane per launch.  Launch c moves
 * local tokens [c*L, c*L + L) of every rank's range (fewer in the last), all
 * P planes of them, with k the fewest launches and L the equal length for
 * which each rank's send slice (L*P*H*D*2) and receive slice
 * (W*L*P*max_j(H_j)*D*2) fit in window_bytes; one launch if everything fits.
 * The window bounds the same bytes per launch as in one-plane mode and the
 * result is identical, but every launch touches whole token rows of both
 * sides: on token-major buffers that is the unchunked rate, where one plane
 * per launch leaves the other planes' bytes between each row it touches and
 * runs 3-5 % slower on B200.  H3_ERR_WINDOW if the window cannot hold one
 * token of every plane.
 */
#define H3_LAUNCH_CHUNK_TOKENS 2

/* Optional launch overrides for h3_*_ex; zero fields mean "library default". */
typedef struct h3_launch_config {
    int32_t variant;             /* 0 = default, H3_VARIANT_VECTOR or H3_VARIANT_BULK (relayouts) */
    int32_t ctas_per_sm;         /* 0 = default: one CTA per row; n caps the grid at n per SM */
    int32_t flags;               /* H3_LAUNCH_* bits; other bits: H3_ERR_INVALID_ARG */
    int32_t reserved1;           /* must be 0 */
} h3_launch_config;

/* ABI version of the loaded library (H3RR_ABI_VERSION it was built with). */
H3RR_API int32_t h3_abi_version(void);

/* Short static English description of a status code. */
H3RR_API const char* h3_status_string(h3_status status);

/* The cudaError_t value behind the calling thread's most recent H3_ERR_CUDA
 * (0 if none), and, if message is not NULL, the CUDA runtime's static text
 * for it.  Kept per thread; a later H3_ERR_CUDA on the thread replaces it. */
H3RR_API int32_t h3_last_cuda_error(const char** message);

/*
 * h3_partition - the partition contract, host only ("Distributed H3
 * Execution", "Partition Contract").
 *
 *   n_tokens, n_heads, world : T, H, W.  W >= 1; W <= T and W <= H, else
 *                              H3_ERR_EMPTY_PARTITION.
 *   seg_bounds  [n_segs+1]   : packed segment boundaries, 0 = b_0 < b_1 <
 *                              ... < b_S = T (strictly increasing, else
 *                              H3_ERR_INVALID_ARG).  May be NULL iff n_segs == 0,
 *                              in which case the segment outputs below are
 *                              not touched and may be NULL.
 *   token_starts [world+1]   : out, ts_0 .. ts_W (int64).
 *   head_starts  [world+1]   : out, hs_0 .. hs_W (int32).
 *   piece_offsets [world+1]  : out.  Rank r's clipped pieces are
 *                              k = piece_offsets[r] .. piece_offsets[r+1]-1.
 *   local_seg_ids [n_segs+world-1] : out, global segment index of piece k.
 *   local_bounds [n_segs+2*world-1] : out.  Rank r's rebased bounds are
 *                              local_bounds[piece_offsets[r] + r ...
 *                              piece_offsets[r+1] + r] (pieces + 1 values,
 *                              first 0, last T_r).
 * A segment whose intersection with [ts_r, te_r) is empty gives no piece.
 * All arrays are caller-allocated host memory.
 */
H3RR_API h3_status h3_partition(int64_t n_tokens, int32_t n_heads, int32_t world,
                       const int64_t* seg_bounds, int32_t n_segs,
                       int64_t* token_starts, int32_t* head_starts,
                       int64_t* local_bounds, int32_t* local_seg_ids,
                       int32_t* piece_offsets);

/*
 * h3_seq_to_head - Ulysses sequence->head relayout ("Distributed H3
 * Execution", intro: QKV sequence-to-head all-to-all).
 *
 *   send[world] : device, rank r's [T_r, P, H, D] BF16 (T_r tokens, all heads).
 *   recv[world] : device, rank j's [T, P, H_j, D] BF16, written.
 *   out_j[t, p, h, d] = send_{r(t)}[t - ts_{r(t)}, p, hs_j + h, d]   (bit copy)
 *   n_tokens T, planes P (3 = QKV, 4 = QKVG, 1 = a single operand),
 *   n_heads H, head_dim D, world W.
 *   window_bytes : 0 = one launch over all planes.  > 0 = chunked mode (FastVideo
 *                  PR #1807, "Problem and behavior"): one batch plane p per
 *                  launch, as long as the largest per-rank send slice of one
 *                  plane (max_r T_r*H*D*2) and the largest per-rank receive
 *                  slice (max_j T*H_j*D*2) are <= window_bytes.  A plane larger
 *                  than that is split by tokens: k launches per plane, launch
 *                  c moving local tokens [c*L, c*L + L) of every rank's range
 *                  (fewer in the last), with k the fewest chunks and L the
 *                  equal length for which L*H*D*2 <= window_bytes and
 *                  W*L*max_j(H_j)*D*2 <= window_bytes (h3_relayout_chunk_plan
 *                  reports k and L).  H3_ERR_WINDOW only if not even L = 1
 *                  fits.  The result is identical either way.
 *                  (h3_seq_to_head_ex with H3_LAUNCH_CHUNK_TOKENS cuts the
 *                  same window into token ranges of all planes instead.)
 */
H3RR_API h3_status h3_seq_to_head(const void* const* send, void* const* recv,
                         int64_t n_tokens, int32_t planes, int32_t n_heads,
                         int32_t head_dim, int32_t world, int64_t window_bytes,
                         void* stream, h3_exec_info* info);

/*
 * h3_relayout_chunk_plan - host only: how the chunked relayouts (and the
 * h3_*_rank relayouts) cut their work under window_bytes.
 *   tokens_per_chunk : out, L: tokens of each rank per launch (max_r T_r when
 *                      a whole plane fits the window or window_bytes == 0).
 *   chunks           : out, launches of a one-GPU call: 1 if window_bytes == 0,
 *                      else planes * k (k token chunks per plane).
 * Errors as h3_seq_to_head's argument checks (H3_ERR_EMPTY_PARTITION,
 * H3_ERR_WINDOW, H3_ERR_INVALID_ARG on NULL outputs or non-positive sizes).
 */
H3RR_API h3_status h3_relayout_chunk_plan(int64_t n_tokens, int32_t planes, int32_t n_heads,
                                          int32_t head_dim, int32_t world, int64_t window_bytes,
                                          int64_t* tokens_per_chunk, int64_t* chunks);

/*
 * h3_relayout_chunk_plan_ex - as h3_relayout_chunk_plan for the chunk shape
 * that `flags` selects (0, or H3_LAUNCH_CHUNK_TOKENS: token ranges over all
 * planes; H3_LAUNCH_SERIAL is accepted and changes nothing).
 *   chunks            : out, launches of a one-GPU call (1 if window_bytes == 0;
 *                       planes * k one plane per launch; k token ranges with
 *                       H3_LAUNCH_CHUNK_TOKENS).
 *   planes_per_launch : out (may be NULL), 1 one plane per launch, else P.
 */
H3RR_API h3_status h3_relayout_chunk_plan_ex(int64_t n_tokens, int32_t planes, int32_t n_heads,
                                             int32_t head_dim, int32_t world, int64_t window_bytes,
                                             int32_t flags, int64_t* tokens_per_chunk,
                                             int64_t* chunks, int32_t* planes_per_launch);

/*
 * h3_head_to_seq - inverse head->sequence relayout ("Distributed H3
 * Execution", intro: inverse head-to-sequence all-to-all around attention).
 *
 *   send[world] : device, rank j's [T, P, H_j, D] BF16.
 *   recv[world] : device, rank r's [T_r, P, H, D] BF16, written.
 *   out_r[t', p, hs_j + h, d] = send_j[ts_r + t', p, h, d]   (bit copy)
 *   Other arguments as h3_seq_to_head (the window bounds the per-rank head-
 *   side slice of one plane and the per-rank sequence-side slice).
 */
H3RR_API h3_status h3_head_to_seq(const void* const* send, void* const* recv,
                         int64_t n_tokens, int32_t planes, int32_t n_heads,
                         int32_t head_dim, int32_t world, int64_t window_bytes,
                         void* stream, h3_exec_info* info);

/*
 * h3_ragged_reduce_scatter - tensor-mode ragged reduce-scatter ("Distributed
 * H3 Execution", "Partition Contract": rank partials summed, token rows
 * assigned, projection bias added exactly once after the reduction).
 *
 *   partials[world] : device, rank w's partial output [T, C] BF16 (no bias).
 *   bias            : device [C] BF16, or NULL for no bias.
 *   out[world]      : device, rank r's rows [T_r, C] BF16, written.
 *   out_r[t', c] = bf16_rne( ((p_0 + p_1) + ... + p_{W-1}) + bias[c] ),
 *     t = ts_r + t', every term widened exactly to binary32, the sum taken
 *     in binary32 in rank order 0..W-1 starting from p_0, the bias added
 *     once after the sum, rounded to BF16 to nearest, ties to even.  No
 *     flush-to-zero; Inf and NaN propagate (a NaN result may be any NaN).
 *   n_tokens T, cols C (C % 8 == 0), world W.
 */
H3RR_API h3_status h3_ragged_reduce_scatter(const void* const* partials, const void* bias,
                                   void* const* out, int64_t n_tokens, int64_t cols,
                                   int32_t world, void* stream, h3_exec_info* info);

/*
 * h3_ragged_reduce_scatter_gated - the ragged reduce-scatter fused with
 * residual gating per packed segment ("Distributed H3 Execution", "Partition
 * Contract": segment boundaries clipped to each rank's token interval and
 * rebased before AdaLN modulation and residual gating).
 *
 *   partials, bias, n_tokens T, cols C, world W : as h3_ragged_reduce_scatter.
 *   gate       : device [S, C] BF16, one gating row per packed segment.
 *   seg_bounds : host [S+1], 0 = b_0 < b_1 < ... < b_S = T (as h3_partition),
 *                1 <= S <= H3RR_MAX_GATE_SEGMENTS; read during the call only.
 *   x[world]   : device, rank r's residual rows [T_r, C] BF16.
 *   out[world] : device, rank r's [T_r, C] BF16, written; out[r] may be x[r]
 *                itself (in place) but must not partly overlap it or overlap
 *                anything else.
 *   For rank r, local row t' (t = ts_r + t'), k = the segment holding t
 *   (equivalently, the global index of the rank's clipped piece holding t'):
 *     y          = the h3_ragged_reduce_scatter output element (BF16)
 *     out_r[t',c] = bf16_rne( x_r[t',c] + gate[k,c] * y )   in binary32
 *   (the BF16 x BF16 product is exact in binary32; one rounding in the add,
 *   then round to nearest even).  Equal, bit for bit, to running
 *   h3_ragged_reduce_scatter and then the gating; one launch, and y is never
 *   written to memory.
 */
#define H3RR_MAX_GATE_SEGMENTS 256
H3RR_API h3_status h3_ragged_reduce_scatter_gated(const void* const* partials, const void* bias,
                                                  const void* gate, const int64_t* seg_bounds,
                                                  int32_t n_segs, const void* const* x,
                                                  void* const* out, int64_t n_tokens, int64_t cols,
                                                  int32_t world, void* stream, h3_exec_info* info);

/*
 * h3_seq_to_head_layout / h3_head_to_seq_layout - the relayouts with
 * plane-major buffers on either side.  layout is a bit set:
 *   H3_LAYOUT_SEQ_PLANE_MAJOR  sequence-side rank r is [P, T_r, H, D] (plane p
 *                              a contiguous [T_r, H, D] block: separate Q, K, V
 *                              projection outputs) instead of [T_r, P, H, D];
 *   H3_LAYOUT_HEAD_PLANE_MAJOR head-side rank j is [P, T, H_j, D] (plane p a
 *                              contiguous [T, H_j, D] block: the Q, K and V an
 *                              attention kernel takes) instead of [T, P, H_j, D].
 * The element maps are those of h3_seq_to_head / h3_head_to_seq; only where
 * element (t, p, h, d) sits in each buffer changes.  Buffer sizes are the same,
 * so every check (alignment, overlap, window) is unchanged.  layout 0 equals the
 * plain calls.  Unknown bits are H3_ERR_INVALID_ARG; cfg (nullable) as in the
 * _ex calls, except that H3_VARIANT_BULK with a non-zero layout is
 * H3_ERR_UNSUPPORTED.
 */
#define H3_LAYOUT_SEQ_PLANE_MAJOR 1
#define H3_LAYOUT_HEAD_PLANE_MAJOR 2
H3RR_API h3_status h3_seq_to_head_layout(const void* const* send, void* const* recv,
                                         int64_t n_tokens, int32_t planes, int32_t n_heads,
                                         int32_t head_dim, int32_t world, int64_t window_bytes,
                                         int32_t layout, void* stream, const h3_launch_config* cfg,
                                         h3_exec_info* info);
H3RR_API h3_status h3_head_to_seq_layout(const void* const* send, void* const* recv,
                                         int64_t n_tokens, int32_t planes, int32_t n_heads,
                                         int32_t head_dim, int32_t world, int64_t window_bytes,
                                         int32_t layout, void* stream, const h3_launch_config* cfg,
                                         h3_exec_info* info);

/*
 * h3_ragged_all_gather - ragged all-gather of token rows ("Distributed H3
 * Execution", intro: ragged row gathering, whose temporary collective padding
 * is removed before model operations; "Validation": ragged gather and
 * reduce-scatter behaviour).  The companion of h3_ragged_reduce_scatter: rank
 * r holds rows ts_r .. te_r-1, afterwards every rank holds all T rows.
 *
 *   in[world]  : device, rank r's rows [T_r, C], 16-bit elements (BF16).
 *   out[world] : device, rank j's [T, C], written.
 *   out_j[t, c] = in_{r(t)}[t - ts_{r(t)}, c]   (bit copy; nothing padded)
 *   n_tokens T, cols C (C % 8 == 0), world W.  Errors as
 *   h3_ragged_reduce_scatter.
 */
H3RR_API h3_status h3_ragged_all_gather(const void* const* in, void* const* out,
                                        int64_t n_tokens, int64_t cols, int32_t world,
                                        void* stream, h3_exec_info* info);
/* With launch overrides: variant 0 / H3_VARIANT_VECTOR (registers) or
 * H3_VARIANT_BULK (bulk copies through shared memory; H3_ERR_UNSUPPORTED if
 * four rows of C*2 bytes do not fit in shared memory, rows above about 57 KB
 * on B200), and ctas_per_sm. */
H3RR_API h3_status h3_ragged_all_gather_ex(const void* const* in, void* const* out,
                                           int64_t n_tokens, int64_t cols, int32_t world,
                                           void* stream, const h3_launch_config* cfg,
                                           h3_exec_info* info);

/*
 * Same as h3_seq_to_head / h3_head_to_seq / h3_ragged_reduce_scatter with
 * explicit launch overrides (cfg may be NULL).  Every variant computes the
 * same bytes; the overrides exist for tuning and for testing each variant.
 * An unknown variant returns H3_ERR_INVALID_ARG.  H3_VARIANT_BULK relayouts
 * stage four rows of H*D*2 bytes in shared memory: H3_ERR_UNSUPPORTED if they
 * do not fit (rows above about 57 KB on B200), or with a non-zero layout.
 */
H3RR_API h3_status h3_seq_to_head_ex(const void* const* send, void* const* recv,
                            int64_t n_tokens, int32_t planes, int32_t n_heads,
                            int32_t head_dim, int32_t world, int64_t window_bytes,
                            void* stream, const h3_launch_config* cfg,
                            h3_exec_info* info);
H3RR_API h3_status h3_head_to_seq_ex(const void* const* send, void* const* recv,
                            int64_t n_tokens, int32_t planes, int32_t n_heads,
                            int32_t head_dim, int32_t world, int64_t window_bytes,
                            void* stream, const h3_launch_config* cfg,
                            h3_exec_info* info);
H3RR_API h3_status h3_ragged_reduce_scatter_ex(const void* const* partials, const void* bias,
                                      void* const* out, int64_t n_tokens, int64_t cols,
                                      int32_t world, void* stream,
                                      const h3_launch_config* cfg, h3_exec_info* info);

/*
 * h3_seq_to_head_staged / h3_head_to_seq_staged - the same relayouts staged
 * through a caller-provided window buffer, the way a registered-window
 * transport moves them (FastVideo PR #1807, "Problem and behavior": one
 * batch plane at a time through a window of at most 896,000,000 bytes).
 *
 * Work is cut into chunks of one plane and at most
 * floor(window_bytes / (H*D*2)) tokens; each chunk is packed into `window`
 * (head-side rank j's block [n, H_j, D] at byte offset n*hs_j*D*2) and then
 * unpacked into the outputs: two launches per chunk, every byte read and
 * written twice.  Planes larger than the window are therefore split by
 * tokens.  The results equal h3_seq_to_head / h3_head_to_seq bit for bit.
 *
 *   window       : device scratch, caller-owned, 16-byte aligned, at least
 *                  one token row (H*D*2 bytes); must not overlap any input or
 *                  output; its contents on return are unspecified.  Calls that
 *                  share one window must not overlap in time.
 *   window_bytes : usable bytes of window (>= H*D*2, else H3_ERR_WINDOW).
 *   Other arguments, layouts and errors as h3_seq_to_head / h3_head_to_seq.
 */
H3RR_API h3_status h3_seq_to_head_staged(const void* const* send, void* const* recv,
                                         int64_t n_tokens, int32_t planes, int32_t n_heads,
                                         int32_t head_dim, int32_t world, void* window,
                                         int64_t window_bytes, void* stream, h3_exec_info* info);
H3RR_API h3_status h3_head_to_seq_staged(const void* const* send, void* const* recv,
                                         int64_t n_tokens, int32_t planes, int32_t n_heads,
                                         int32_t head_dim, int32_t world, void* window,
                                         int64_t window_bytes, void* stream, h3_exec_info* info);

/*
 * h3_seq_to_head_staged_noalloc - h3_seq_to_head_staged with a window that
 * lives inside the library, so that, once set up (below), a call allocates
 * no device memory at all.
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory themselves: for example a plugin that
 * only receives tensors from a host framework whose caching allocator owns
 * the whole memory budget, or a latency-critical loop in which cudaMalloc
 * or cudaFree would synchronise the device.  Such callers still pass their
 * inputs and outputs; only the staging window is provided here.
 *
 * The window is a file-scope device array of H3RR_STATIC_WINDOW_BYTES
 * (16 MiB).  The call never calls cudaMalloc or cudaFree, nor any allocating
 * library routine.
 *
 *   window_bytes : how much of the array to use, 0 = all of it.  Values
 *                  above H3RR_STATIC_WINDOW_BYTES (or negative) are rejected
 *                  with H3_ERR_UNSUPPORTED before anything is launched; a
 *                  window smaller than one token row (H*D*2 bytes) is
 *                  H3_ERR_WINDOW.
 *   Other arguments, layouts, results and errors as h3_seq_to_head_staged.
 *
 * The first call on a device (more exactly, in each CUDA context: again after
 * cudaDeviceReset) sets the entry point up: it looks up the array's device
 * address with cudaGetSymbolAddress, with that device current, and keeps it
 * for later calls in that context.  Under CUDA's default lazy module loading
 * that lookup is also when the runtime loads the array onto the device, and
 * the load reserves the 16 MiB there: the first call can therefore fail with
 * H3_ERR_CUDA (h3_last_cuda_error: cudaErrorMemoryAllocation) when the
 * device is full, and it may synchronise.  Only later calls allocate
 * nothing.  So make the first call early: before a caching allocator reserves
 * its whole budget, and before any stream capture.  From then on the device
 * holds the array until the process exits (with eager module loading, every
 * device the process uses holds it from the start).  Every call on a device shares
 * the one array and leaves its last chunk in it: nothing in it needs to
 * start at zero, because each chunk is written in full before it is read.
 * Calls that overlap on the GPU (for example on two streams without ordering
 * between them) race on the array and corrupt each other's output; order
 * them on one stream or with events.
 */
#define H3RR_STATIC_WINDOW_BYTES (16ll << 20)
H3RR_API h3_status h3_seq_to_head_staged_noalloc(const void* const* send, void* const* recv,
                                                 int64_t n_tokens, int32_t planes,
                                                 int32_t n_heads, int32_t head_dim, int32_t world,
                                                 int64_t window_bytes, void* stream,
                                                 h3_exec_info* info);

/*
 * h3_staged_plan - host only: the chunking the staged calls use.
 *   chunk_tokens : out, tokens per chunk (the last chunk of a plane may hold fewer).
 *   chunks       : out, chunks in all (planes * ceil(T / chunk_tokens)); the
 *                  staged calls enqueue 2 * chunks launches.
 * Returns H3_ERR_WINDOW if window_bytes < H*D*2, H3_ERR_INVALID_ARG on
 * non-positive sizes or NULL outputs.
 */
H3RR_API h3_status h3_staged_plan(int64_t n_tokens, int32_t planes, int32_t n_heads,
                                  int32_t head_dim, int64_t window_bytes,
                                  int64_t* chunk_tokens, int64_t* chunks);

/*
 * h3_bulk_wait_timeouts - how many bounded waits of the bulk kernels
 * (H3_VARIANT_BULK relayouts and all-gather) expired on the current device
 * since the count was last cleared.  Each wait on a shared-memory barrier gives up after a fixed
 * number of polls instead of spinning forever; an expiry means that launch's
 * output is incomplete.  Synchronises `stream`; reset != 0 clears the count.
 * count: host out-param.  Returns H3_ERR_CUDA if the copy fails.
 */
H3RR_API h3_status h3_bulk_wait_timeouts(void* stream, uint32_t* count, int32_t reset);

/*
 * h3_bounded_wait_selftest - diagnostic with no counterpart on the pages:
 * runs, in one tiny kernel, the bounded shared-memory-barrier wait the bulk
 * kernels use, on a barrier that expects one arrival.  arrive_first = 0: no
 * arrival ever comes, so the wait must give up after `polls` tries and
 * *expired becomes 1; arrive_first = 1: the arrival completes the phase
 * first and *expired becomes 0.  polls in [1, 2^24].  Synchronises `stream`.
 * Shows that an expired wait returns control (and leaves the context usable)
 * without faulting or trapping.  expired: host out-param (-1 until set).
 * Errors: H3_ERR_INVALID_ARG on bad arguments, H3_ERR_CUDA on a failed
 * launch or copy.
 */
H3RR_API h3_status h3_bounded_wait_selftest(uint32_t polls, int32_t arrive_first, void* stream,
                                            int32_t* expired);

/* ------------------------------------------------------------------------
 * One rank per GPU.  The calls above keep all W virtual ranks in one GPU's
 * memory.  With one rank per GPU (each process drives one GPU), rank k's share of
 * each operation is computed by the calls below, which pull what rank k
 * needs from every rank's buffer with plain 16- or 32-byte loads (no TMA,
 * no multicast) and write only rank k's own output.  The W rank calls
 * together write exactly what the one-GPU call writes, bit for bit
 * ("Distributed H3 Execution", "Remaining GPU Gates": identity of the real
 * collective at 2-8 GPUs and distributed-versus-single parity).
 *
 * Pointer arrays hold the W ranks' buffers as addresses the current device
 * can load from: its own buffer and the peers' buffers mapped with
 * h3_ipc_open (or any other peer mapping).  The peers' buffers must be
 * complete before the call is enqueued and unchanged until it has finished;
 * the caller orders this across processes (for example a stream
 * synchronisation and a host barrier on each side).  Arguments are checked
 * as in the one-GPU calls, plus 0 <= rank < world (else H3_ERR_INVALID_ARG);
 * overlap is checked between this rank's output and every input address
 * range.  The bulk variant is not offered (H3_ERR_UNSUPPORTED); cfg as in
 * the _ex calls otherwise.  Launch order as above.
 * ------------------------------------------------------------------------ */

/* Rank k's head-side buffer: recv [T, P, H_k, D] (this GPU) gets
 * recv[t, p, h, d] = send[r(t)][t - ts_{r(t)}, p, hs_k + h, d]
 * from send[world], the sequence-side buffers [T_r, P, H, D] of all ranks.
 * window_bytes as h3_seq_to_head: the same chunk plan over all ranks' slices,
 * so that all ranks chunk alike. */
H3RR_API h3_status h3_seq_to_head_rank(const void* const* send, void* recv, int64_t n_tokens,
                                       int32_t planes, int32_t n_heads, int32_t head_dim,
                                       int32_t world, int32_t rank, int64_t window_bytes,
                                       void* stream, const h3_launch_config* cfg,
                                       h3_exec_info* info);

/* Rank k's sequence-side buffer: recv [T_k, P, H, D] (this GPU) gets
 * recv[t', p, hs_j + h, d] = send[j][ts_k + t', p, h, d] from send[world],
 * the head-side buffers [T, P, H_j, D] of all ranks.  Under a window that
 * splits planes into token chunks, info->chunks is the plan's count and
 * info->launches counts only the chunks that hold tokens of rank k (the
 * last chunk of a plane may hold none of a smaller rank's tokens). */
H3RR_API h3_status h3_head_to_seq_rank(const void* const* send, void* recv, int64_t n_tokens,
                                       int32_t planes, int32_t n_heads, int32_t head_dim,
                                       int32_t world, int32_t rank, int64_t window_bytes,
                                       void* stream, const h3_launch_config* cfg,
                                       h3_exec_info* info);

/* Rank k's rows of the ragged reduce-scatter: out [T_k, C] (this GPU) gets
 * out[t', c] = bf16_rne(((p_0 + ... + p_{W-1}) + bias)[ts_k + t', c]) in
 * binary32, rank order, from partials[world] ([T, C] each, any rank's GPU);
 * bias [C] or NULL (read from wherever it is). */
H3RR_API h3_status h3_ragged_reduce_scatter_rank(const void* const* partials, const void* bias,
                                                 void* out, int64_t n_tokens, int64_t cols,
                                                 int32_t world, int32_t rank, void* stream,
                                                 const h3_launch_config* cfg,
                                                 h3_exec_info* info);

/* Rank k's rows of the gated reduce-scatter (h3_ragged_reduce_scatter_gated
 * with one rank per GPU): out [T_k, C] = bf16_rne(x + gate[seg(t)] * y) for
 * t = ts_k + t', y = rank k's reduce-scatter rows; x [T_k, C] this rank's
 * residual (out == x runs in place); gate [S, C] and seg_bounds [S+1] (host,
 * global packed bounds, 0 = b_0 < ... < b_S = T, S <= H3RR_MAX_GATE_SEGMENTS)
 * as in the one-GPU call.  Inside, the segments are clipped to [ts_k, te_k)
 * and rebased ("Distributed H3 Execution", "Partition Contract"), as
 * h3_partition reports them for rank k. */
H3RR_API h3_status h3_ragged_reduce_scatter_gated_rank(const void* const* partials,
                                                       const void* bias, const void* gate,
                                                       const int64_t* seg_bounds, int32_t n_segs,
                                                       const void* x, void* out,
                                                       int64_t n_tokens, int64_t cols,
                                                       int32_t world, int32_t rank, void* stream,
                                                       const h3_launch_config* cfg,
                                                       h3_exec_info* info);

/* Rank k's copy of the ragged all-gather: out [T, C] (this GPU) gets every
 * rank's rows, out[t, c] = in[r(t)][t - ts_{r(t)}, c], from in[world]
 * ([T_r, C] each). */
H3RR_API h3_status h3_ragged_all_gather_rank(const void* const* in, void* out, int64_t n_tokens,
                                             int64_t cols, int32_t world, int32_t rank,
                                             void* stream, const h3_launch_config* cfg,
                                             h3_exec_info* info);

/*
 * CUDA IPC for the pointer arrays above.  h3_ipc_export describes the
 * device buffer at `ptr` (any address inside a cudaMalloc allocation of the
 * current device): the allocation's IPC handle and the buffer's offset in
 * it.  Send the struct to the peers by any means (it is plain bytes).
 * h3_ipc_open maps a peer's buffer into this process on the current device
 * (peer access enabled lazily) and returns its address; h3_ipc_close unmaps
 * it (same pointer and struct).  Mappings are counted per device and
 * allocation: buffers that share an allocation share one mapping, which the
 * last close releases (a close that matches no open: H3_ERR_INVALID_ARG).
 * A process cannot open its own handles.  Close only after the last kernel
 * reading the mapping has finished.  Memory from virtual-memory-management
 * allocators (cuMemCreate, expandable segments) has no IPC handle: export
 * returns H3_ERR_CUDA.  NULL arguments: H3_ERR_INVALID_ARG.
 */
#define H3_IPC_HANDLE_BYTES 64
typedef struct h3_ipc_handle {
    unsigned char handle[H3_IPC_HANDLE_BYTES]; /* cudaIpcMemHandle_t of the allocation */
    int64_t offset;                            /* buffer address - allocation base */
    int64_t alloc_bytes;                       /* size of the allocation */
} h3_ipc_handle;
H3RR_API h3_status h3_ipc_export(const void* ptr, h3_ipc_handle* out);
H3RR_API h3_status h3_ipc_open(const h3_ipc_handle* handle, void** ptr);
H3RR_API h3_status h3_ipc_close(void* ptr, const h3_ipc_handle* handle);

#ifdef __cplusplus
}
#endif

#endif /* H3RR_H */
