// C ABI entry points for one rank per GPU (include/h3rr.h, "One rank per
// GPU"): rank k's share of each operation, pulled from every rank's buffer.
//
// "Distributed H3 Execution", "Remaining GPU Gates": the real collective at
// 2-8 GPUs must give what the single-GPU path gives.  Each rank call below
// writes exactly rank k's part of the one-GPU call's output:
//
//   seq->head  rank k's [T, P, H_k, D] head-side buffer; a kernel of its own
//              (one contiguous run of H_k heads per (t, p) row).
//   head->seq  rank k's [T_k, P, H, D] rows: the one-GPU head->seq kernel run
//              over a single-rank token split of T_k tokens, with every
//              head-side pointer advanced to row (ts_k, 0).
//   reduce     rank k's [T_k, C] rows: the one-GPU reduce-scatter kernel over
//              a single-rank split, every partial advanced to row ts_k.
//   all-gather rank k's [T, C]: the one-GPU all-gather kernel writing one
//              output.
//   gated      rank k's [T_k, C]: the one-GPU gated kernel over the one-rank
//              split, with the segments clipped to [ts_k, te_k) and rebased
//              (the partition contract's per-rank segments) and the gate
//              pointer advanced to the first of them: a rank's token range
//              meets consecutive segments, so local piece i is segment
//              s_0 + i.
//
// Inputs may be on other GPUs (mapped with h3_ipc_open); the kernels read them
// with plain vector loads.  All checks run before anything is enqueued.
#include <cstring>

#include "h3rr_internal.h"

using namespace h3rr;

namespace {

h3_status fail(cudaError_t err) { return record_cuda_failure(err); }

void fill_info(h3_exec_info* info, int launches, int chunks, const LaunchShape& shape,
               int planes_per_launch)
{
    if (!info)
        return;
    info->launches = launches;
    info->chunks = chunks;
    info->grid = shape.grid;
    info->block = shape.block;
    info->variant = shape.variant;
    info->planes_per_launch = planes_per_launch;
}

// Checks of a relayout rank call; on success *ch is the call's launch plan.
h3_status check_relayout_rank(bool seq_to_head, const void* const* send, const void* recv,
                              int64_t n_tokens, int32_t planes, int32_t n_heads, int32_t head_dim,
                              int32_t world, int32_t rank, int64_t window_bytes,
                              const h3_launch_config* cfg, RelayoutChunks* ch)
{
    if (window_bytes < 0)
        return H3_ERR_INVALID_ARG;
    if (cfg && cfg->variant == H3_VARIANT_BULK)
        return H3_ERR_UNSUPPORTED;
    if (cfg && cfg->variant != 0 && cfg->variant != H3_VARIANT_VECTOR)
        return H3_ERR_INVALID_ARG;
    if (!config_ok(cfg, H3_LAUNCH_SERIAL | H3_LAUNCH_CHUNK_TOKENS))
        return H3_ERR_INVALID_ARG;
    h3_status st = check_world(n_tokens, n_heads, world);
    if (st != H3_OK)
        return st;
    if (rank < 0 || rank >= world || !send || !recv)
        return H3_ERR_INVALID_ARG;
    st = check_relayout_sizes(n_tokens, planes, n_heads, head_dim);
    if (st != H3_OK)
        return st;
    const Split ts = make_split(n_tokens, world);
    const Split hs = make_split(n_heads, world);
    const uint64_t row_bytes = uint64_t(n_heads) * head_dim * 2;
    const uint64_t head_bytes = uint64_t(head_dim) * 2;
    uint64_t in_bytes[kMaxWorld];
    for (int r = 0; r < world; ++r) {
        if (!send[r])
            return H3_ERR_INVALID_ARG;
        if (!aligned16(send[r]))
            return H3_ERR_MISALIGNED;
        in_bytes[r] = seq_to_head ? uint64_t(ts.size(r)) * planes * row_bytes
                                  : uint64_t(n_tokens) * planes * uint64_t(hs.size(r)) * head_bytes;
    }
    if (!aligned16(recv))
        return H3_ERR_MISALIGNED;
    const uint64_t out_bytes = seq_to_head
                                   ? uint64_t(n_tokens) * planes * uint64_t(hs.size(rank)) * head_bytes
                                   : uint64_t(ts.size(rank)) * planes * row_bytes;
    void* out[1] = {const_cast<void*>(recv)};
    st = check_no_overlap(send, in_bytes, world, out, &out_bytes, 1);
    if (st != H3_OK)
        return st;
    // The window bounds every rank's slices, exactly as in the one-GPU call,
    // so that all ranks chunk alike.
    return plan_relayout(ts, hs, n_tokens, planes, row_bytes, head_bytes, window_bytes,
                         token_range_chunks(cfg), ch);
}

// Inputs one rank call may check: W partials, the gate rows, the residual
// and the bias.
constexpr int kMaxRankInputs = kMaxWorld + 3;

// Checks of a reduce-scatter or all-gather rank call (rows of `cols` BF16):
// n_in inputs of in_rows[i] rows each, plus one optional row (extra_in).
h3_status check_rows_rank(const void* const* in, const uint64_t* in_rows, const void* extra_in,
                          const void* out, uint64_t out_rows, int64_t cols, int32_t n_in_rows)
{
    if (n_in_rows < 0 || n_in_rows + (extra_in ? 1 : 0) > kMaxRankInputs)
        return H3_ERR_INVALID_ARG;
    const uint64_t row_bytes = uint64_t(cols) * 2;
    const void* inputs[kMaxRankInputs];
    uint64_t in_bytes[kMaxRankInputs];
    for (int r = 0; r < n_in_rows; ++r) {
        if (!in[r])
            return H3_ERR_INVALID_ARG;
        if (!aligned16(in[r]))
            return H3_ERR_MISALIGNED;
        inputs[r] = in[r];
        in_bytes[r] = in_rows[r] * row_bytes;
    }
    int n_in = n_in_rows;
    if (extra_in) {
        if (!aligned16(extra_in))
            return H3_ERR_MISALIGNED;
        inputs[n_in] = extra_in;
        in_bytes[n_in] = row_bytes;
        ++n_in;
    }
    if (!aligned16(out))
        return H3_ERR_MISALIGNED;
    void* outs[1] = {const_cast<void*>(out)};
    const uint64_t out_bytes = out_rows * row_bytes;
    return check_no_overlap(inputs, in_bytes, n_in, outs, &out_bytes, 1);
}

h3_status check_cols(int64_t n_tokens, int64_t cols, int32_t world, int32_t rank,
                     const void* in, const void* out)
{
    h3_status st = check_world(n_tokens, world, world);
    if (st != H3_OK)
        return st;
    if (cols < 1 || !in || !out || rank < 0 || rank >= world)
        return H3_ERR_INVALID_ARG;
    if (cols % 8 != 0)
        return H3_ERR_MISALIGNED;
    if (rows_beyond_limits(n_tokens, cols))
        return H3_ERR_UNSUPPORTED;
    return H3_OK;
}

}  // namespace

extern "C" {

h3_status h3_seq_to_head_rank(const void* const* send, void* recv, int64_t n_tokens,
                              int32_t planes, int32_t n_heads, int32_t head_dim, int32_t world,
                              int32_t rank, int64_t window_bytes, void* stream,
                              const h3_launch_config* cfg, h3_exec_info* info)
{
    clear_info(info);
    RelayoutChunks ch;
    h3_status st = check_relayout_rank(true, send, recv, n_tokens, planes, n_heads, head_dim, world,
                                       rank, window_bytes, cfg, &ch);
    if (st != H3_OK)
        return st;
    const Split ts = make_split(n_tokens, world);
    const Split hs = make_split(n_heads, world);
    const int64_t head_vecs = int64_t(head_dim) * 2 / kVecBytes;
    PullArgs a;
    std::memset(&a, 0, sizeof(a));
    for (int r = 0; r < world; ++r)
        a.src[r] = static_cast<const char*>(send[r]);
    a.dst = static_cast<char*>(recv);
    a.W = world;
    a.T = int32_t(n_tokens);
    a.P = planes;
    a.tq = int32_t(ts.q);
    a.tm = int32_t(ts.m);
    a.row_vecs = int32_t(int64_t(n_heads) * head_vecs);
    a.run_vecs = int32_t(hs.size(rank) * head_vecs);
    a.col0_vecs = int32_t(hs.start(rank) * head_vecs);
    const int plane_groups = ch.plane_groups;
    const int per_launch = ch.per_launch;
    const int chunks = int(plane_groups * ch.per_group);
    const bool programmatic = programmatic_launch(cfg);
    LaunchShape shape;
    int launched = 0;
    for (int g = 0; g < plane_groups; ++g) {
        for (int64_t c = 0; c < ch.per_group; ++c) {
            int64_t cq = 0, cm = 0, t0 = 0;
            chunk_split(ts, ch, c, &cq, &cm, &t0);
            a.cq = int32_t(cq);
            a.cm = int32_t(cm);
            a.t0 = int32_t(t0);
            a.plane0 = g * per_launch;
            a.nplanes = per_launch;
            a.rows = int32_t((cq * world + cm) * per_launch);
            a.wait_late = launched > 0 ? 1 : 0;  // chunks are disjoint (see h3_launch_config)
            const cudaError_t err = launch_pull_seq_to_head(a, cfg ? cfg->ctas_per_sm : 0,
                                                            static_cast<cudaStream_t>(stream),
                                                            &shape, programmatic);
            if (err != cudaSuccess) {
                fill_info(info, launched, chunks, shape, per_launch);
                return fail(err);
            }
            ++launched;
        }
    }
    fill_info(info, launched, chunks, shape, per_launch);
    return H3_OK;
}

h3_status h3_head_to_seq_rank(const void* const* send, void* recv, int64_t n_tokens,
                              int32_t planes, int32_t n_heads, int32_t head_dim, int32_t world,
                              int32_t rank, int64_t window_bytes, void* stream,
                              const h3_launch_config* cfg, h3_exec_info* info)
{
    clear_info(info);
    RelayoutChunks ch;
    h3_status st = check_relayout_rank(false, send, recv, n_tokens, planes, n_heads, head_dim,
                                       world, rank, window_bytes, cfg, &ch);
    if (st != H3_OK)
        return st;
    const Split ts = make_split(n_tokens, world);
    const Split hs = make_split(n_heads, world);
    const int64_t head_bytes = int64_t(head_dim) * 2;
    const int64_t t_start = ts.start(rank);
    const int64_t t_rows = ts.size(rank);
    // A one-rank token split of T_k tokens: every row belongs to "rank 0",
    // whose sequence-side buffer is this rank's; head-side row (t', p) of the
    // advanced pointers is global row (ts_k + t', p).
    RelayoutArgs a;
    std::memset(&a, 0, sizeof(a));
    a.seq[0] = static_cast<char*>(recv);
    for (int j = 0; j < world; ++j)
        a.head[j] = const_cast<char*>(static_cast<const char*>(send[j])) +
                    t_start * planes * hs.size(j) * head_bytes;
    a.T = int32_t(t_rows);
    a.P = planes;
    a.W = world;
    a.tq = int32_t(t_rows);
    a.tm = 0;
    a.hq = int32_t(hs.q);
    a.hm = int32_t(hs.m);
    a.row_vecs = int32_t(int64_t(n_heads) * head_bytes / kVecBytes);
    a.head_vecs = int32_t(head_bytes / kVecBytes);
    const int plane_groups = ch.plane_groups;
    const int per_launch = ch.per_launch;
    const int chunks = int(plane_groups * ch.per_group);
    const bool programmatic = programmatic_launch(cfg);
    const int variant = cfg ? cfg->variant : 0;
    LaunchShape shape;
    int launched = 0;
    for (int g = 0; g < plane_groups; ++g) {
        for (int64_t c = 0; c < ch.per_group; ++c) {
            // This rank's tokens of chunk c of the plan all ranks share; the
            // last chunk may hold none of them.
            const int64_t t0 = c * ch.tokens;
            int64_t n = t_rows - t0;
            if (n > ch.tokens)
                n = ch.tokens;
            if (n <= 0)
                continue;
            a.cq = int32_t(n);
            a.cm = 0;
            a.t0 = int32_t(t0);
            a.plane0 = g * per_launch;
            a.nplanes = per_launch;
            a.rows = int32_t(n * per_launch);
            a.wait_late = launched > 0 ? 1 : 0;
            const cudaError_t err =
                launch_relayout(false, a, variant, cfg ? cfg->ctas_per_sm : 0,
                                static_cast<cudaStream_t>(stream), &shape, false, programmatic);
            if (err != cudaSuccess) {
                fill_info(info, launched, chunks, shape, per_launch);
                return fail(err);
            }
            ++launched;
        }
    }
    fill_info(info, launched, chunks, shape, per_launch);
    return H3_OK;
}

h3_status h3_ragged_reduce_scatter_rank(const void* const* partials, const void* bias, void* out,
                                        int64_t n_tokens, int64_t cols, int32_t world,
                                        int32_t rank, void* stream, const h3_launch_config* cfg,
                                        h3_exec_info* info)
{
    clear_info(info);
    h3_status st = check_cols(n_tokens, cols, world, rank, partials, out);
    if (st != H3_OK)
        return st;
    if (cfg && cfg->variant != 0 && cfg->variant != H3_VARIANT_REDUCE)
        return H3_ERR_INVALID_ARG;
    if (!config_ok(cfg))
        return H3_ERR_INVALID_ARG;
    const Split ts = make_split(n_tokens, world);
    uint64_t in_rows[kMaxWorld] = {};
    for (int r = 0; r < world; ++r)
        in_rows[r] = uint64_t(n_tokens);
    st = check_rows_rank(partials, in_rows, bias, out, uint64_t(ts.size(rank)), cols, world);
    if (st != H3_OK)
        return st;
    const int64_t row_bytes = cols * 2;
    const int64_t t_rows = ts.size(rank);
    ReduceArgs a;
    std::memset(&a, 0, sizeof(a));
    for (int r = 0; r < world; ++r)
        a.part[r] = static_cast<const char*>(partials[r]) + ts.start(rank) * row_bytes;
    a.out[0] = static_cast<char*>(out);
    a.bias = static_cast<const char*>(bias);
    a.T = int32_t(t_rows);
    a.W = world;
    a.tq = int32_t(t_rows);  // one-rank split: every row is this rank's
    a.tm = 0;
    a.row_vecs = int32_t(cols / 8);
    a.row_bytes = row_bytes;
    LaunchShape shape;
    const cudaError_t err =
        launch_reduce_scatter(a, cfg ? cfg->ctas_per_sm : 0, static_cast<cudaStream_t>(stream),
                              &shape, programmatic_launch(cfg));
    if (err != cudaSuccess)
        return fail(err);
    fill_info(info, 1, 1, shape, 1);
    return H3_OK;
}

h3_status h3_ragged_reduce_scatter_gated_rank(const void* const* partials, const void* bias,
                                              const void* gate, const int64_t* seg_bounds,
                                              int32_t n_segs, const void* x, void* out,
                                              int64_t n_tokens, int64_t cols, int32_t world,
                                              int32_t rank, void* stream,
                                              const h3_launch_config* cfg, h3_exec_info* info)
{
    clear_info(info);
    h3_status st = check_cols(n_tokens, cols, world, rank, partials, out);
    if (st != H3_OK)
        return st;
    if (!x || !gate || !seg_bounds)
        return H3_ERR_INVALID_ARG;
    if (cfg && cfg->variant != 0 && cfg->variant != H3_VARIANT_REDUCE_GATED)
        return H3_ERR_INVALID_ARG;
    if (!config_ok(cfg))
        return H3_ERR_INVALID_ARG;
    if (n_segs < 1 || n_segs > H3RR_MAX_GATE_SEGMENTS)
        return n_segs < 1 ? H3_ERR_INVALID_ARG : H3_ERR_UNSUPPORTED;
    if (seg_bounds[0] != 0 || seg_bounds[n_segs] != n_tokens)
        return H3_ERR_INVALID_ARG;
    for (int32_t k = 0; k < n_segs; ++k)
        if (seg_bounds[k + 1] <= seg_bounds[k])
            return H3_ERR_INVALID_ARG;
    if (!aligned16(gate) || !aligned16(x))
        return H3_ERR_MISALIGNED;
    const Split ts = make_split(n_tokens, world);
    const int64_t row_bytes = cols * 2;
    const int64_t t0 = ts.start(rank);
    const int64_t t_rows = ts.size(rank);
    // Inputs: partials, gate and (unless in place) x; the bias rides along.
    const void* ins[kMaxRankInputs];
    uint64_t in_rows[kMaxRankInputs];
    int n_in = 0;
    for (int r = 0; r < world; ++r) {
        ins[n_in] = partials[r];
        in_rows[n_in++] = uint64_t(n_tokens);
    }
    ins[n_in] = gate;
    in_rows[n_in++] = uint64_t(n_segs);
    if (x != out) {
        ins[n_in] = x;
        in_rows[n_in++] = uint64_t(t_rows);
    }
    st = check_rows_rank(ins, in_rows, bias, out, uint64_t(t_rows), cols, n_in);
    if (st != H3_OK)
        return st;
    int64_t local_bounds[kMaxGateSegs + 1];
    int32_t seg_ids[kMaxGateSegs];
    const int32_t pieces = clip_segments(seg_bounds, n_segs, t0, t0 + t_rows, local_bounds, seg_ids);
    GatedArgs g;
    std::memset(&g, 0, sizeof(g));
    for (int r = 0; r < world; ++r)
        g.r.part[r] = static_cast<const char*>(partials[r]) + t0 * row_bytes;
    g.r.out[0] = static_cast<char*>(out);
    g.x[0] = static_cast<const char*>(x);
    g.r.bias = static_cast<const char*>(bias);
    g.r.T = int32_t(t_rows);
    g.r.W = world;
    g.r.tq = int32_t(t_rows);
    g.r.tm = 0;
    g.r.row_vecs = int32_t(cols / 8);
    g.r.row_bytes = row_bytes;
    g.gate = static_cast<const char*>(gate) + int64_t(seg_ids[0]) * row_bytes;
    g.n_segs = pieces;
    for (int32_t i = 0; i <= pieces; ++i)
        g.seg_bounds[i] = int32_t(local_bounds[i]);
    LaunchShape shape;
    const cudaError_t err = launch_reduce_scatter_gated(g, static_cast<cudaStream_t>(stream), &shape,
                                                        programmatic_launch(cfg));
    if (err != cudaSuccess)
        return fail(err);
    fill_info(info, 1, 1, shape, 1);
    return H3_OK;
}

h3_status h3_ragged_all_gather_rank(const void* const* in, void* out, int64_t n_tokens,
                                    int64_t cols, int32_t world, int32_t rank, void* stream,
                                    const h3_launch_config* cfg, h3_exec_info* info)
{
    clear_info(info);
    h3_status st = check_cols(n_tokens, cols, world, rank, in, out);
    if (st != H3_OK)
        return st;
    if (cfg && cfg->variant == H3_VARIANT_BULK)
        return H3_ERR_UNSUPPORTED;
    if (cfg && cfg->variant != 0 && cfg->variant != H3_VARIANT_VECTOR)
        return H3_ERR_INVALID_ARG;
    if (!config_ok(cfg))
        return H3_ERR_INVALID_ARG;
    const Split ts = make_split(n_tokens, world);
    uint64_t in_rows[kMaxWorld] = {};
    for (int r = 0; r < world; ++r)
        in_rows[r] = uint64_t(ts.size(r));
    st = check_rows_rank(in, in_rows, nullptr, out, uint64_t(n_tokens), cols, world);
    if (st != H3_OK)
        return st;
    GatherArgs a;
    std::memset(&a, 0, sizeof(a));
    for (int r = 0; r < world; ++r)
        a.in[r] = static_cast<const char*>(in[r]);
    a.out[0] = static_cast<char*>(out);
    a.T = int32_t(n_tokens);
    a.W = 1;  // one output: this rank's
    a.n_in = world;
    a.tq = int32_t(ts.q);
    a.tm = int32_t(ts.m);
    a.row_vecs = int32_t(cols / 8);
    a.row_bytes = cols * 2;
    LaunchShape shape;
    const cudaError_t err =
        launch_all_gather(a, 0, cfg ? cfg->ctas_per_sm : 0, static_cast<cudaStream_t>(stream),
                          &shape, programmatic_launch(cfg));
    if (err != cudaSuccess)
        return fail(err);
    fill_info(info, 1, 1, shape, 1);
    return H3_OK;
}

}  // extern "C"
