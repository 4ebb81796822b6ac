// C ABI entry points (include/h3rr.h): argument checks, the launch plan and
// the kernel launches.  Every check runs before anything is enqueued; on an
// error nothing is launched.
#include <climits>
#include <cstring>

#include "h3rr_internal.h"

using namespace h3rr;

namespace {

// CUDA error behind the calling thread's most recent H3_ERR_CUDA.
thread_local int t_last_cuda_error = 0;

h3_status cuda_failure(cudaError_t err)
{
    t_last_cuda_error = int(err);
    cudaGetLastError();  // clear a non-sticky launch error
    return H3_ERR_CUDA;
}

}  // namespace

namespace h3rr {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

void clear_info(h3_exec_info* info)
{
    if (info)
        std::memset(info, 0, sizeof(*info));
}

// Launch-config fields every entry point checks the same way.
bool config_ok(const h3_launch_config* cfg, int32_t allowed)
{
    return !cfg || (cfg->ctas_per_sm >= 0 && (cfg->flags & ~allowed) == 0 && cfg->reserved1 == 0);
}

bool token_range_chunks(const h3_launch_config* cfg) { return cfg && (cfg->flags & H3_LAUNCH_CHUNK_TOKENS); }

bool rows_beyond_limits(int64_t n_tokens, int64_t cols)
{
    return n_tokens > kMaxInt32 || cols / 8 > kMaxRowVecs ||
           n_tokens > int64_t(kMaxSideBytes / uint64_t(cols * 2));
}

h3_status check_relayout_sizes(int64_t n_tokens, int32_t planes, int32_t n_heads, int32_t head_dim)
{
    if (planes < 1 || head_dim < 1 || n_heads < 1 || n_tokens < 1)
        return H3_ERR_INVALID_ARG;
    if ((int64_t(head_dim) * 2) % kVecBytes != 0)
        return H3_ERR_MISALIGNED;
    const int64_t row_bytes = int64_t(n_heads) * head_dim * 2;
    if (n_tokens > kMaxInt32 || n_tokens * planes > kMaxInt32 || row_bytes / kVecBytes > kMaxRowVecs)
        return H3_ERR_UNSUPPORTED;
    // Every side of the relayout is T*P rows of row_bytes; bounding it keeps
    // every byte count of the checks and the launch plan within 64 bits
    // (the plan multiplies it by at most the rank count).
    if (n_tokens * planes > int64_t(kMaxSideBytes / uint64_t(row_bytes)))
        return H3_ERR_UNSUPPORTED;
    return H3_OK;
}

bool programmatic_launch(const h3_launch_config* cfg) { return !(cfg && (cfg->flags & H3_LAUNCH_SERIAL)); }

// Partition checks shared by the relayouts and the reduce-scatter
// ("Distributed H3 Execution", intro: empty token or head partitions are
// rejected).
h3_status check_world(int64_t n_tokens, int64_t n_heads, int32_t world)
{
    if (world < 1 || n_tokens < 0 || n_heads < 0)
        return H3_ERR_INVALID_ARG;
    if (world > kMaxWorld)
        return H3_ERR_UNSUPPORTED;
    if (n_tokens < world || n_heads < world)
        return H3_ERR_EMPTY_PARTITION;
    return H3_OK;
}

// Outputs may not overlap inputs or each other (FastVideo PR #1807, "Problem
// and behavior": outputs keep storage of their own).
h3_status check_no_overlap(const void* const* in, const uint64_t* in_bytes, int n_in,
                           void* const* out, const uint64_t* out_bytes, int n_out)
{
    for (int i = 0; i < n_out; ++i) {
        const uintptr_t o = reinterpret_cast<uintptr_t>(out[i]);
        for (int k = 0; k < n_in; ++k)
            if (ranges_overlap(o, out_bytes[i], reinterpret_cast<uintptr_t>(in[k]), in_bytes[k]))
                return H3_ERR_INVALID_ARG;
        for (int k = i + 1; k < n_out; ++k)
            if (ranges_overlap(o, out_bytes[i], reinterpret_cast<uintptr_t>(out[k]), out_bytes[k]))
                return H3_ERR_INVALID_ARG;
    }
    return H3_OK;
}

}  // namespace h3rr

namespace {

// Shared checks of the relayout calls: world, shapes, pointers, alignment,
// overlap.  `extra_out` (nullable) is one more output range (the window).
h3_status check_relayout_args(bool seq_to_head, const void* const* send, void* const* recv,
                              int64_t n_tokens, int32_t planes, int32_t n_heads, int32_t head_dim,
                              int32_t world, void* extra_out, uint64_t extra_bytes)
{
    h3_status st = check_world(n_tokens, n_heads, world);
    if (st != H3_OK)
        return st;
    if (!send || !recv)
        return H3_ERR_INVALID_ARG;
    st = check_relayout_sizes(n_tokens, planes, n_heads, head_dim);
    if (st != H3_OK)
        return st;
    const Split ts = make_split(n_tokens, world);
    const Split hs = make_split(n_heads, world);
    const uint64_t row_bytes = uint64_t(n_heads) * head_dim * 2;
    const uint64_t head_bytes = uint64_t(head_dim) * 2;
    uint64_t seq_bytes[kMaxWorld];
    uint64_t head_side_bytes[kMaxWorld + 1];
    void* outs[kMaxWorld + 1];
    for (int r = 0; r < world; ++r) {
        if (!send[r] || !recv[r])
            return H3_ERR_INVALID_ARG;
        if (!aligned16(send[r]) || !aligned16(recv[r]))
            return H3_ERR_MISALIGNED;
        seq_bytes[r] = uint64_t(ts.size(r)) * planes * row_bytes;
        head_side_bytes[r] = uint64_t(n_tokens) * planes * uint64_t(hs.size(r)) * head_bytes;
    }
    const uint64_t* in_bytes = seq_to_head ? seq_bytes : head_side_bytes;
    uint64_t out_bytes[kMaxWorld + 1];
    for (int r = 0; r < world; ++r) {
        outs[r] = recv[r];
        out_bytes[r] = seq_to_head ? head_side_bytes[r] : seq_bytes[r];
    }
    int n_out = world;
    if (extra_out) {
        outs[n_out] = extra_out;
        out_bytes[n_out] = extra_bytes;
        ++n_out;
    }
    return check_no_overlap(send, in_bytes, world, outs, out_bytes, n_out);
}

h3_status relayout(bool seq_to_head, const void* const* send, void* const* recv,
                   int64_t n_tokens, int32_t planes, int32_t n_heads, int32_t head_dim,
                   int32_t world, int64_t window_bytes, void* stream,
                   const h3_launch_config* cfg, h3_exec_info* info, int32_t layout = 0)
{
    clear_info(info);
    if (layout & ~(H3_LAYOUT_SEQ_PLANE_MAJOR | H3_LAYOUT_HEAD_PLANE_MAJOR))
        return H3_ERR_INVALID_ARG;
    if (layout != 0 && cfg && cfg->variant == H3_VARIANT_BULK)
        return H3_ERR_UNSUPPORTED;  // the bulk kernel moves token-major rows only
    if (window_bytes < 0)
        return H3_ERR_INVALID_ARG;
    if (cfg && cfg->variant != 0 && cfg->variant != H3_VARIANT_VECTOR && cfg->variant != H3_VARIANT_BULK)
        return H3_ERR_INVALID_ARG;
    if (!config_ok(cfg, H3_LAUNCH_SERIAL | H3_LAUNCH_CHUNK_TOKENS))
        return H3_ERR_INVALID_ARG;
    h3_status st = check_relayout_args(seq_to_head, send, recv, n_tokens, planes, n_heads, head_dim,
                                       world, nullptr, 0);
    if (st != H3_OK)
        return st;

    const Split ts = make_split(n_tokens, world);
    const Split hs = make_split(n_heads, world);
    const uint64_t row_bytes = uint64_t(n_heads) * head_dim * 2;  // one (token, plane) row
    const uint64_t head_bytes = uint64_t(head_dim) * 2;

    // Chunked mode (FastVideo PR #1807, "Problem and behavior"): one batch
    // plane per launch, each rank's send and receive slices within the
    // window; a plane too large for the window is split by tokens.  With
    // H3_LAUNCH_CHUNK_TOKENS the same window is cut into token ranges of
    // every plane instead.
    RelayoutChunks ch;
    st = plan_relayout(ts, hs, n_tokens, planes, row_bytes, head_bytes, window_bytes,
                       token_range_chunks(cfg), &ch);
    if (st != H3_OK)
        return st;

    RelayoutArgs a;
    std::memset(&a, 0, sizeof(a));
    for (int r = 0; r < world; ++r) {
        char* s = const_cast<char*>(static_cast<const char*>(send[r]));
        char* d = static_cast<char*>(recv[r]);
        a.seq[r] = seq_to_head ? s : d;
        a.head[r] = seq_to_head ? d : s;
    }
    a.T = int32_t(n_tokens);
    a.P = planes;
    a.W = world;
    a.tq = int32_t(ts.q);
    a.tm = int32_t(ts.m);
    a.hq = int32_t(hs.q);
    a.hm = int32_t(hs.m);
    a.row_vecs = int32_t(row_bytes / kVecBytes);
    a.head_vecs = int32_t(head_bytes / kVecBytes);
    a.seq_pm = (layout & H3_LAYOUT_SEQ_PLANE_MAJOR) ? 1 : 0;
    a.head_pm = (layout & H3_LAYOUT_HEAD_PLANE_MAJOR) ? 1 : 0;

    const int variant = cfg ? cfg->variant : 0;
    const int ctas_per_sm = cfg ? cfg->ctas_per_sm : 0;
    if (variant == H3_VARIANT_BULK) {
        int device = 0;
        const cudaError_t err = cudaGetDevice(&device);
        if (err != cudaSuccess)
            return cuda_failure(err);
        if (!relayout_bulk_fits(a, device))
            return H3_ERR_UNSUPPORTED;  // the bulk kernel's row stages do not fit in shared memory
    }
    const int plane_groups = ch.plane_groups;
    const int per_launch = ch.per_launch;
    const int chunks = int(plane_groups * ch.per_group);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    LaunchShape shape;
    int launched = 0;
    const bool programmatic = programmatic_launch(cfg);
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
            // Chunks are disjoint rows of every buffer: a later chunk's launch
            // depends on nothing the previous one does and only has to
            // finish after it.
            a.wait_late = launched > 0 ? 1 : 0;
            const cudaError_t err = launch_relayout(seq_to_head, a, variant, ctas_per_sm, s,
                                                    &shape, layout != 0, programmatic);
            if (err != cudaSuccess) {
                if (info) {
                    info->launches = launched;
                    info->chunks = chunks;
                }
                return cuda_failure(err);
            }
            ++launched;
        }
    }
    if (info) {
        info->launches = launched;
        info->chunks = chunks;
        info->grid = shape.grid;
        info->block = shape.block;
        info->variant = shape.variant;
        info->planes_per_launch = per_launch;
    }
    return H3_OK;
}

// Tokens per chunk of a staged call: as many whole token rows (H*D*2 bytes)
// as the window holds, at most T; H3_ERR_WINDOW below one row.
h3_status staged_plan(int64_t n_tokens, int32_t n_heads, int32_t head_dim, int64_t window_bytes,
                      int64_t* chunk_tokens)
{
    const int64_t row_bytes = int64_t(n_heads) * head_dim * 2;
    if (row_bytes <= 0)
        return H3_ERR_INVALID_ARG;
    if (window_bytes < row_bytes)
        return H3_ERR_WINDOW;
    int64_t n = window_bytes / row_bytes;
    if (n > n_tokens)
        n = n_tokens;
    *chunk_tokens = n;
    return H3_OK;
}

h3_status relayout_staged(bool seq_to_head, const void* const* send, void* const* recv,
                          int64_t n_tokens, int32_t planes, int32_t n_heads, int32_t head_dim,
                          int32_t world, void* window, int64_t window_bytes, void* stream,
                          h3_exec_info* info)
{
    clear_info(info);
    if (!window || window_bytes < 0)
        return H3_ERR_INVALID_ARG;
    if (!aligned16(window))
        return H3_ERR_MISALIGNED;
    h3_status st = check_relayout_args(seq_to_head, send, recv, n_tokens, planes, n_heads, head_dim,
                                       world, window, uint64_t(window_bytes));
    if (st != H3_OK)
        return st;
    int64_t chunk_tokens = 0;
    st = staged_plan(n_tokens, n_heads, head_dim, window_bytes, &chunk_tokens);
    if (st != H3_OK)
        return st;
    const Split ts = make_split(n_tokens, world);
    const Split hs = make_split(n_heads, world);
    StagedArgs a;
    std::memset(&a, 0, sizeof(a));
    for (int r = 0; r < world; ++r) {
        char* s = const_cast<char*>(static_cast<const char*>(send[r]));
        char* d = static_cast<char*>(recv[r]);
        a.seq[r] = seq_to_head ? s : d;
        a.head[r] = seq_to_head ? d : s;
    }
    a.window = static_cast<char*>(window);
    a.T = int32_t(n_tokens);
    a.P = planes;
    a.W = world;
    a.tq = int32_t(ts.q);
    a.tm = int32_t(ts.m);
    a.hq = int32_t(hs.q);
    a.hm = int32_t(hs.m);
    a.row_vecs = int32_t(int64_t(n_heads) * head_dim * 2 / kVecBytes);
    a.head_vecs = int32_t(int64_t(head_dim) * 2 / kVecBytes);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    LaunchShape shape;
    int chunks = 0;
    for (int32_t p = 0; p < planes; ++p) {
        for (int64_t t0 = 0; t0 < n_tokens; t0 += chunk_tokens) {
            a.p = p;
            a.t0 = int32_t(t0);
            a.n = int32_t(n_tokens - t0 < chunk_tokens ? n_tokens - t0 : chunk_tokens);
            const cudaError_t err = launch_staged_chunk(seq_to_head, a, s, &shape);
            if (err != cudaSuccess) {
                if (info) {
                    info->launches = 2 * chunks;
                    info->chunks = chunks;
                }
                return cuda_failure(err);
            }
            ++chunks;
        }
    }
    if (info) {
        info->launches = 2 * chunks;
        info->chunks = chunks;
        info->grid = shape.grid;
        info->block = shape.block;
        info->variant = shape.variant;
        info->planes_per_launch = 1;
    }
    return H3_OK;
}

}  // namespace

namespace h3rr {

h3_status staged_relayout_with_window(bool seq_to_head, const void* const* send, void* const* recv,
                                      int64_t n_tokens, int32_t planes, int32_t n_heads,
                                      int32_t head_dim, int32_t world, void* window,
                                      int64_t window_bytes, void* stream, h3_exec_info* info)
{
    return relayout_staged(seq_to_head, send, recv, n_tokens, planes, n_heads, head_dim, world,
                           window, window_bytes, stream, info);
}

h3_status record_cuda_failure(cudaError_t err) { return cuda_failure(err); }

}  // namespace h3rr

extern "C" {

h3_status h3_seq_to_head_staged(const void* const* send, void* const* recv, int64_t n_tokens,
                                int32_t planes, int32_t n_heads, int32_t head_dim, int32_t world,
                                void* window, int64_t window_bytes, void* stream, h3_exec_info* info)
{
    return relayout_staged(true, send, recv, n_tokens, planes, n_heads, head_dim, world, window,
                           window_bytes, stream, info);
}

h3_status h3_head_to_seq_staged(const void* const* send, void* const* recv, int64_t n_tokens,
                                int32_t planes, int32_t n_heads, int32_t head_dim, int32_t world,
                                void* window, int64_t window_bytes, void* stream, h3_exec_info* info)
{
    return relayout_staged(false, send, recv, n_tokens, planes, n_heads, head_dim, world, window,
                           window_bytes, stream, info);
}

h3_status h3_staged_plan(int64_t n_tokens, int32_t planes, int32_t n_heads, int32_t head_dim,
                         int64_t window_bytes, int64_t* chunk_tokens, int64_t* chunks)
{
    if (!chunk_tokens || !chunks || n_tokens < 1 || planes < 1 || n_heads < 1 || head_dim < 1 ||
        window_bytes < 0)
        return H3_ERR_INVALID_ARG;
    int64_t n = 0;
    const h3_status st = staged_plan(n_tokens, n_heads, head_dim, window_bytes, &n);
    if (st != H3_OK)
        return st;
    *chunk_tokens = n;
    *chunks = int64_t(planes) * ((n_tokens + n - 1) / n);
    return H3_OK;
}


h3_status h3_relayout_chunk_plan_ex(int64_t n_tokens, int32_t planes, int32_t n_heads,
                                    int32_t head_dim, int32_t world, int64_t window_bytes,
                                    int32_t flags, int64_t* tokens_per_chunk, int64_t* chunks,
                                    int32_t* planes_per_launch)
{
    if (!tokens_per_chunk || !chunks || planes < 1 || head_dim < 1 || window_bytes < 0 ||
        (flags & ~(H3_LAUNCH_SERIAL | H3_LAUNCH_CHUNK_TOKENS)) != 0)
        return H3_ERR_INVALID_ARG;
    h3_status st = check_world(n_tokens, n_heads, world);
    if (st != H3_OK)
        return st;
    st = check_relayout_sizes(n_tokens, planes, n_heads, head_dim);
    if (st != H3_OK)
        return st;
    const Split ts = make_split(n_tokens, world);
    const Split hs = make_split(n_heads, world);
    RelayoutChunks ch;
    const h3_status pst = plan_relayout(ts, hs, n_tokens, planes, uint64_t(n_heads) * head_dim * 2,
                                        uint64_t(head_dim) * 2, window_bytes,
                                        (flags & H3_LAUNCH_CHUNK_TOKENS) != 0, &ch);
    if (pst != H3_OK)
        return pst;
    *tokens_per_chunk = ch.tokens;
    *chunks = int64_t(ch.plane_groups) * ch.per_group;
    if (planes_per_launch)
        *planes_per_launch = ch.per_launch;
    return H3_OK;
}

h3_status h3_relayout_chunk_plan(int64_t n_tokens, int32_t planes, int32_t n_heads,
                                 int32_t head_dim, int32_t world, int64_t window_bytes,
                                 int64_t* tokens_per_chunk, int64_t* chunks)
{
    return h3_relayout_chunk_plan_ex(n_tokens, planes, n_heads, head_dim, world, window_bytes, 0,
                                     tokens_per_chunk, chunks, nullptr);
}

int32_t h3_abi_version(void) { return H3RR_ABI_VERSION; }

int32_t h3_last_cuda_error(const char** message)
{
    if (message)
        *message = t_last_cuda_error ? cudaGetErrorString(cudaError_t(t_last_cuda_error)) : "no error";
    return t_last_cuda_error;
}

const char* h3_status_string(h3_status status)
{
    switch (status) {
        case H3_OK: return "ok";
        case H3_ERR_INVALID_ARG: return "invalid argument";
        case H3_ERR_EMPTY_PARTITION: return "empty token or head partition";
        case H3_ERR_MISALIGNED: return "pointer or run not 16-byte aligned";
        case H3_ERR_WINDOW: return "the byte window cannot hold the data of one token";
        case H3_ERR_UNSUPPORTED: return "unsupported size or world";
        case H3_ERR_CUDA: return "CUDA launch error";
    }
    return "unknown status";
}

h3_status h3_partition(int64_t n_tokens, int32_t n_heads, int32_t world,
                       const int64_t* seg_bounds, int32_t n_segs, int64_t* token_starts,
                       int32_t* head_starts, int64_t* local_bounds, int32_t* local_seg_ids,
                       int32_t* piece_offsets)
{
    h3_status st = check_world(n_tokens, n_heads, world);
    if (st != H3_OK)
        return st;
    if (!token_starts || !head_starts || n_segs < 0)
        return H3_ERR_INVALID_ARG;
    if (n_segs > 0) {
        if (!seg_bounds || !local_bounds || !local_seg_ids || !piece_offsets)
            return H3_ERR_INVALID_ARG;
        if (seg_bounds[0] != 0 || seg_bounds[n_segs] != n_tokens)
            return H3_ERR_INVALID_ARG;
        for (int32_t k = 0; k < n_segs; ++k)
            if (seg_bounds[k + 1] <= seg_bounds[k])
                return H3_ERR_INVALID_ARG;
    }
    const Split ts = make_split(n_tokens, world);
    const Split hs = make_split(n_heads, world);
    for (int32_t r = 0; r <= world; ++r) {
        token_starts[r] = ts.start(r);
        head_starts[r] = int32_t(hs.start(r));
    }
    if (n_segs == 0)
        return H3_OK;
    int32_t pieces = 0;
    for (int32_t r = 0; r < world; ++r) {
        piece_offsets[r] = pieces;
        pieces += clip_segments(seg_bounds, n_segs, token_starts[r], token_starts[r + 1],
                                local_bounds + pieces + r, local_seg_ids + pieces);
    }
    piece_offsets[world] = pieces;
    return H3_OK;
}

h3_status h3_seq_to_head_ex(const void* const* send, void* const* recv, int64_t n_tokens,
                            int32_t planes, int32_t n_heads, int32_t head_dim, int32_t world,
                            int64_t window_bytes, void* stream, const h3_launch_config* cfg,
                            h3_exec_info* info)
{
    return relayout(true, send, recv, n_tokens, planes, n_heads, head_dim, world, window_bytes,
                    stream, cfg, info);
}

h3_status h3_head_to_seq_ex(const void* const* send, void* const* recv, int64_t n_tokens,
                            int32_t planes, int32_t n_heads, int32_t head_dim, int32_t world,
                            int64_t window_bytes, void* stream, const h3_launch_config* cfg,
                            h3_exec_info* info)
{
    return relayout(false, send, recv, n_tokens, planes, n_heads, head_dim, world, window_bytes,
                    stream, cfg, info);
}

h3_status h3_seq_to_head_layout(const void* const* send, void* const* recv, int64_t n_tokens,
                                int32_t planes, int32_t n_heads, int32_t head_dim, int32_t world,
                                int64_t window_bytes, int32_t layout, void* stream,
                                const h3_launch_config* cfg, h3_exec_info* info)
{
    return relayout(true, send, recv, n_tokens, planes, n_heads, head_dim, world, window_bytes,
                    stream, cfg, info, layout);
}

h3_status h3_head_to_seq_layout(const void* const* send, void* const* recv, int64_t n_tokens,
                                int32_t planes, int32_t n_heads, int32_t head_dim, int32_t world,
                                int64_t window_bytes, int32_t layout, void* stream,
                                const h3_launch_config* cfg, h3_exec_info* info)
{
    return relayout(false, send, recv, n_tokens, planes, n_heads, head_dim, world, window_bytes,
                    stream, cfg, info, layout);
}

h3_status h3_seq_to_head(const void* const* send, void* const* recv, int64_t n_tokens,
                         int32_t planes, int32_t n_heads, int32_t head_dim, int32_t world,
                         int64_t window_bytes, void* stream, h3_exec_info* info)
{
    return relayout(true, send, recv, n_tokens, planes, n_heads, head_dim, world, window_bytes,
                    stream, nullptr, info);
}

h3_status h3_head_to_seq(const void* const* send, void* const* recv, int64_t n_tokens,
                         int32_t planes, int32_t n_heads, int32_t head_dim, int32_t world,
                         int64_t window_bytes, void* stream, h3_exec_info* info)
{
    return relayout(false, send, recv, n_tokens, planes, n_heads, head_dim, world, window_bytes,
                    stream, nullptr, info);
}

h3_status h3_ragged_reduce_scatter_ex(const void* const* partials, const void* bias,
                                      void* const* out, int64_t n_tokens, int64_t cols,
                                      int32_t world, void* stream, const h3_launch_config* cfg,
                                      h3_exec_info* info)
{
    clear_info(info);
    h3_status st = check_world(n_tokens, world, world);
    if (st != H3_OK)
        return st;
    if (cols < 1 || !partials || !out)
        return H3_ERR_INVALID_ARG;
    if (cfg && (cfg->variant != 0 && cfg->variant != H3_VARIANT_REDUCE))
        return H3_ERR_INVALID_ARG;
    if (!config_ok(cfg))
        return H3_ERR_INVALID_ARG;
    if (cols % 8 != 0)
        return H3_ERR_MISALIGNED;
    if (rows_beyond_limits(n_tokens, cols))
        return H3_ERR_UNSUPPORTED;
    const Split ts = make_split(n_tokens, world);
    const uint64_t row_bytes = uint64_t(cols) * 2;
    uint64_t in_bytes[kMaxWorld + 1];
    uint64_t out_bytes[kMaxWorld];
    const void* inputs[kMaxWorld + 1];
    for (int r = 0; r < world; ++r) {
        if (!partials[r] || !out[r])
            return H3_ERR_INVALID_ARG;
        if (!aligned16(partials[r]) || !aligned16(out[r]))
            return H3_ERR_MISALIGNED;
        inputs[r] = partials[r];
        in_bytes[r] = uint64_t(n_tokens) * row_bytes;
        out_bytes[r] = uint64_t(ts.size(r)) * row_bytes;
    }
    int n_in = world;
    if (bias) {
        if (!aligned16(bias))
            return H3_ERR_MISALIGNED;
        inputs[n_in] = bias;
        in_bytes[n_in] = row_bytes;
        ++n_in;
    }
    st = check_no_overlap(inputs, in_bytes, n_in, out, out_bytes, world);
    if (st != H3_OK)
        return st;

    ReduceArgs a;
    std::memset(&a, 0, sizeof(a));
    for (int r = 0; r < world; ++r) {
        a.part[r] = static_cast<const char*>(partials[r]);
        a.out[r] = static_cast<char*>(out[r]);
    }
    a.bias = static_cast<const char*>(bias);
    a.T = int32_t(n_tokens);
    a.W = world;
    a.tq = int32_t(ts.q);
    a.tm = int32_t(ts.m);
    a.row_vecs = int32_t(cols / 8);
    a.row_bytes = int64_t(row_bytes);
    LaunchShape shape;
    const cudaError_t err = launch_reduce_scatter(a, cfg ? cfg->ctas_per_sm : 0,
                                                  static_cast<cudaStream_t>(stream), &shape,
                                                  programmatic_launch(cfg));
    if (err != cudaSuccess)
        return cuda_failure(err);
    if (info) {
        info->launches = 1;
        info->chunks = 1;
        info->grid = shape.grid;
        info->block = shape.block;
        info->variant = shape.variant;
        info->planes_per_launch = 1;
    }
    return H3_OK;
}

h3_status h3_bulk_wait_timeouts(void* stream, uint32_t* count, int32_t reset)
{
    if (!count)
        return H3_ERR_INVALID_ARG;
    unsigned int v = 0, g = 0;
    cudaError_t err = read_bulk_wait_timeouts(&v, reset != 0, static_cast<cudaStream_t>(stream));
    if (err == cudaSuccess)
        err = read_gather_wait_timeouts(&g, reset != 0, static_cast<cudaStream_t>(stream));
    if (err != cudaSuccess)
        return cuda_failure(err);
    *count = v + g;
    return H3_OK;
}

h3_status h3_ragged_all_gather(const void* const* in, void* const* out, int64_t n_tokens,
                               int64_t cols, int32_t world, void* stream, h3_exec_info* info)
{
    return h3_ragged_all_gather_ex(in, out, n_tokens, cols, world, stream, nullptr, info);
}

h3_status h3_ragged_all_gather_ex(const void* const* in, void* const* out, int64_t n_tokens,
                                  int64_t cols, int32_t world, void* stream,
                                  const h3_launch_config* cfg, h3_exec_info* info)
{
    clear_info(info);
    h3_status st = check_world(n_tokens, world, world);
    if (st != H3_OK)
        return st;
    if (cols < 1 || !in || !out)
        return H3_ERR_INVALID_ARG;
    if (cfg && cfg->variant != 0 && cfg->variant != H3_VARIANT_VECTOR && cfg->variant != H3_VARIANT_BULK)
        return H3_ERR_INVALID_ARG;
    if (!config_ok(cfg))
        return H3_ERR_INVALID_ARG;
    if (cols % 8 != 0)
        return H3_ERR_MISALIGNED;
    if (rows_beyond_limits(n_tokens, cols))
        return H3_ERR_UNSUPPORTED;
    const Split ts = make_split(n_tokens, world);
    const uint64_t row_bytes = uint64_t(cols) * 2;
    uint64_t in_bytes[kMaxWorld] = {};
    uint64_t out_bytes[kMaxWorld] = {};
    for (int r = 0; r < world; ++r) {
        if (!in[r] || !out[r])
            return H3_ERR_INVALID_ARG;
        if (!aligned16(in[r]) || !aligned16(out[r]))
            return H3_ERR_MISALIGNED;
        in_bytes[r] = uint64_t(ts.size(r)) * row_bytes;
        out_bytes[r] = uint64_t(n_tokens) * row_bytes;
    }
    st = check_no_overlap(in, in_bytes, world, out, out_bytes, world);
    if (st != H3_OK)
        return st;
    GatherArgs a;
    std::memset(&a, 0, sizeof(a));
    for (int r = 0; r < world; ++r) {
        a.in[r] = static_cast<const char*>(in[r]);
        a.out[r] = static_cast<char*>(out[r]);
    }
    a.T = int32_t(n_tokens);
    a.W = world;
    a.n_in = world;
    a.tq = int32_t(ts.q);
    a.tm = int32_t(ts.m);
    a.row_vecs = int32_t(cols / 8);
    a.row_bytes = int64_t(row_bytes);
    const int variant = cfg ? cfg->variant : 0;
    if (variant == H3_VARIANT_BULK) {
        int device = 0;
        const cudaError_t derr = cudaGetDevice(&device);
        if (derr != cudaSuccess)
            return cuda_failure(derr);
        if (!all_gather_bulk_fits(a, device))
            return H3_ERR_UNSUPPORTED;  // the bulk kernel's row stages do not fit in shared memory
    }
    LaunchShape shape;
    const cudaError_t err = launch_all_gather(a, variant, cfg ? cfg->ctas_per_sm : 0,
                                              static_cast<cudaStream_t>(stream), &shape,
                                              programmatic_launch(cfg));
    if (err != cudaSuccess)
        return cuda_failure(err);
    if (info) {
        info->launches = 1;
        info->chunks = 1;
        info->grid = shape.grid;
        info->block = shape.block;
        info->variant = shape.variant;
        info->planes_per_launch = 1;
    }
    return H3_OK;
}

h3_status h3_ragged_reduce_scatter_gated(const void* const* partials, const void* bias,
                                         const void* gate, const int64_t* seg_bounds,
                                         int32_t n_segs, const void* const* x, void* const* out,
                                         int64_t n_tokens, int64_t cols, int32_t world,
                                         void* stream, h3_exec_info* info)
{
    clear_info(info);
    h3_status st = check_world(n_tokens, world, world);
    if (st != H3_OK)
        return st;
    if (cols < 1 || !partials || !out || !x || !gate || !seg_bounds)
        return H3_ERR_INVALID_ARG;
    if (n_segs < 1 || n_segs > H3RR_MAX_GATE_SEGMENTS)
        return n_segs < 1 ? H3_ERR_INVALID_ARG : H3_ERR_UNSUPPORTED;
    if (seg_bounds[0] != 0 || seg_bounds[n_segs] != n_tokens)
        return H3_ERR_INVALID_ARG;
    for (int32_t k = 0; k < n_segs; ++k)
        if (seg_bounds[k + 1] <= seg_bounds[k])
            return H3_ERR_INVALID_ARG;
    if (cols % 8 != 0)
        return H3_ERR_MISALIGNED;
    if (rows_beyond_limits(n_tokens, cols))
        return H3_ERR_UNSUPPORTED;
    if (!aligned16(gate) || (bias && !aligned16(bias)))
        return H3_ERR_MISALIGNED;
    const Split ts = make_split(n_tokens, world);
    const uint64_t row_bytes = uint64_t(cols) * 2;
    for (int r = 0; r < world; ++r) {
        if (!partials[r] || !out[r] || !x[r])
            return H3_ERR_INVALID_ARG;
        if (!aligned16(partials[r]) || !aligned16(out[r]) || !aligned16(x[r]))
            return H3_ERR_MISALIGNED;
    }
    // Outputs against every input and each other; out[r] may be x[r] exactly.
    for (int r = 0; r < world; ++r) {
        const uintptr_t o = reinterpret_cast<uintptr_t>(out[r]);
        const uint64_t on = uint64_t(ts.size(r)) * row_bytes;
        const bool in_place = out[r] == x[r];
        for (int k = 0; k < world; ++k) {
            if (ranges_overlap(o, on, reinterpret_cast<uintptr_t>(partials[k]), uint64_t(n_tokens) * row_bytes))
                return H3_ERR_INVALID_ARG;
            if (!(in_place && k == r) &&
                ranges_overlap(o, on, reinterpret_cast<uintptr_t>(x[k]), uint64_t(ts.size(k)) * row_bytes))
                return H3_ERR_INVALID_ARG;
            if (k > r && ranges_overlap(o, on, reinterpret_cast<uintptr_t>(out[k]),
                                        uint64_t(ts.size(k)) * row_bytes))
                return H3_ERR_INVALID_ARG;
        }
        if (ranges_overlap(o, on, reinterpret_cast<uintptr_t>(gate), uint64_t(n_segs) * row_bytes) ||
            (bias && ranges_overlap(o, on, reinterpret_cast<uintptr_t>(bias), row_bytes)))
            return H3_ERR_INVALID_ARG;
    }
    GatedArgs g;
    std::memset(&g, 0, sizeof(g));
    for (int r = 0; r < world; ++r) {
        g.r.part[r] = static_cast<const char*>(partials[r]);
        g.r.out[r] = static_cast<char*>(out[r]);
        g.x[r] = static_cast<const char*>(x[r]);
    }
    g.r.bias = static_cast<const char*>(bias);
    g.r.T = int32_t(n_tokens);
    g.r.W = world;
    g.r.tq = int32_t(ts.q);
    g.r.tm = int32_t(ts.m);
    g.r.row_vecs = int32_t(cols / 8);
    g.r.row_bytes = int64_t(row_bytes);
    g.gate = static_cast<const char*>(gate);
    g.n_segs = n_segs;
    for (int32_t k = 0; k <= n_segs; ++k)
        g.seg_bounds[k] = int32_t(seg_bounds[k]);
    LaunchShape shape;
    const cudaError_t err =
        launch_reduce_scatter_gated(g, static_cast<cudaStream_t>(stream), &shape, true);
    if (err != cudaSuccess)
        return cuda_failure(err);
    if (info) {
        info->launches = 1;
        info->chunks = 1;
        info->grid = shape.grid;
        info->block = shape.block;
        info->variant = shape.variant;
        info->planes_per_launch = 1;
    }
    return H3_OK;
}

h3_status h3_ragged_reduce_scatter(const void* const* partials, const void* bias, void* const* out,
                                   int64_t n_tokens, int64_t cols, int32_t world, void* stream,
                                   h3_exec_info* info)
{
    return h3_ragged_reduce_scatter_ex(partials, bias, out, n_tokens, cols, world, stream, nullptr,
                                       info);
}

}  // extern "C"
