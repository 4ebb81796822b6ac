/*
 * Plain, slow CPU oracle for the H3 Ulysses relayouts and the tensor-mode
 * ragged reduce-scatter.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the benchmark's
 * CPU-baseline / reference arm do.  It shares no code, header, table or
 * helper with the CUDA library; it is written from the definitions on the
 * pages, one scalar element at a time, with no blocking or fusion.
 *
 * Sources (page title, section):
 *   [DIST]  h3-blackwell-runtime "Distributed H3 Execution" (DISTRIBUTED.md):
 *           intro (two modes, no empty partitions, packed sequence kept),
 *           section "Partition Contract" (head table, token ranges,
 *           segment clip + rebase, ragged reduce-scatter, bias once).
 *   [PR]    FastVideo PR #1807 "[perf] Harden Ulysses agreement and tune
 *           bounded H3 transfers", section "Problem and behavior" (one batch
 *           plane at a time, 896,000,000-byte window).
 *
 * Element type: BF16 values are carried as their raw 16-bit patterns
 * (uint16_t).  The relayouts copy those patterns; the reduction widens them to
 * IEEE binary32 exactly, adds in binary32 in rank order 0..W-1, adds the bias
 * once after the sum, and rounds back to BF16 to nearest, ties to even.
 *
 * Build: plain C99, gcc -O1 -ffp-contract=off (adds only; no contraction,
 * no fast-math, no flush-to-zero).
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* BF16 <-> binary32                                                          */
/* ------------------------------------------------------------------------ */

/* BF16 is the upper half of a binary32 word, so widening is exact: put the
 * 16 bits on top and zero the rest. */
float h3o_bf16_to_f32(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Narrow binary32 to BF16, round to nearest, ties to even.
 *
 * Keep the upper 16 bits (truncation toward zero in magnitude) and look at the
 * 16 discarded bits: above one half of a BF16 unit -> bump the kept magnitude
 * by one unit; exactly one half -> bump only if the kept pattern is odd; below
 * one half -> keep.  Bumping the integer pattern carries into the exponent
 * correctly (including the largest finite value rounding up to infinity),
 * because for one sign the bit patterns are ordered like the magnitudes.
 * NaN stays NaN: the sign and the top payload bits are kept and the quiet bit
 * is forced, so a NaN never collapses to infinity. */
uint16_t h3o_f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint32_t exponent = (u >> 23) & 0xFFu;
    uint32_t mantissa = u & 0x7FFFFFu;
    if (exponent == 0xFFu && mantissa != 0u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint16_t kept = (uint16_t)(u >> 16);
    uint32_t dropped = u & 0xFFFFu;
    if (dropped > 0x8000u)
        kept = (uint16_t)(kept + 1u);
    else if (dropped == 0x8000u && (kept & 1u))
        kept = (uint16_t)(kept + 1u);
    return kept;
}

void h3o_bf16_to_f32_array(const uint16_t* in, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = h3o_bf16_to_f32(in[i]);
}

void h3o_f32_to_bf16_array(const float* in, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = h3o_f32_to_bf16_rne(in[i]);
}

/* ------------------------------------------------------------------------ */
/* Partition contract [DIST, "Partition Contract"]                            */
/* ------------------------------------------------------------------------ */

/* Balanced quotient/remainder split of n items over w ranks: every rank gets
 * n/w items and the first n%w ranks one more (the printed head table: W=6
 * gives 10,10,9,9,9,9).  starts has w+1 entries: rank i owns
 * [starts[i], starts[i+1]).  Empty parts are rejected [DIST, intro]:
 * returns -1 when w < 1 or n < w, else 0. */
int32_t h3o_partition_range(int64_t n, int32_t w, int64_t* starts)
{
    if (w < 1 || n < (int64_t)w)
        return -1;
    int64_t q = n / w;
    int64_t rem = n % w;
    starts[0] = 0;
    for (int32_t i = 0; i < w; ++i)
        starts[i + 1] = starts[i] + q + (i < rem ? 1 : 0);
    return 0;
}

/* Rank that owns item x under the split in starts (linear scan). */
static int32_t owner_of(const int64_t* starts, int32_t w, int64_t x)
{
    for (int32_t i = 0; i < w; ++i)
        if (x < starts[i + 1])
            return i;
    return -1;
}

int32_t h3o_owner(const int64_t* starts, int32_t w, int64_t x)
{
    return owner_of(starts, w, x);
}

/* Clip packed segments to one rank's token interval [ts, te) and rebase them
 * [DIST, "Partition Contract": segment boundaries are clipped to each rank's
 * token interval and rebased].  bounds has n_segs+1 entries, 0 = b_0 < b_1 <
 * ... < b_n = T.  Every segment k whose intersection with [ts, te) is not
 * empty gives one piece; pieces keep the order of the segments.  Writes the
 * rebased piece starts to local_bounds[0..n) and te-ts to local_bounds[n],
 * and the global segment index of each piece to seg_ids[0..n).  Returns n. */
int32_t h3o_clip_segments(const int64_t* bounds, int32_t n_segs,
                          int64_t ts, int64_t te,
                          int64_t* local_bounds, int32_t* seg_ids)
{
    int32_t n = 0;
    for (int32_t k = 0; k < n_segs; ++k) {
        int64_t a = bounds[k] > ts ? bounds[k] : ts;
        int64_t b = bounds[k + 1] < te ? bounds[k + 1] : te;
        if (a < b) {
            local_bounds[n] = a - ts;
            seg_ids[n] = k;
            ++n;
        }
    }
    local_bounds[n] = te - ts;
    return n;
}

/* ------------------------------------------------------------------------ */
/* Ulysses relayouts [DIST, intro: sequence-to-head all-to-all on QKV and    */
/* the inverse head-to-sequence all-to-all around attention]                  */
/*                                                                            */
/* Sequence side, rank r: [T_r, P, H, D], tokens ts_r .. te_r-1 of the packed */
/* sequence, all H heads.  Head side, rank j: [T, P, H_j, D], every token,    */
/* heads hs_j .. he_j-1.  Both row-major, element = one BF16 pattern.         */
/* ------------------------------------------------------------------------ */

/* seq -> head: walk every element of every sequence-side buffer and put it
 * where its head's owner keeps it.  Returns -1 on an empty partition. */
int32_t h3o_seq_to_head(const uint16_t* const* send, uint16_t* const* recv,
                        int64_t T, int32_t P, int32_t H, int32_t D, int32_t W)
{
    int64_t* ts = (int64_t*)malloc(sizeof(int64_t) * (size_t)(W + 1));
    int64_t* hs = (int64_t*)malloc(sizeof(int64_t) * (size_t)(W + 1));
    int32_t rc = -1;
    if (!ts || !hs)
        goto done;
    if (h3o_partition_range(T, W, ts) || h3o_partition_range(H, W, hs))
        goto done;
    for (int32_t r = 0; r < W; ++r) {
        int64_t Tr = ts[r + 1] - ts[r];
        for (int64_t tl = 0; tl < Tr; ++tl) {
            int64_t t = ts[r] + tl;
            for (int32_t p = 0; p < P; ++p) {
                for (int32_t h = 0; h < H; ++h) {
                    int32_t j = owner_of(hs, W, h);
                    int64_t Hj = hs[j + 1] - hs[j];
                    int64_t hl = h - hs[j];
                    for (int32_t d = 0; d < D; ++d) {
                        int64_t src = ((tl * P + p) * H + h) * D + d;
                        int64_t dst = ((t * P + p) * Hj + hl) * D + d;
                        recv[j][dst] = send[r][src];
                    }
                }
            }
        }
    }
    rc = 0;
done:
    free(ts);
    free(hs);
    return rc;
}

/* head -> seq: fill every element of every sequence-side buffer from the
 * head-side buffer of the rank that owns its head.  Returns -1 on an empty
 * partition. */
int32_t h3o_head_to_seq(const uint16_t* const* send, uint16_t* const* recv,
                        int64_t T, int32_t P, int32_t H, int32_t D, int32_t W)
{
    int64_t* ts = (int64_t*)malloc(sizeof(int64_t) * (size_t)(W + 1));
    int64_t* hs = (int64_t*)malloc(sizeof(int64_t) * (size_t)(W + 1));
    int32_t rc = -1;
    if (!ts || !hs)
        goto done;
    if (h3o_partition_range(T, W, ts) || h3o_partition_range(H, W, hs))
        goto done;
    for (int32_t r = 0; r < W; ++r) {
        int64_t Tr = ts[r + 1] - ts[r];
        for (int64_t tl = 0; tl < Tr; ++tl) {
            int64_t t = ts[r] + tl;
            for (int32_t p = 0; p < P; ++p) {
                for (int32_t h = 0; h < H; ++h) {
                    int32_t j = owner_of(hs, W, h);
                    int64_t Hj = hs[j + 1] - hs[j];
                    int64_t hl = h - hs[j];
                    for (int32_t d = 0; d < D; ++d) {
                        int64_t dst = ((tl * P + p) * H + h) * D + d;
                        int64_t src = ((t * P + p) * Hj + hl) * D + d;
                        recv[r][dst] = send[j][src];
                    }
                }
            }
        }
    }
    rc = 0;
done:
    free(ts);
    free(hs);
    return rc;
}

/* Gather form of seq -> head, one output element at a time, for sampled
 * checks at sizes the full loops cannot hold: element out_elem[i] of head-side
 * rank j's buffer [T, P, H_j, D] is element src_elem[i] of sequence-side rank
 * src_rank[i]'s buffer [T_r, P, H, D].  Returns -1 on a bad partition or an
 * index out of range. */
int32_t h3o_seq_to_head_locate(int64_t T, int32_t P, int32_t H, int32_t D,
                               int32_t W, int32_t j, int64_t n,
                               const int64_t* out_elem,
                               int32_t* src_rank, int64_t* src_elem)
{
    int64_t* ts = (int64_t*)malloc(sizeof(int64_t) * (size_t)(W + 1));
    int64_t* hs = (int64_t*)malloc(sizeof(int64_t) * (size_t)(W + 1));
    int32_t rc = -1;
    if (!ts || !hs)
        goto done;
    if (h3o_partition_range(T, W, ts) || h3o_partition_range(H, W, hs))
        goto done;
    if (j < 0 || j >= W)
        goto done;
    {
        int64_t Hj = hs[j + 1] - hs[j];
        for (int64_t i = 0; i < n; ++i) {
            int64_t e = out_elem[i];
            if (e < 0 || e >= T * P * Hj * D)
                goto done;
            int64_t d = e % D;
            e /= D;
            int64_t hl = e % Hj;
            e /= Hj;
            int64_t p = e % P;
            int64_t t = e / P;
            int32_t r = owner_of(ts, W, t);
            src_rank[i] = r;
            src_elem[i] = (((t - ts[r]) * P + p) * H + (hs[j] + hl)) * D + d;
        }
    }
    rc = 0;
done:
    free(ts);
    free(hs);
    return rc;
}

/* Gather form of head -> seq: element out_elem[i] of sequence-side rank r's
 * buffer [T_r, P, H, D] is element src_elem[i] of head-side rank src_rank[i]'s
 * buffer [T, P, H_j, D]. */
int32_t h3o_head_to_seq_locate(int64_t T, int32_t P, int32_t H, int32_t D,
                               int32_t W, int32_t r, int64_t n,
                               const int64_t* out_elem,
                               int32_t* src_rank, int64_t* src_elem)
{
    int64_t* ts = (int64_t*)malloc(sizeof(int64_t) * (size_t)(W + 1));
    int64_t* hs = (int64_t*)malloc(sizeof(int64_t) * (size_t)(W + 1));
    int32_t rc = -1;
    if (!ts || !hs)
        goto done;
    if (h3o_partition_range(T, W, ts) || h3o_partition_range(H, W, hs))
        goto done;
    if (r < 0 || r >= W)
        goto done;
    {
        int64_t Tr = ts[r + 1] - ts[r];
        for (int64_t i = 0; i < n; ++i) {
            int64_t e = out_elem[i];
            if (e < 0 || e >= Tr * P * H * D)
                goto done;
            int64_t d = e % D;
            e /= D;
            int64_t h = e % H;
            e /= H;
            int64_t p = e % P;
            int64_t tl = e / P;
            int32_t j = owner_of(hs, W, h);
            int64_t Hj = hs[j + 1] - hs[j];
            src_rank[i] = j;
            src_elem[i] = (((ts[r] + tl) * P + p) * Hj + (h - hs[j])) * D + d;
        }
    }
    rc = 0;
done:
    free(ts);
    free(hs);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Tensor-mode ragged reduce-scatter [DIST, "Partition Contract": each rank  */
/* computes a partial output, a ragged reduce-scatter sums them and assigns  */
/* token rows; the projection bias is left out of the partials and added     */
/* exactly once after the reduction]                                          */
/* ------------------------------------------------------------------------ */

/* One output element from W partial values and an optional bias value:
 * binary32 sum in rank order 0..W-1, starting from partial 0 itself (not
 * from +0, which would turn an all -0 sum into +0), then the bias once. */
static uint16_t reduce_one(const uint16_t* vals, int32_t W, const uint16_t* bias_val)
{
    float acc = h3o_bf16_to_f32(vals[0]);
    for (int32_t w = 1; w < W; ++w)
        acc = acc + h3o_bf16_to_f32(vals[w]);
    if (bias_val)
        acc = acc + h3o_bf16_to_f32(*bias_val);
    return h3o_f32_to_bf16_rne(acc);
}

/* Reduce rows without the scatter: partials[w] are [rows, C], bias is [C] or
 * NULL, out is [rows, C].  Used for sampled rows at full sizes. */
void h3o_reduce_rows(const uint16_t* const* partials, const uint16_t* bias,
                     uint16_t* out, int64_t rows, int64_t C, int32_t W)
{
    uint16_t* vals = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)W);
    if (!vals)
        return;
    for (int64_t t = 0; t < rows; ++t) {
        for (int64_t c = 0; c < C; ++c) {
            for (int32_t w = 0; w < W; ++w)
                vals[w] = partials[w][t * C + c];
            out[t * C + c] = reduce_one(vals, W, bias ? &bias[c] : NULL);
        }
    }
    free(vals);
}

/* Full ragged reduce-scatter: partials[w] are [T, C]; rank r receives rows
 * ts_r .. te_r-1 of the reduced result in out[r], [T_r, C].  Returns -1 on an
 * empty partition. */
int32_t h3o_ragged_reduce_scatter(const uint16_t* const* partials,
                                  const uint16_t* bias, uint16_t* const* out,
                                  int64_t T, int64_t C, int32_t W)
{
    int64_t* ts = (int64_t*)malloc(sizeof(int64_t) * (size_t)(W + 1));
    uint16_t* vals = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)W);
    int32_t rc = -1;
    if (!ts || !vals)
        goto done;
    if (h3o_partition_range(T, W, ts))
        goto done;
    for (int32_t r = 0; r < W; ++r) {
        for (int64_t tl = 0; tl < ts[r + 1] - ts[r]; ++tl) {
            int64_t t = ts[r] + tl;
            for (int64_t c = 0; c < C; ++c) {
                for (int32_t w = 0; w < W; ++w)
                    vals[w] = partials[w][t * C + c];
                out[r][tl * C + c] = reduce_one(vals, W, bias ? &bias[c] : NULL);
            }
        }
    }
    rc = 0;
done:
    free(ts);
    free(vals);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Ragged all-gather of token rows ["Distributed H3 Execution", intro: ragged */
/* row gathering; "Validation": ragged gather and reduce-scatter behaviour]   */
/* ------------------------------------------------------------------------ */

/* Every rank receives all T rows: out[j] is [T, C], and its row t is row
 * t - ts_r of in[r], r the rank that owns token t.  in[r] is [T_r, C].
 * Element = one 16-bit pattern, copied as is.  Returns -1 on an empty
 * partition. */
int32_t h3o_ragged_all_gather(const uint16_t* const* in, uint16_t* const* out,
                              int64_t T, int64_t C, int32_t W)
{
    int64_t* ts = (int64_t*)malloc(sizeof(int64_t) * (size_t)(W + 1));
    int32_t rc = -1;
    if (!ts)
        goto done;
    if (h3o_partition_range(T, W, ts))
        goto done;
    for (int32_t j = 0; j < W; ++j) {
        for (int64_t t = 0; t < T; ++t) {
            int32_t r = owner_of(ts, W, t);
            for (int64_t c = 0; c < C; ++c)
                out[j][t * C + c] = in[r][(t - ts[r]) * C + c];
        }
    }
    rc = 0;
done:
    free(ts);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Relayouts with plane-major buffers                                          */
/* Sequence side, rank r: [T_r, P, H, D] (token-major) or [P, T_r, H, D]      */
/* (plane-major: plane p of rank r is one contiguous [T_r, H, D] block).      */
/* Head side, rank j: [T, P, H_j, D] or [P, T, H_j, D].  Same element maps as  */
/* h3o_seq_to_head / h3o_head_to_seq; only the buffer index of (t, p, h, d)    */
/* changes.                                                                    */
/* ------------------------------------------------------------------------ */

static int64_t seq_index(int64_t tl, int64_t Tr, int64_t p, int64_t P, int64_t h, int64_t H,
                         int64_t d, int64_t D, int32_t plane_major)
{
    if (plane_major)
        return ((p * Tr + tl) * H + h) * D + d;
    return ((tl * P + p) * H + h) * D + d;
}

static int64_t head_index(int64_t t, int64_t T, int64_t p, int64_t P, int64_t hl, int64_t Hj,
                          int64_t d, int64_t D, int32_t plane_major)
{
    if (plane_major)
        return ((p * T + t) * Hj + hl) * D + d;
    return ((t * P + p) * Hj + hl) * D + d;
}

/* seq -> head (dir = 1) or head -> seq (dir = 0) with the given layouts. */
int32_t h3o_relayout_layout(const uint16_t* const* send, uint16_t* const* recv, int64_t T,
                            int32_t P, int32_t H, int32_t D, int32_t W, int32_t dir,
                            int32_t seq_plane_major, int32_t head_plane_major)
{
    int64_t* ts = (int64_t*)malloc(sizeof(int64_t) * (size_t)(W + 1));
    int64_t* hs = (int64_t*)malloc(sizeof(int64_t) * (size_t)(W + 1));
    int32_t rc = -1;
    if (!ts || !hs)
        goto done;
    if (h3o_partition_range(T, W, ts) || h3o_partition_range(H, W, hs))
        goto done;
    for (int32_t r = 0; r < W; ++r) {
        int64_t Tr = ts[r + 1] - ts[r];
        for (int64_t tl = 0; tl < Tr; ++tl) {
            int64_t t = ts[r] + tl;
            for (int32_t p = 0; p < P; ++p) {
                for (int32_t h = 0; h < H; ++h) {
                    int32_t j = owner_of(hs, W, h);
                    int64_t Hj = hs[j + 1] - hs[j];
                    for (int32_t d = 0; d < D; ++d) {
                        int64_t si = seq_index(tl, Tr, p, P, h, H, d, D, seq_plane_major);
                        int64_t hi = head_index(t, T, p, P, h - hs[j], Hj, d, D, head_plane_major);
                        if (dir)
                            recv[j][hi] = send[r][si];
                        else
                            recv[r][si] = send[j][hi];
                    }
                }
            }
        }
    }
    rc = 0;
done:
    free(ts);
    free(hs);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Ragged reduce-scatter followed by residual gating per packed segment       */
/* ["Distributed H3 Execution", "Partition Contract": segment boundaries are  */
/* clipped to each rank's token interval and rebased before AdaLN modulation  */
/* and residual gating; rank partials are summed by the ragged reduce-scatter */
/* and the bias is added once after the reduction].                           */
/*                                                                            */
/* For rank r and its local row t' (global token t = ts_r + t'):              */
/*   y        = the reduce-scatter output element (BF16, as defined above)    */
/*   k        = the global segment of the rank's clipped piece holding t'     */
/*   out[t',c] = bf16_rne( f(x[t',c]) + f(gate[k,c]) * f(y) )                  */
/* in binary32: the product of two BF16 values is exact in binary32, then one */
/* binary32 add, then round to BF16.  x and out are [T_r, C]; gate is [S, C]. */
/* ------------------------------------------------------------------------ */
int32_t h3o_reduce_scatter_gated(const uint16_t* const* partials, const uint16_t* bias,
                                 const uint16_t* gate, const int64_t* bounds, int32_t n_segs,
                                 const uint16_t* const* x, uint16_t* const* out,
                                 int64_t T, int64_t C, int32_t W)
{
    int64_t* ts = (int64_t*)malloc(sizeof(int64_t) * (size_t)(W + 1));
    uint16_t* vals = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)W);
    int64_t* local_bounds = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_segs + 1));
    int32_t* seg_ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n_segs + 1));
    int32_t rc = -1;
    if (!ts || !vals || !local_bounds || !seg_ids)
        goto done;
    if (h3o_partition_range(T, W, ts))
        goto done;
    for (int32_t r = 0; r < W; ++r) {
        int32_t pieces = h3o_clip_segments(bounds, n_segs, ts[r], ts[r + 1], local_bounds, seg_ids);
        int32_t piece = 0;
        for (int64_t tl = 0; tl < ts[r + 1] - ts[r]; ++tl) {
            while (piece + 1 < pieces && tl >= local_bounds[piece + 1])
                ++piece;
            int64_t k = seg_ids[piece];
            int64_t t = ts[r] + tl;
            for (int64_t c = 0; c < C; ++c) {
                for (int32_t w = 0; w < W; ++w)
                    vals[w] = partials[w][t * C + c];
                uint16_t y = reduce_one(vals, W, bias ? &bias[c] : NULL);
                float g = h3o_bf16_to_f32(gate[k * C + c]);
                float prod = g * h3o_bf16_to_f32(y);
                float sum = h3o_bf16_to_f32(x[r][tl * C + c]) + prod;
                out[r][tl * C + c] = h3o_f32_to_bf16_rne(sum);
            }
        }
    }
    rc = 0;
done:
    free(ts);
    free(vals);
    free(local_bounds);
    free(seg_ids);
    return rc;
}

