/* Plain-C use of the library's C ABI (include/h3rr.h) on a GPU: no Python,
 * no torch.  Buffers come from cudaMalloc, work goes on a stream the program
 * creates, and every result is compared bit for bit with the plain-C oracle
 * (oracle/h3_oracle.c, linked as test infrastructure).  Built and run by
 * tests/test_gpu_c_program.py.
 *
 * Cases: both Ulysses relayouts ("Distributed H3 Execution", intro), whole,
 * one batch plane per launch and in token chunks of a plane (FastVideo PR
 * #1807, "Problem and behavior"), and in token ranges of every plane
 * (H3_LAUNCH_CHUNK_TOKENS); the ragged reduce-scatter and the ragged
 * all-gather
 * ("Distributed H3 Execution", "Partition Contract"). */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "h3rr.h"

/* The oracle's entry points. */
int32_t h3o_partition_range(int64_t n, int32_t w, int64_t* starts);
int32_t h3o_seq_to_head(const uint16_t* const* send, uint16_t* const* recv, int64_t T, int32_t P,
                        int32_t H, int32_t D, int32_t W);
int32_t h3o_head_to_seq(const uint16_t* const* send, uint16_t* const* recv, int64_t T, int32_t P,
                        int32_t H, int32_t D, int32_t W);
int32_t h3o_ragged_reduce_scatter(const uint16_t* const* partials, const uint16_t* bias,
                                  uint16_t* const* out, int64_t T, int64_t C, int32_t W);
int32_t h3o_ragged_all_gather(const uint16_t* const* in, uint16_t* const* out, int64_t T,
                              int64_t C, int32_t W);

#define MAXW 8

static int failures = 0;

static void expect(int cond, const char* what)
{
    if (!cond) {
        fprintf(stderr, "FAIL: %s\n", what);
        ++failures;
    }
}

static int cuda_ok(cudaError_t err, const char* what)
{
    if (err != cudaSuccess) {
        fprintf(stderr, "FAIL: %s: %s\n", what, cudaGetErrorString(err));
        ++failures;
        return 0;
    }
    return 1;
}

/* Seeded 64-bit LCG (Knuth's MMIX constants); the upper bits are used. */
static uint64_t rng_state;

static uint32_t next_u32(void)
{
    rng_state = rng_state * 6364136223846793005ULL + 1442695040888963407ULL;
    return (uint32_t)(rng_state >> 32);
}

/* Any 16-bit pattern (the relayouts copy bits). */
static void fill_bits(uint16_t* x, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        x[i] = (uint16_t)(next_u32() >> 16);
}

/* Finite BF16 values: random sign and mantissa, exponent field 100..140
 * (magnitudes 2^-27 .. 2^14), so sums cancel and round but never overflow. */
static void fill_finite_bf16(uint16_t* x, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) {
        uint32_t r = next_u32();
        uint32_t sign = r & 1u, mant = (r >> 1) & 0x7fu, expo = 100u + (r >> 8) % 41u;
        x[i] = (uint16_t)((sign << 15) | (expo << 7) | mant);
    }
}

static uint16_t* host_alloc(int64_t elems)
{
    uint16_t* p = (uint16_t*)malloc((size_t)(elems > 0 ? elems : 1) * sizeof(uint16_t));
    if (!p) {
        fprintf(stderr, "FAIL: host allocation\n");
        exit(2);
    }
    return p;
}

static void* dev_alloc(int64_t elems)
{
    void* p = NULL;
    if (!cuda_ok(cudaMalloc(&p, (size_t)(elems > 0 ? elems : 1) * sizeof(uint16_t)), "cudaMalloc"))
        exit(2);
    return p;
}

static void to_dev(void* d, const uint16_t* h, int64_t elems)
{
    cuda_ok(cudaMemcpy(d, h, (size_t)elems * sizeof(uint16_t), cudaMemcpyHostToDevice), "H2D");
}

static int same_as_dev(const void* d, const uint16_t* want, int64_t elems)
{
    uint16_t* got = host_alloc(elems);
    int same = 0;
    if (cuda_ok(cudaMemcpy(got, d, (size_t)elems * sizeof(uint16_t), cudaMemcpyDeviceToHost), "D2H"))
        same = memcmp(got, want, (size_t)elems * sizeof(uint16_t)) == 0;
    free(got);
    return same;
}

/* seq->head then head->seq of a [T, P, H, D] operand over W ranks. */
static void relayout_case(int64_t T, int32_t P, int32_t H, int32_t D, int32_t W, int64_t window,
                          int32_t flags, cudaStream_t stream)
{
    int64_t ts[MAXW + 1], hs[MAXW + 1];
    uint16_t *send[MAXW], *want[MAXW], *back_want[MAXW];
    void *d_send[MAXW], *d_heads[MAXW], *d_back[MAXW];
    h3_exec_info info;
    char what[160];
    int32_t r;
    expect(h3o_partition_range(T, W, ts) == 0 && h3o_partition_range(H, W, hs) == 0,
           "oracle partition");
    for (r = 0; r < W; ++r) {
        int64_t n = (ts[r + 1] - ts[r]) * P * H * D;
        send[r] = host_alloc(n);
        back_want[r] = host_alloc(n);
        fill_bits(send[r], n);
        d_send[r] = dev_alloc(n);
        d_back[r] = dev_alloc(n);
        to_dev(d_send[r], send[r], n);
    }
    for (r = 0; r < W; ++r) {
        int64_t n = T * P * (hs[r + 1] - hs[r]) * D;
        want[r] = host_alloc(n);
        d_heads[r] = dev_alloc(n);
    }
    expect(h3o_seq_to_head((const uint16_t* const*)send, want, T, P, H, D, W) == 0, "oracle s2h");
    expect(h3o_head_to_seq((const uint16_t* const*)want, back_want, T, P, H, D, W) == 0,
           "oracle h2s");

    {
        int64_t tokens = 0, chunks = 0;
        int32_t per_launch = 0;
        h3_launch_config cfg;
        memset(&cfg, 0, sizeof(cfg));
        cfg.flags = flags;
        expect(h3_relayout_chunk_plan_ex(T, P, H, D, W, window, flags, &tokens, &chunks,
                                         &per_launch) == H3_OK,
               "chunk plan");
        expect(h3_seq_to_head_ex((const void* const*)d_send, d_heads, T, P, H, D, W, window, stream,
                                 &cfg, &info) == H3_OK, "h3_seq_to_head status");
        expect(info.launches == chunks && info.chunks == chunks && info.planes_per_launch == per_launch,
               "seq->head launches");
        expect(h3_head_to_seq_ex((const void* const*)d_heads, d_back, T, P, H, D, W, window, stream,
                                 &cfg, &info) == H3_OK, "h3_head_to_seq status");
        expect(info.launches == chunks && info.planes_per_launch == per_launch, "head->seq launches");
    }
    cuda_ok(cudaStreamSynchronize(stream), "relayout sync");
    for (r = 0; r < W; ++r) {
        snprintf(what, sizeof what, "seq->head T=%lld P=%d W=%d window=%lld rank %d", (long long)T,
                 (int)P, (int)W, (long long)window, (int)r);
        expect(same_as_dev(d_heads[r], want[r], T * P * (hs[r + 1] - hs[r]) * D), what);
        snprintf(what, sizeof what, "head->seq T=%lld P=%d W=%d window=%lld rank %d", (long long)T,
                 (int)P, (int)W, (long long)window, (int)r);
        expect(same_as_dev(d_back[r], back_want[r], (ts[r + 1] - ts[r]) * P * H * D), what);
        expect(memcmp(back_want[r], send[r],
                      (size_t)((ts[r + 1] - ts[r]) * P * H * D) * sizeof(uint16_t)) == 0,
               "oracle round trip is the identity");
    }
    for (r = 0; r < W; ++r) {
        free(send[r]);
        free(want[r]);
        free(back_want[r]);
        cudaFree(d_send[r]);
        cudaFree(d_heads[r]);
        cudaFree(d_back[r]);
    }
}

/* Reduce-scatter of W partials [T, C] + bias, then all-gather of its rows. */
static void reduce_gather_case(int64_t T, int64_t C, int32_t W, cudaStream_t stream)
{
    int64_t ts[MAXW + 1];
    uint16_t *partials[MAXW], *bias, *red[MAXW], *full;
    uint16_t* gathered_want[MAXW];
    void *d_part[MAXW], *d_bias, *d_red[MAXW], *d_gath[MAXW];
    h3_exec_info info;
    char what[160];
    int32_t r;
    expect(h3o_partition_range(T, W, ts) == 0, "oracle partition");
    for (r = 0; r < W; ++r) {
        partials[r] = host_alloc(T * C);
        fill_finite_bf16(partials[r], T * C);
        d_part[r] = dev_alloc(T * C);
        to_dev(d_part[r], partials[r], T * C);
        red[r] = host_alloc((ts[r + 1] - ts[r]) * C);
        d_red[r] = dev_alloc((ts[r + 1] - ts[r]) * C);
        gathered_want[r] = host_alloc(T * C);
        d_gath[r] = dev_alloc(T * C);
    }
    bias = host_alloc(C);
    fill_finite_bf16(bias, C);
    d_bias = dev_alloc(C);
    to_dev(d_bias, bias, C);
    full = host_alloc(T * C);

    expect(h3o_ragged_reduce_scatter((const uint16_t* const*)partials, bias, red, T, C, W) == 0,
           "oracle reduce-scatter");
    expect(h3o_ragged_all_gather((const uint16_t* const*)red, gathered_want, T, C, W) == 0,
           "oracle all-gather");
    for (r = 0; r < W; ++r)
        memcpy(full + ts[r] * C, red[r], (size_t)((ts[r + 1] - ts[r]) * C) * sizeof(uint16_t));

    expect(h3_ragged_reduce_scatter((const void* const*)d_part, d_bias, d_red, T, C, W, stream,
                                    &info) == H3_OK, "h3_ragged_reduce_scatter status");
    expect(h3_ragged_all_gather((const void* const*)d_red, d_gath, T, C, W, stream, &info) == H3_OK,
           "h3_ragged_all_gather status");
    cuda_ok(cudaStreamSynchronize(stream), "reduce sync");
    for (r = 0; r < W; ++r) {
        snprintf(what, sizeof what, "reduce-scatter T=%lld C=%lld W=%d rank %d", (long long)T,
                 (long long)C, (int)W, (int)r);
        expect(same_as_dev(d_red[r], red[r], (ts[r + 1] - ts[r]) * C), what);
        snprintf(what, sizeof what, "all-gather T=%lld C=%lld W=%d rank %d", (long long)T,
                 (long long)C, (int)W, (int)r);
        expect(same_as_dev(d_gath[r], gathered_want[r], T * C), what);
        expect(memcmp(gathered_want[r], full, (size_t)(T * C) * sizeof(uint16_t)) == 0,
               "oracle all-gather is the concatenation");
    }
    for (r = 0; r < W; ++r) {
        free(partials[r]);
        free(red[r]);
        free(gathered_want[r]);
        cudaFree(d_part[r]);
        cudaFree(d_red[r]);
        cudaFree(d_gath[r]);
    }
    free(bias);
    free(full);
    cudaFree(d_bias);
}

int main(void)
{
    cudaStream_t stream;
    rng_state = 20240607u;
    if (!cuda_ok(cudaSetDevice(0), "cudaSetDevice") ||
        !cuda_ok(cudaStreamCreateWithFlags(&stream, cudaStreamNonBlocking), "stream"))
        return 2;
    expect(h3_abi_version() == H3RR_ABI_VERSION, "abi version");

    relayout_case(1000, 3, 56, 128, 6, 0, 0, stream);
    /* one plane per launch: the window holds the largest plane slice (rank
     * 0's 167 tokens x 56 heads and 1000 tokens x 10 heads, both x 256 B) */
    relayout_case(1000, 3, 56, 128, 6, 1000 * 10 * 256, 0, stream);
    /* a window of a third of a plane: every plane in token chunks (at most 55
     * tokens of every rank fit, so 4 chunks of 42 per plane) */
    relayout_case(1000, 3, 56, 128, 6, 1000 * 10 * 256 / 3, 0, stream);
    /* the same window cut into token ranges of all three planes: at most 18
     * tokens of every rank fit, so 10 launches of 17 */
    relayout_case(1000, 3, 56, 128, 6, 1000 * 10 * 256 / 3, H3_LAUNCH_CHUNK_TOKENS, stream);
    relayout_case(777, 4, 56, 128, 8, 0, 0, stream);
    relayout_case(97, 2, 9, 8, 3, 0, 0, stream);
    reduce_gather_case(777, 7168, 8, stream);
    reduce_gather_case(1000, 2048, 6, stream);
    reduce_gather_case(33, 24, 1, stream);

    cudaStreamDestroy(stream);
    if (failures) {
        fprintf(stderr, "%d failure(s)\n", failures);
        return 1;
    }
    printf("c gpu parity ok\n");
    return 0;
}
