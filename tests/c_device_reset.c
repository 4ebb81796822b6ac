/* The library across cudaDeviceReset, from plain C on the GPU.  State the
 * library keeps per CUDA context -- the static window's device address
 * (h3_seq_to_head_staged_noalloc) and the bulk kernels' shared-memory opt-in
 * -- must be set up again in the device's next context, not reused from the
 * destroyed one.  Each round allocates its buffers with cudaMalloc, runs the
 * bulk seq->head and the allocation-free staged seq->head, and compares both
 * with the plain-C oracle bit for bit; between the rounds the program resets
 * the device (which ends only its own context).  Built and run by
 * tests/test_gpu_c_program.py. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "h3rr.h"

int32_t h3o_partition_range(int64_t n, int32_t w, int64_t* starts);
int32_t h3o_seq_to_head(const uint16_t* const* send, uint16_t* const* recv, int64_t T, int32_t P,
                        int32_t H, int32_t D, int32_t W);

#define W 4
enum { T = 700, P = 3, H = 56, D = 128 };

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

static uint64_t rng_state;

/* Seeded 64-bit LCG (Knuth's MMIX constants); the upper bits are used. */
static uint16_t next_bits(void)
{
    rng_state = rng_state * 6364136223846793005ULL + 1442695040888963407ULL;
    return (uint16_t)(rng_state >> 48);
}

static void round_trip(int round)
{
    int64_t ts[W + 1], hs[W + 1];
    uint16_t *send[W], *want[W], *got;
    void *d_send[W], *d_heads[W];
    cudaStream_t stream;
    h3_exec_info info;
    h3_launch_config cfg;
    char what[96];
    int r;
    if (!cuda_ok(cudaSetDevice(0), "cudaSetDevice") ||
        !cuda_ok(cudaStreamCreateWithFlags(&stream, cudaStreamNonBlocking), "stream"))
        return;
    expect(h3o_partition_range(T, W, ts) == 0 && h3o_partition_range(H, W, hs) == 0, "partition");
    got = (uint16_t*)malloc((size_t)T * P * H * D * sizeof(uint16_t));
    for (r = 0; r < W; ++r) {
        int64_t n = (ts[r + 1] - ts[r]) * P * H * D, m = T * P * (hs[r + 1] - hs[r]) * D, i;
        send[r] = (uint16_t*)malloc((size_t)n * sizeof(uint16_t));
        want[r] = (uint16_t*)malloc((size_t)m * sizeof(uint16_t));
        for (i = 0; i < n; ++i)
            send[r][i] = next_bits();
        cuda_ok(cudaMalloc(&d_send[r], (size_t)n * 2), "cudaMalloc send");
        cuda_ok(cudaMalloc(&d_heads[r], (size_t)m * 2), "cudaMalloc heads");
        cuda_ok(cudaMemcpy(d_send[r], send[r], (size_t)n * 2, cudaMemcpyHostToDevice), "copy in");
    }
    expect(h3o_seq_to_head((const uint16_t* const*)send, want, T, P, H, D, W) == 0, "oracle");

    /* the bulk kernel: its four row stages need more than the default 48 KB of shared memory */
    memset(&cfg, 0, sizeof(cfg));
    cfg.variant = H3_VARIANT_BULK;
    expect(h3_seq_to_head_ex((const void* const*)d_send, d_heads, T, P, H, D, W, 0, stream, &cfg,
                             &info) == H3_OK && info.variant == H3_VARIANT_BULK, "bulk status");
    cuda_ok(cudaStreamSynchronize(stream), "bulk sync");
    for (r = 0; r < W; ++r) {
        int64_t m = T * P * (hs[r + 1] - hs[r]) * D;
        cuda_ok(cudaMemcpy(got, d_heads[r], (size_t)m * 2, cudaMemcpyDeviceToHost), "copy out");
        snprintf(what, sizeof what, "round %d: bulk seq->head rank %d", round, r);
        expect(memcmp(got, want[r], (size_t)m * 2) == 0, what);
        cuda_ok(cudaMemset(d_heads[r], 0x5a, (size_t)m * 2), "memset");
    }

    /* the allocation-free staged call: chunks of 9 tokens in the static window */
    expect(h3_seq_to_head_staged_noalloc((const void* const*)d_send, d_heads, T, P, H, D, W,
                                         9 * H * D * 2, stream, &info) == H3_OK,
           "noalloc status");
    cuda_ok(cudaStreamSynchronize(stream), "noalloc sync");
    for (r = 0; r < W; ++r) {
        int64_t m = T * P * (hs[r + 1] - hs[r]) * D;
        cuda_ok(cudaMemcpy(got, d_heads[r], (size_t)m * 2, cudaMemcpyDeviceToHost), "copy out");
        snprintf(what, sizeof what, "round %d: no-alloc staged seq->head rank %d", round, r);
        expect(memcmp(got, want[r], (size_t)m * 2) == 0, what);
    }

    for (r = 0; r < W; ++r) {
        cudaFree(d_send[r]);
        cudaFree(d_heads[r]);
        free(send[r]);
        free(want[r]);
    }
    free(got);
    cudaStreamDestroy(stream);
}

int main(void)
{
    rng_state = 20261203u;
    round_trip(0);
    /* ends this process's context on the device; the next round runs in a new one */
    cuda_ok(cudaDeviceReset(), "cudaDeviceReset");
    round_trip(1);
    if (failures) {
        fprintf(stderr, "%d failure(s)\n", failures);
        return 1;
    }
    printf("c device reset ok\n");
    return 0;
}
