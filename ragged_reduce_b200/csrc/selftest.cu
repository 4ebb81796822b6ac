// Self-test of the bounded barrier wait the bulk kernels rely on
// (h3_bounded_wait_selftest).  One thread initialises a shared-memory
// barrier for one arrival and waits on its first phase with a given poll
// limit.  With no arrival the phase never completes, so the wait must give
// up after `polls` tries and say so; with one arrival first it must succeed.
// No copy is in flight and every wait is bounded, so nothing can hang.
#include "bulk_copy.cuh"
#include "h3rr_internal.h"

namespace h3rr {
namespace {

__device__ int32_t g_selftest_expired = -1;

__global__ void __launch_bounds__(32) bounded_wait_probe_kernel(uint32_t polls, int32_t arrive_first)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0)
        return;
    mbar_init(&bar, 1);
    mbar_fence_init();
    if (arrive_first)
        mbar_arrive(&bar);
    const bool completed = mbar_wait(&bar, 0, polls);
    g_selftest_expired = completed ? 0 : 1;
}

}  // namespace

cudaError_t run_bounded_wait_probe(uint32_t polls, int32_t arrive_first, cudaStream_t stream,
                                   int32_t* expired)
{
    const int32_t unset = -1;
    cudaError_t err = cudaMemcpyToSymbolAsync(g_selftest_expired, &unset, sizeof(unset), 0,
                                              cudaMemcpyHostToDevice, stream);
    if (err != cudaSuccess)
        return err;
    bounded_wait_probe_kernel<<<1, 32, 0, stream>>>(polls, arrive_first);
    err = cudaGetLastError();
    if (err != cudaSuccess)
        return err;
    err = cudaMemcpyFromSymbolAsync(expired, g_selftest_expired, sizeof(int32_t), 0,
                                    cudaMemcpyDeviceToHost, stream);
    if (err != cudaSuccess)
        return err;
    return cudaStreamSynchronize(stream);
}

}  // namespace h3rr

extern "C" h3_status h3_bounded_wait_selftest(uint32_t polls, int32_t arrive_first, void* stream,
                                             int32_t* expired)
{
    if (!expired || polls < 1 || polls > h3rr::kBulkWaitLimit || (arrive_first != 0 && arrive_first != 1))
        return H3_ERR_INVALID_ARG;
    *expired = -1;
    const cudaError_t err =
        h3rr::run_bounded_wait_probe(polls, arrive_first, static_cast<cudaStream_t>(stream), expired);
    if (err != cudaSuccess)
        return h3rr::record_cuda_failure(err);
    return H3_OK;
}
