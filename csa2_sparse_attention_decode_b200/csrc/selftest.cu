// Self-test of the bounded-wait path every kernel uses: one CTA waits on an
// mbarrier that nothing completes, gives up after a fixed number of polls
// and records CSA2_DEV_TIMEOUT in the error word, as a kernel whose producer
// stalled would.  Nothing faults or hangs; the context stays usable.
#include "common.cuh"
#include "umma.cuh"

namespace csa2 {
namespace {

__global__ void wait_timeout_probe_kernel(int32_t *err, uint32_t polls)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        umma::mbar_init(&bar, 1);
        umma::mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !umma::mbar_wait(&bar, 0, polls)) set_error(err, CSA2_DEV_TIMEOUT);
}

}  // namespace
}  // namespace csa2

extern "C" csa2_status csa2_selftest_wait_timeout(int32_t *error_word, uint32_t polls, csa2_stream_t stream)
{
    if (!error_word || polls == 0 || polls > (1u << 16)) return CSA2_ERR_INVALID_ARG;
    csa2::wait_timeout_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(error_word, polls);
    return cudaGetLastError() == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}
