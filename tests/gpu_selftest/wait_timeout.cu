// Test-only kernel: a bounded wait on an mbarrier that nothing completes.
//
// Uses the library's own wait helper (pkv_common.cuh), so the test checks the
// exact code the decode kernel runs when a bulk copy never lands: the wait
// must give up after its time limit, report PKV_DEVERR_TIMEOUT through the
// error word and let the kernel finish, leaving the context usable.
#include "pkv_common.cuh"

namespace {

__global__ void wait_on_a_barrier_nobody_completes(int *dev_err, int *finished) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        pkv::mbar_init(&bar, 1);  // one arrival expected; none will come
        pkv::fence_barrier_init();
    }
    __syncthreads();
    if (!pkv::mbar_wait(&bar, 0)) pkv::set_error(dev_err, PKV_DEVERR_TIMEOUT);
    __syncthreads();
    if (threadIdx.x == 0) *finished = 1;
}

}  // namespace

extern "C" int pkv_selftest_wait_timeout(int *dev_err, int *finished, void *stream) {
    wait_on_a_barrier_nobody_completes<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(dev_err, finished);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}
