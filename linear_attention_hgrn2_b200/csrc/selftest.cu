// selftest.cu -- check of the library's failure reporting on the GPU.
//
// Every wait inside the library's kernels is bounded (mbar_wait); when a wait gives up, the
// kernel records HGRN2_ERR_TIMEOUT in the device status word, leaves its loop and exits, and
// the host reads the word with hgrn2_get_device_status.  This kernel exercises that path
// without any fault: one block waits, through the same helper, on an mbarrier that nothing
// ever arrives at, gives up after `polls` polls, records the timeout and exits normally.
#include "tc_common.cuh"

namespace hgrn2 {

namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(uint32_t polls) {
    using namespace tc;
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);   // one arrival expected; none is ever made
        fence_mbar_init();
    }
    __syncthreads();
    const bool done = mbar_wait(&bar, 0, polls);
    if (!done && threadIdx.x == 0) set_status(HGRN2_ERR_TIMEOUT);
}

}  // namespace

}  // namespace hgrn2

extern "C" hgrn2_status hgrn2_selftest_wait_timeout(unsigned int polls, cudaStream_t stream) {
    if (polls < 1 || polls > (1u << 24)) return HGRN2_ERR_INVALID_ARG;
    hgrn2::wait_timeout_kernel<<<1, 32, 0, stream>>>(polls);
    return cudaGetLastError() == cudaSuccess ? HGRN2_OK : HGRN2_ERR_CUDA;
}
