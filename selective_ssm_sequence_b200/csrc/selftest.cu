// selftest.cu -- the library's failure path exercised on purpose, without a
// fault: one thread block waits on an mbarrier that nothing ever signals, with
// the same bounded-poll wait the pipelined kernels use, gives up after `polls`
// polls and records HM_ERR_TIMEOUT in the device error word.  The context
// stays usable; the host reads the status with hm_get_device_error.
#include "tc_common.cuh"

namespace hm {

namespace {

__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(uint32_t polls, DevErr err) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);   // one arrival expected; none is ever made
        tc::mbar_fence_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) {
        bool done = false;
        for (uint32_t i = 0; i < polls && !done; ++i) done = tc::mbar_try_wait(&bar, 0);
        if (!done) report_error(err, HM_ERR_TIMEOUT, KID_SELFTEST, 1);
    }
}

}  // namespace

}  // namespace hm

extern "C" {

hm_status hm_selftest_wait_timeout(uint32_t polls, hm_stream_t stream) {
    if (polls == 0 || polls > (1u << 20)) return HM_ERR_INVALID_ARG;
    unsigned int *w = hm::device_error_word();
    if (!w) return HM_ERR_CUDA;
    hm::wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(polls, hm::DevErr{w});
    hm::count_launches(1);
    return cudaGetLastError() == cudaSuccess ? HM_OK : HM_ERR_CUDA;
}

}  // extern "C"
