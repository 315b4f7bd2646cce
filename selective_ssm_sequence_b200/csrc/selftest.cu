// selftest.cu -- the library's failure path exercised on purpose, without a
// fault: one thread block waits on an mbarrier that nothing ever signals,
// through tc::mbar_wait -- the bounded wait every pipelined kernel of the
// library uses -- with a small poll limit.  The wait gives up, raises the
// block's abort flag and records HM_ERR_TIMEOUT (kernel id, block, site) in
// the device error word, exactly as a stalled pipeline would; the other lanes
// see the abort flag and leave with it.  The context stays usable; the host
// reads the status with hm_get_device_error.
#include "tc_common.cuh"

namespace hm {

namespace {

__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(uint32_t polls, DevErr err) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);   // one arrival expected; none is ever made
        abort_flag = 0;
        tc::mbar_fence_init();
    }
    __syncwarp();
    bool ok = true;
    if (threadIdx.x == 0) ok = tc::mbar_wait(&bar, 0, &abort_flag, err, KID_SELFTEST, 1, polls);
    // the whole warp leaves together, as the pipelined kernels' roles do
    ok = __all_sync(0xffffffffu, ok);
    (void)ok;
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
