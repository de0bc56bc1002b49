// tq_selftest.cu -- exercises the device-side failure path every kernel relies on: a bounded
// mbarrier wait that runs out reports TQ_ERR_TIMEOUT through dev_status and returns, leaving the
// context usable.  The barrier is initialised and never arrived at, so nothing faults or hangs.
#include "tq_internal.cuh"
#include "tq_sm100.cuh"

namespace tq {
namespace {

__global__ void wait_timeout_kernel(uint64_t timeout_ns, int32_t *dev_status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        abort_flag = 0;
        sm100::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // no thread ever arrives: the wait can only end by its time limit
        const bool done = sm100::mbar_wait_ns(&bar, 0, (volatile int *)&abort_flag, timeout_ns);
        if (!done && dev_status) atomicExch(dev_status, (int)TQ_ERR_TIMEOUT);
    }
}

}  // namespace
}  // namespace tq

extern "C" tq_status tq_selftest_wait_timeout(int32_t *dev_status, uint32_t timeout_ms, tq_stream_t stream) {
    if (!dev_status || timeout_ms == 0 || timeout_ms > 10000) return TQ_ERR_INVALID_ARG;
    tq::wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)timeout_ms * 1000000ull, dev_status);
    return cudaGetLastError() == cudaSuccess ? TQ_OK : TQ_ERR_CUDA;
}
