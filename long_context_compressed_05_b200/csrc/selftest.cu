// Self-test of the bounded device-side wait that every pipelined kernel here uses (no counterpart in
// the method): one thread waits on an mbarrier phase that nothing completes, gives up after the wait
// limit, records HCSA_ERR_TIMEOUT in the device status word and returns.  Nothing faults or hangs, and
// the context stays usable for the next call.
#include "tc_common.cuh"

namespace hcsa {
namespace {

__global__ void wait_timeout_selftest_kernel(int *status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        tc::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)tc::mbar_wait(&bar, 0, status);   // no arrival will ever come
}

}  // namespace
}  // namespace hcsa

extern "C" hcsa_status hcsa_selftest_wait_timeout(void *stream) {
    int *st = hcsa::device_status_ptr();
    if (!st) return HCSA_ERR_CUDA;
    hcsa::wait_timeout_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(st);
    hcsa::count_launch();
    return hcsa::check_launch();
}
