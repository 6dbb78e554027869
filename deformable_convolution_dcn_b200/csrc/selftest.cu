// Failure-detection self-test: one thread waits on an mbarrier that nothing
// ever arrives at, through the same bounded wait every tensor-core kernel uses.
// The wait gives up after `limit` clock cycles, records kStatusTimeout in the
// device status word and returns, so the kernel ends normally: nothing faults,
// traps or hangs, and the next dcn_check_status() reports DCN_ERR_TIMEOUT.
#include "kernels.h"
#include "tc_ptx.cuh"

namespace dcn {
namespace {

__global__ void selftest_wait_kernel(unsigned* status, long long limit) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(ptx::smem_u32(&bar), 1);
        abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::mbar_wait(ptx::smem_u32(&bar), 0, &abort_flag, status, limit);
    }
}

}  // namespace

cudaError_t selftest_wait_timeout(long long limit_cycles, cudaStream_t st) {
    unsigned* status = nullptr;
    cudaError_t e = status_word_ptr(&status);
    if (e != cudaSuccess) return e;
    selftest_wait_kernel<<<1, 32, 0, st>>>(status, limit_cycles);
    return cudaGetLastError();
}

}  // namespace dcn
