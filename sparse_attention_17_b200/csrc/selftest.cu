// selftest.cu -- exercises the library's failure path for pipeline waits.
//
// Every wait of the kernels on an mbarrier (a stage of copies, a tensor-core commit) is
// bounded in time by mbar_wait: when the phase never completes -- a bug, or a copy that
// never lands -- the waiting thread records DSA_DEVERR_TIMEOUT in the device error word
// and the kernel unwinds, so the context stays usable and the host learns of it from
// dsa_check_device_errors.  This kernel waits on an mbarrier that nothing arrives on, so
// that the same bounded wait runs out; it touches no memory but its own shared memory and
// the error word.
#include "dsa_common.cuh"
#include "launch.h"

namespace dsa {

namespace {

__global__ void wait_timeout_selftest_kernel(unsigned* err, int* gave_up) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival expected; none will come
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) *gave_up = mbar_wait(&bar, 0, &abort_flag, err) ? 0 : 1;
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(int* gave_up, cudaStream_t stream, const DevCtx& ctx) {
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(ctx.err, gave_up);
    return cudaGetLastError();
}

}  // namespace dsa
