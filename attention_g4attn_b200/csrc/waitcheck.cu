// waitcheck.cu -- self-test of the bounded device waits.
//
// One thread initialises an mbarrier that expects one arrival, which nothing ever makes,
// and waits on it with the same bounded wait the attention kernels use.  The wait gives up
// after the poll limit (or 2 s), records G4ATTN_ERR_TIMEOUT in the device status word and
// returns; the kernel holds no copies, MMAs or tensor memory, so giving up is clean.
#include "kernels.h"
#include "sm100.cuh"

namespace g4 {
namespace {

__global__ void wait_selftest_kernel(int* status, long long limit) {
    __shared__ uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const WaitCtl wc{limit, status};
        mbar_wait(&bar, 0, wc, (volatile int*)&abort);   // gives up: nothing arrives
    }
}

}  // namespace

cudaError_t launch_wait_selftest(int* status, long long limit, cudaStream_t stream) {
    wait_selftest_kernel<<<1, 32, 0, stream>>>(status, limit);
    return cudaGetLastError();
}

}  // namespace g4
