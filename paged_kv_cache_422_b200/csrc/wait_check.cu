// The time-bounded wait of the tensor-core kernels, checked on its own.  Every mbarrier
// wait in the prefill and shared-prefix kernels gives up after kWaitLimitNs (2 s), ORs
// NVPA_FLAG_TIMEOUT into the caller's error word and winds its CTA down, so a protocol
// error or a lost copy ends in a status, never in a hung GPU.  This kernel waits, with
// that same function, on a barrier that nothing arrives at: the wait must run out, set
// the flag and return, and the context must stay usable for the next call.
#include "nvpa_internal.h"
#include "sm100.cuh"

namespace nvpa {

using namespace sm100;

namespace {

__global__ void __launch_bounds__(32) bounded_wait_check_kernel(int32_t* err_flag) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, &abort_flag, err_flag);
}

}  // namespace

nvpa_status_t run_bounded_wait_check(int32_t* err_flag, cudaStream_t stream) {
    bounded_wait_check_kernel<<<1, 32, 0, stream>>>(err_flag);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_failure(e, "bounded wait check launch");
    count_launches(1);
    return NVPA_OK;
}

}  // namespace nvpa
