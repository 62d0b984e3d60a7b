// selftest.cu -- exercises the failure path of the kernels' bounded waits on the GPU.
//
// Every pipeline wait of the decode kernel is bounded: when its mbarrier phase does not complete
// within the bound, the wait gives up, the CTA raises the timeout bit of the device error word and
// exits, and mla_check_status reports MLA_ERR_TIMEOUT with the context still usable. This kernel
// runs the same wait primitive on an mbarrier that nothing ever arrives on, with a caller-chosen
// bound, so that path can be tested without any fault.
#include "common.cuh"
#include "sm100_ptx.cuh"

namespace mla {

__global__ void selftest_wait_kernel(long long spin_cycles) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        abort_flag = 0;
        sm100::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (!sm100::mbar_wait_for(&bar, 0, &abort_flag, spin_cycles)) raise_error(kErrTimeout);
        sm100::mbar_arrive(&bar);  // complete the phase, leaving the barrier consistent
    }
}

}  // namespace mla

extern "C" int mla_selftest_wait_timeout(int64_t spin_cycles, void *stream) {
    if (spin_cycles < 100000 || spin_cycles > 4000000000LL) return MLA_ERR_INVALID_ARG;
    const int rc = mla::check_device();
    if (rc != MLA_OK) return rc;
    mla::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((long long)spin_cycles);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
