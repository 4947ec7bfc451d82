// selftest.cu -- checks of the failure-detection path that fault nothing.
//
// Every device wait in this library is bounded: the grid barriers of the
// permuting quantizer and the mbarrier waits of the GEMM give up after
// fg8::kWaitLimitNs, record FG8_ERR_TIMEOUT in the caller's status word and
// return, so the CUDA context stays usable.  These kernels run exactly those
// wait routines on a condition that nothing will ever satisfy, so a test can
// watch the timeout happen and check the status.
#include "fg8_common.cuh"
#include "fg8_tma.cuh"

namespace {

using namespace fg8::tma;

// one CTA waits for two arrivals: the barrier never completes
__global__ void wait_on_grid_barrier_never_reached(uint32_t* counter, int32_t* status) {
    fg8::grid_barrier(counter, gridDim.x + 1, status);
}

// an mbarrier that nothing arrives on
__global__ void wait_on_mbarrier_never_completed(int32_t* status) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    mbar_wait(smem_u32(&bar), 0, &abort_flag, status);
}

}  // namespace

extern "C" fg8_status fg8_selftest_wait_timeout(int which, uint32_t* scratch, int32_t* dev_status,
                                                fg8_stream_t stream) {
    cudaStream_t st = (cudaStream_t)stream;
    if (!dev_status) return FG8_ERR_INVALID_ARG;
    if (which == 0) {
        if (!scratch) return FG8_ERR_INVALID_ARG;
        if (cudaMemsetAsync(scratch, 0, sizeof(uint32_t), st) != cudaSuccess) return FG8_ERR_CUDA;
        wait_on_grid_barrier_never_reached<<<1, 32, 0, st>>>(scratch, dev_status);
    } else if (which == 1) {
        wait_on_mbarrier_never_completed<<<1, 32, 0, st>>>(dev_status);
    } else {
        return FG8_ERR_INVALID_ARG;
    }
    return fg8h::launch_status();
}
