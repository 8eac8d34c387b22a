// Self-test of the kernels' bounded mbarrier wait, in a library of its own
// (libabattn_selftest.so) so that the measured kernels stay untouched.
//
// One warp waits on an mbarrier that nothing ever arrives on, with the same
// mbar_wait the kernels use: after its limit (about a second of SM clock) the
// wait gives up, raises the abort flag and the timeout bit of the device
// error word, and the kernel returns.  Nothing traps, faults or spins without
// end, so the CUDA context stays usable; the host reads the error word as a
// status, as abattn_check does for the kernels.
#include <cstdio>

#include "../csrc/common.cuh"
#include "../../include/abattn.h"
#include "../../include/abattn_selftest.h"

namespace abattn {
namespace {

__global__ void stalled_wait_kernel(int *waited) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // expects one arrival, which never comes
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const bool ok = mbar_wait(&bar, 0, reinterpret_cast<volatile int *>(&abort_flag));
    if (threadIdx.x == 0) *waited = ok ? 1 : 0;
}

int status_of(cudaError_t e) {
    if (e == cudaSuccess) return ABATTN_OK;
    fprintf(stderr, "abattn selftest: CUDA error %s\n", cudaGetErrorString(e));
    return ABATTN_ERR_CUDA;
}

}  // namespace
}  // namespace abattn

extern "C" __attribute__((visibility("default"))) int abattn_selftest_stalled_wait(int *waited, void *stream) {
    using namespace abattn;
    if (waited == nullptr) return ABATTN_ERR_NULL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int *d_waited = nullptr;
    cudaError_t e = cudaMalloc(&d_waited, sizeof(int));
    if (e != cudaSuccess) return status_of(e);
    int rc = ABATTN_OK;
    const int minus_one = -1;
    uint32_t word = 0;
    const uint32_t zero = 0;
    if ((e = cudaMemcpyAsync(d_waited, &minus_one, sizeof(int), cudaMemcpyHostToDevice, st)) != cudaSuccess) {
        rc = status_of(e);
    } else {
        stalled_wait_kernel<<<1, 32, 0, st>>>(d_waited);
        if ((e = cudaGetLastError()) != cudaSuccess || (e = cudaStreamSynchronize(st)) != cudaSuccess ||
            (e = cudaMemcpy(waited, d_waited, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess ||
            (e = cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word))) != cudaSuccess ||
            (e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero))) != cudaSuccess) {
            rc = status_of(e);
        } else if (word & kErrTimeout) {
            rc = ABATTN_ERR_TIMEOUT;
        }
    }
    cudaFree(d_waited);
    return rc;
}
