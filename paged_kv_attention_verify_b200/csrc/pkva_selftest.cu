// Self-test of the bounded device wait that every kernel of this library uses.
//
// One block initialises an mbarrier that nothing will complete and waits on it with the
// same polling as the kernels, but with a caller-chosen time limit. The wait must give up
// and report PKVA_DEVERR_TIMEOUT in the error word instead of hanging the GPU: this is how
// a lost asynchronous copy would surface from attn_run (through attn_check).
#include <cuda_runtime.h>

#include <string>

#include "pkva.h"
#include "pkva_ptx.cuh"

namespace pkva {
void set_last_error(const std::string& msg);
namespace {

__global__ void wait_timeout_kernel(int* err, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x != 0) return;
    const unsigned long long t0 = global_timer_ns();
    while (!mbar_try_wait(&bar, 0)) {                 // phase 0 never completes
        if (global_timer_ns() - t0 > limit_ns) {
            atomicOr(err, PKVA_DEVERR_TIMEOUT);
            return;
        }
    }
}

}  // namespace
}  // namespace pkva

extern "C" int pkva_selftest_wait_timeout(long long limit_ns, int32_t* device_error) {
    using namespace pkva;
    if (limit_ns <= 0 || limit_ns > 1000000000LL || !device_error) {
        set_last_error("pkva_selftest_wait_timeout: limit must be in (0, 1 s] and device_error non-NULL");
        return PKVA_EINVAL;
    }
    int* d_err = nullptr;
    cudaError_t e = cudaMalloc(&d_err, sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(d_err, 0, sizeof(int));
    if (e == cudaSuccess) {
        wait_timeout_kernel<<<1, 32>>>(d_err, (unsigned long long)limit_ns);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    int h = 0;
    if (e == cudaSuccess) e = cudaMemcpy(&h, d_err, sizeof(int), cudaMemcpyDeviceToHost);
    cudaFree(d_err);
    if (e != cudaSuccess) {
        set_last_error(std::string("pkva_selftest_wait_timeout: ") + cudaGetErrorString(e));
        return PKVA_ECUDA;
    }
    *device_error = h;
    return PKVA_OK;
}
