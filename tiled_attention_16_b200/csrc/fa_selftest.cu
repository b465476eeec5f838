// fa_selftest.cu — a self-test of the failure detection every kernel of the
// library relies on: the bounded mbarrier wait, the device status word it
// records into, and the CTA abort flag that ends the other waits of the CTA.
//
// One CTA, two waiting threads, two mbarriers that nothing ever completes.
// Thread 0 waits on the first; after the wait limit it records `site` in the
// status word and raises the abort flag.  Thread 32 starts waiting on the
// second a quarter of the limit later, so its own limit comes after the first
// one's; it must leave through the abort flag without recording `site2`.  No
// global memory, TMA, tensor-core or TMEM work is involved: the kernel ends
// after about one wait limit whatever happens.
#include "sm100.cuh"

#include "fa.h"

#include <cuda_runtime.h>

namespace fa {
namespace {

__global__ void __launch_bounds__(64) fa_selftest_wait_kernel(int site, int site2) {
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ int abort_word;
    volatile int* abort_flag = &abort_word;
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        mbar_wait(&bars[0], 0, abort_flag, site);   // nothing arrives: gives up at the limit
    } else if (threadIdx.x == 32) {
        const unsigned long long t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < kWaitLimitNs / 4) {
        }
        mbar_wait(&bars[1], 0, abort_flag, site2);  // ends through the abort flag
    }
}

}  // namespace
}  // namespace fa

extern "C" {

fa_status fa_selftest_wait_timeout(int site, int site2, void* stream) {
    if (site < 0 || site > 31 || site2 < 0 || site2 > 31 || site == site2) return FA_ERR_INVALID_ARG;
    fa::fa_selftest_wait_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(site, site2);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"
