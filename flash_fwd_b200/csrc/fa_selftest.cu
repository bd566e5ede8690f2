// fa_selftest.cu -- failure-detection self-test (fa_selftest_wait_timeout in
// include/fa.h).  It runs the library's own bounded wait (wait_bar of
// fa_common.cuh) on an mbarrier phase that nothing completes, so that a test
// can watch the timeout path end to end on a GPU: the wait gives up after its
// bound, raises the CTA's abort flag (every other waiting warp then leaves at
// once), records FA_ERR_TIMEOUT and the site in the device words, and the
// kernel returns.  No access is out of bounds, nothing is left in flight, and
// the context stays usable.  This translation unit has its own copies of the
// device words (they are static), read back by the entry point itself.
#include <cuda_runtime.h>

#include "fa.h"
#include "fa_common.cuh"

namespace {

constexpr unsigned long long kStaggerNs = 100000000ull;   // 100 ms between the warps' waits

__global__ void __launch_bounds__(1024, 1) selftest_wait_kernel() {
    __shared__ __align__(8) unsigned long long bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        fa::mbar_init(fa::smem_u32(&bar), 1);   // one arrival completes phase 0; none comes
        abort_flag = 0;
        fa::mbar_fence_init();
    }
    __syncthreads();
    // warp w starts its wait w x 100 ms after the CTA starts: when the first
    // warp reaches the bound, the last ones are still well inside their own
    // bounds and can only leave early through the abort flag
    const unsigned long long t0 = fa::globaltimer();
    const unsigned long long delay = (threadIdx.x >> 5) * kStaggerNs;
    while (fa::globaltimer() - t0 < delay) __nanosleep(1000);
    fa::wait_bar(fa::smem_u32(&bar), 0u, &abort_flag);
}

}  // namespace

extern "C" FA_API int fa_selftest_wait_timeout(int warps, void *stream, int *site) {
    if (warps < 1 || warps > 32 || !site) return FA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int zero[6] = {0, 0, 0, 0, 0, 0};
    if (cudaMemcpyToSymbol(fa::g_dev_status, zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
    if (cudaMemcpyToSymbol(fa::g_dev_site, zero, 5 * sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
    selftest_wait_kernel<<<1, 32 * warps, 0, s>>>();
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return FA_ERR_CUDA;
    int status = 0;
    if (cudaMemcpyFromSymbol(&status, fa::g_dev_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
    if (cudaMemcpyFromSymbol(site, fa::g_dev_site, 5 * sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
    return status;
}
