// Diagnostic: the library's bounded mbarrier wait, exercised on a barrier that
// nothing arrives at.  The wait must give up by itself (after its bound, about
// 2 s at most), report PA_DEVERR_TIMEOUT and let the kernel return, leaving the
// context usable.  No fault, trap or endless loop is involved.
#include "pa_device.cuh"
#include "pa_host.h"

namespace pa {

__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel(int32_t* err_word, int32_t* outcome) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncwarp();
    const bool done = __all_sync(0xffffffffu, mbar_wait(&bar, 0));  // phase 0 never completes
    if (threadIdx.x == 0) {
        if (!done) report(err_word, PA_DEVERR_TIMEOUT);
        if (outcome) *outcome = done ? 1 : 0;
    }
}

}  // namespace pa

extern "C" int pa_selftest_bounded_wait(int32_t* err_word, int32_t* outcome, void* stream) {
    using namespace pa;
    if ((err_word && !aligned4(err_word)) || (outcome && !aligned4(outcome))) return PA_ERR_INVALID_ARG;
    bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err_word, outcome);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
