// selftest.cu -- self-tests of two device-side assumptions.
//
// ebl_selftest_wait_timeout: the bounded pipeline wait that every kernel here
// uses.  One thread waits, with a short limit, on an mbarrier that nothing
// arrives on; the wait must give up, the kernel must report EBL_ST_TIMEOUT in
// the status word and return, and the CUDA context must stay usable.
//
// ebl_selftest_score_error: the distance between the approximate score the
// logits-mode ranking uses and the exact one, against the bound that ranking
// assumes.

#include "../../include/ebl.h"
#include "launch.h"
#include "ptx.cuh"

namespace ebl {
namespace {

__global__ void wait_timeout_kernel(int32_t *__restrict__ status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // expects one arrival that never comes
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort_flag, limit_ns)) atomicOr(status, kStTimeout);
}

}  // namespace
}  // namespace ebl

extern "C" int ebl_selftest_wait_timeout(int32_t *status, unsigned int limit_us, ebl_stream_t stream) {
    if (!status || (reinterpret_cast<uintptr_t>(status) & 3u)) return EBL_EINVAL;
    if (limit_us < 1 || limit_us > 1000000) return EBL_EINVAL;
    ebl::wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(status, 1000ull * limit_us);
    if (cudaGetLastError() != cudaSuccess) return EBL_ECUDA;
    return EBL_OK;
}

extern "C" int ebl_selftest_score_error(const float *x, int64_t n, float *max_err, float *bound, float *exact_out,
                                        ebl_stream_t stream) {
    if (n < 0 || !max_err || (reinterpret_cast<uintptr_t>(max_err) & 3u)) return EBL_EINVAL;
    if (n > 0 && (!x || (reinterpret_cast<uintptr_t>(x) & 3u))) return EBL_EINVAL;
    if (exact_out && (reinterpret_cast<uintptr_t>(exact_out) & 3u)) return EBL_EINVAL;
    if (bound) *bound = ebl::logits_key_error_bound();
    if (ebl::launch_score_error(x, n, max_err, exact_out, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return EBL_ECUDA;
    return EBL_OK;
}
