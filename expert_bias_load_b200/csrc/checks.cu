// checks.cu -- input validation: a scan for NaN and infinities in an fp32 or
// bf16 buffer, reported through the status word.  The router assumes finite
// inputs; a caller that cannot vouch for them runs this first.
//
// A value is NaN or infinite exactly when its exponent bits are all ones
// (IEEE 754 binary32: bits 23..30; bfloat16: bits 7..14).  The buffer is read
// once: a head of at most 15 bytes up to the first 16-byte boundary, 16-byte
// vectors, and a tail, each checked by the same bit test.

#include "../../include/ebl.h"
#include "launch.h"

namespace ebl {
namespace {

constexpr int kCheckThreads = 256;

__device__ __forceinline__ bool word_bad(uint32_t w, bool bf16) {
    if (bf16) return (w & 0x7f80u) == 0x7f80u || (w & 0x7f800000u) == 0x7f800000u;
    return (w & 0x7f800000u) == 0x7f800000u;
}

__device__ __forceinline__ bool elem_bad(const uint8_t *p, bool bf16) {
    if (bf16) return (*reinterpret_cast<const uint16_t *>(p) & 0x7f80u) == 0x7f80u;
    return (*reinterpret_cast<const uint32_t *>(p) & 0x7f800000u) == 0x7f800000u;
}

// head: elements [0, n_head); vectors: 16-byte words [0, n_vec) from vec;
// tail: elements [0, n_tail) from tail.  esize = bytes per element.
__global__ void __launch_bounds__(kCheckThreads) check_finite_kernel(const uint8_t *__restrict__ head, int n_head,
                                                                     const uint4 *__restrict__ vec, int64_t n_vec,
                                                                     const uint8_t *__restrict__ tail, int n_tail,
                                                                     int esize, int32_t *__restrict__ status) {
    const bool bf16 = esize == 2;
    bool bad = false;
    const int64_t stride = (int64_t)gridDim.x * kCheckThreads;
    for (int64_t i = blockIdx.x * (int64_t)kCheckThreads + threadIdx.x; i < n_vec; i += stride) {
        const uint4 v = __ldcs(vec + i);
        bad |= word_bad(v.x, bf16) | word_bad(v.y, bf16) | word_bad(v.z, bf16) | word_bad(v.w, bf16);
    }
    if (blockIdx.x == 0) {
        if (threadIdx.x < n_head) bad |= elem_bad(head + (size_t)threadIdx.x * esize, bf16);
        if (threadIdx.x < n_tail) bad |= elem_bad(tail + (size_t)threadIdx.x * esize, bf16);
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(status, EBL_ST_NONFINITE);
}

}  // namespace

cudaError_t launch_check_finite(const void *p, int64_t n, int bf16, int32_t *status, int num_sms,
                                cudaStream_t stream) {
    if (n == 0) return cudaSuccess;
    const int esize = bf16 ? 2 : 4;
    const uint8_t *b = static_cast<const uint8_t *>(p);
    const uintptr_t addr = reinterpret_cast<uintptr_t>(b);
    int64_t n_head = (int64_t)(((16 - (addr & 15)) & 15) / esize);
    if (n_head > n) n_head = n;
    const int64_t per_vec = 16 / esize;
    const int64_t n_vec = (n - n_head) / per_vec;
    const int64_t n_tail = n - n_head - n_vec * per_vec;
    const uint8_t *vbase = b + n_head * esize;
    const uint8_t *tail = vbase + n_vec * 16;
    int64_t blocks = (n_vec + kCheckThreads - 1) / kCheckThreads;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    check_finite_kernel<<<(int)blocks, kCheckThreads, 0, stream>>>(b, (int)n_head, reinterpret_cast<const uint4 *>(vbase),
                                                                   n_vec, tail, (int)n_tail, esize, status);
    return cudaGetLastError();
}

}  // namespace ebl
