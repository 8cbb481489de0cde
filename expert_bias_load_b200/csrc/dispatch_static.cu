// dispatch_static.cu -- moe_dispatch_static: moe_dispatch for callers that
// cannot allocate device memory.  The dispatch passes need scratch (per-tile
// and per-segment expert counts); here it lives in a fixed-size array that
// belongs to the library instead of a caller-provided workspace.  See
// include/ebl.h for the contract.

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/ebl.h"
#include "launch.h"

namespace {

// The scratch.  Every GPU that loads this library holds it until the process
// exits.  Device code may name it directly; host code must not pass its name
// to a kernel (on the host it is only a stand-in symbol), so the device
// address is looked up once per device with cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_dispatch_scratch[EBL_DISPATCH_STATIC_SCRATCH_BYTES];

// Receives device-side error bits when the caller passes status == NULL.
static __device__ int32_t g_dispatch_static_status;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices];
int32_t *g_status_addr[kMaxDevices];
int g_sms[kMaxDevices];

// One-time set-up for the current device: device addresses of the scratch
// and of the fallback status word, and the SM count.
int setup_current_device(void **scratch, int32_t **status_word, int *sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return EBL_ECUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return EBL_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr, *q = nullptr;
        int n = 0;
        cudaError_t e = cudaGetSymbolAddress(&p, g_dispatch_scratch);
        if (e == cudaSuccess) e = cudaGetSymbolAddress(&q, g_dispatch_static_status);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess || p == nullptr || q == nullptr) {
            (void)cudaGetLastError();
            return EBL_ECUDA;
        }
        g_status_addr[dev] = static_cast<int32_t *>(q);
        g_sms[dev] = n;
        g_scratch_addr[dev] = p;
    }
    *scratch = g_scratch_addr[dev];
    *status_word = g_status_addr[dev];
    *sms = g_sms[dev];
    return EBL_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" int moe_dispatch_static(const uint16_t *hidden, const int32_t *topk_idx, const int32_t *tile_counts,
                                   int T, int d, int N_r, int K, int32_t *offsets, int32_t *perm, int32_t *dest,
                                   uint16_t *dispatched, int32_t *status, ebl_stream_t stream) {
    if (T < 0 || T > 2147483647 - 255) return EBL_EINVAL;
    if (N_r < 1 || N_r > EBL_MAX_EXPERTS || K < 1 || K > EBL_MAX_TOPK || K > N_r) return EBL_EINVAL;
    if ((long long)T * K > 2147483647LL) return EBL_EINVAL;
    if (d < 8 || d % 8 != 0 || d > (1 << 24)) return EBL_EINVAL;
    if (!offsets) return EBL_EINVAL;
    if (T > 0 && (!hidden || !topk_idx || !perm || !dest || !dispatched)) return EBL_EINVAL;
    if (!aligned16(hidden) || !aligned16(dispatched)) return EBL_EINVAL;
    if (!aligned4(topk_idx) || !aligned4(offsets) || !aligned4(perm) || !aligned4(dest)) return EBL_EINVAL;
    if (tile_counts && !aligned4(tile_counts)) return EBL_EINVAL;
    // the problem's scratch must fit the fixed array
    if (ebl::dispatch_workspace_bytes(T, N_r) > (size_t)EBL_DISPATCH_STATIC_SCRATCH_BYTES) return EBL_EINVAL;

    void *scratch = nullptr;
    int32_t *own_status = nullptr;
    int sms = 0;
    int rc = setup_current_device(&scratch, &own_status, &sms);
    if (rc != EBL_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) {
        cudaError_t e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (size_t)(N_r + 1), st);
        if (e != cudaSuccess) {
            (void)cudaGetLastError();
            return EBL_ECUDA;
        }
        return EBL_OK;
    }
    // Every pass overwrites the scratch it later reads, so nothing left there
    // by an earlier call needs clearing.
    cudaError_t e = ebl::launch_dispatch(hidden, topk_idx, tile_counts, T, d, N_r, K, offsets, perm, dest,
                                         dispatched, scratch, status ? status : own_status, sms, st);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return EBL_ECUDA;
    }
    return EBL_OK;
}
