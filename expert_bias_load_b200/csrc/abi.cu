// abi.cu -- the C entry points of libebl.so: argument checks, TMA descriptor
// encoding, kernel launches.  Declarations and contracts are in include/ebl.h.

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/ebl.h"
#include "launch.h"

namespace {

// Library-owned status word used when a caller passes status == NULL.
__device__ int32_t g_internal_status;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int g_num_sms[kMaxDevices];
int32_t *g_status_ptr[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// The last CUDA failure this thread saw inside the library (for ebl_last_cuda_error).
thread_local char g_last_error[160] = "none";

void record_error(const char *where, const char *what) {
    snprintf(g_last_error, sizeof g_last_error, "%s: %s", where, what);
}

int cuda_fail(const char *where, cudaError_t e) {
    record_error(where, cudaGetErrorString(e));
    (void)cudaGetLastError();  // clear a sticky launch error so the caller's context stays usable
    return EBL_ECUDA;
}

struct DeviceInfo {
    int num_sms;
    int32_t *internal_status;
};

// SM count and the internal status address of the current device (cached).
int device_info(DeviceInfo *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    if (dev < 0 || dev >= kMaxDevices) return EBL_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_num_sms[dev] == 0) {
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail("cudaDeviceGetAttribute", e);
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_internal_status);
        if (e != cudaSuccess) return cuda_fail("cudaGetSymbolAddress", e);
        g_status_ptr[dev] = static_cast<int32_t *>(p);
        g_num_sms[dev] = sms;
    }
    out->num_sms = g_num_sms[dev];
    out->internal_status = g_status_ptr[dev];
    return EBL_OK;
}

int get_encoder() {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_encode) return EBL_OK;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess) return cuda_fail("cudaGetDriverEntryPoint", e);
    if (q != cudaDriverEntryPointSuccess || fn == nullptr) {
        record_error("cudaGetDriverEntryPoint", "cuTensorMapEncodeTiled not found");
        return EBL_ECUDA;
    }
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    return EBL_OK;
}

// 2-D bf16 row-major [rows, cols] tensor, box [box_rows, 64 columns], 128-byte swizzle.
int encode_bf16_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char msg[64];
        snprintf(msg, sizeof msg, "CUresult %d", (int)r);
        record_error("cuTensorMapEncodeTiled", msg);
        return EBL_ECUDA;
    }
    return EBL_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int check_topk(int N_r, int K) {
    if (N_r < 1 || N_r > EBL_MAX_EXPERTS) return EBL_EINVAL;
    if (K < 1 || K > EBL_MAX_TOPK || K > N_r) return EBL_EINVAL;
    return EBL_OK;
}

int check_T(int T) { return (T < 0 || T > 2147483647 - 255) ? EBL_EINVAL : EBL_OK; }

}  // namespace

namespace {

int router_gemm_call(const uint16_t *hidden, const uint16_t *W_router, const float *bias, int T, int d, int N_r,
                     int K, int32_t *topk_idx, float *gates, int32_t *counts, int32_t *tile_counts,
                     double *zloss_sum, float *tile_psum, int32_t *status, ebl_stream_t stream) {
    if (check_T(T) || check_topk(N_r, K)) return EBL_EINVAL;
    if (d < 64 || d > (1 << 20) || d % 64 != 0) return EBL_EINVAL;
    if (N_r % 32 != 0) return EBL_EUNSUPPORTED;
    if (!W_router || !bias || !counts) return EBL_EINVAL;
    if (T > 0 && (!hidden || !topk_idx || !gates)) return EBL_EINVAL;  // T-sized buffers may be NULL when T == 0
    if (!aligned16(hidden) || !aligned16(W_router) || !aligned4(bias) || !aligned4(counts)) return EBL_EINVAL;
    if (K % 4 == 0 && (!aligned16(topk_idx) || !aligned16(gates))) return EBL_EINVAL;
    if (!aligned4(topk_idx) || !aligned4(gates) || (tile_counts && !aligned4(tile_counts))) return EBL_EINVAL;
    if (zloss_sum && (reinterpret_cast<uintptr_t>(zloss_sum) & 7u)) return EBL_EINVAL;
    if (tile_psum && (!aligned4(tile_psum) || (T > 0 && !tile_counts))) return EBL_EINVAL;
    if (T == 0) return EBL_OK;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    if ((rc = get_encoder())) return rc;
    CUtensorMap th, tw;
    if ((rc = encode_bf16_2d(&th, hidden, (uint64_t)T, (uint64_t)d, ebl::kTileTokens))) return rc;
    if ((rc = encode_bf16_2d(&tw, W_router, (uint64_t)N_r, (uint64_t)d, (uint32_t)ebl::router_gemm_w_box_rows(N_r))))
        return rc;
    cudaError_t e = ebl::launch_router_gemm(th, tw, bias, T, d, N_r, K, topk_idx, gates, counts, tile_counts,
                                            zloss_sum, tile_psum, status ? status : di.internal_status, di.num_sms,
                                            reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? EBL_OK : cuda_fail("kernel launch", e);
}

}  // namespace

extern "C" {

const char *ebl_strerror(int code) {
    switch (code) {
        case EBL_OK:
            return "ok";
        case EBL_EINVAL:
            return "invalid argument (null pointer, shape, size or alignment)";
        case EBL_EUNSUPPORTED:
            return "unsupported configuration";
        case EBL_ECUDA:
            return "CUDA runtime or driver error";
        case EBL_EDATA:
            return "invalid data";
        default:
            return "unknown error code";
    }
}

int ebl_version(void) { return 10000; }

const char *ebl_last_cuda_error(void) { return g_last_error; }

int ebl_tile_tokens(void) { return ebl::kTileTokens; }

int router_forward(const uint16_t *hidden, const uint16_t *W_router, const float *bias, int T, int d, int N_r,
                   int K, int32_t *topk_idx, float *gates, int32_t *counts, int32_t *tile_counts, int32_t *status,
                   ebl_stream_t stream) {
    return router_gemm_call(hidden, W_router, bias, T, d, N_r, K, topk_idx, gates, counts, tile_counts, nullptr,
                            nullptr, status, stream);
}

int router_forward_zloss(const uint16_t *hidden, const uint16_t *W_router, const float *bias, int T, int d,
                         int N_r, int K, int32_t *topk_idx, float *gates, int32_t *counts, int32_t *tile_counts,
                         double *zloss_sum, int32_t *status, ebl_stream_t stream) {
    if (!zloss_sum) return EBL_EINVAL;
    return router_gemm_call(hidden, W_router, bias, T, d, N_r, K, topk_idx, gates, counts, tile_counts, zloss_sum,
                            nullptr, status, stream);
}

int router_forward_balance(const uint16_t *hidden, const uint16_t *W_router, const float *bias, int T, int d,
                           int N_r, int K, int32_t *topk_idx, float *gates, int32_t *counts, int32_t *tile_counts,
                           float *tile_psum, double *zloss_sum, int32_t *status, ebl_stream_t stream) {
    if (T > 0 && (!tile_counts || !tile_psum)) return EBL_EINVAL;
    return router_gemm_call(hidden, W_router, bias, T, d, N_r, K, topk_idx, gates, counts, tile_counts, zloss_sum,
                            tile_psum, status, stream);
}

int balance_stats_logits(const float *logits, int T, int N_r, float *tile_psum, ebl_stream_t stream) {
    if (check_T(T) || N_r < 1 || N_r > EBL_MAX_EXPERTS) return EBL_EINVAL;
    if (T > 0 && (!logits || !tile_psum)) return EBL_EINVAL;
    if (!aligned4(logits) || !aligned4(tile_psum)) return EBL_EINVAL;
    if (T == 0) return EBL_OK;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    cudaError_t e = ebl::launch_tile_psum_logits(logits, T, N_r, tile_psum, di.num_sms,
                                                 reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? EBL_OK : cuda_fail("kernel launch", e);
}

int seq_balance_loss(const int32_t *tile_counts, const float *tile_psum, int T, int N_r, int K, int seq_len,
                     float alpha, double *loss_seq, double *loss, ebl_stream_t stream) {
    if (check_T(T) || check_topk(N_r, K)) return EBL_EINVAL;
    if (seq_len <= 0 || seq_len % ebl::kTileTokens != 0 || T % seq_len != 0) return EBL_EINVAL;
    if (!(alpha == alpha) || alpha > 3.0e38f || alpha < -3.0e38f) return EBL_EINVAL;  // NaN or infinite
    if (T == 0) return EBL_OK;
    if (!tile_counts || !tile_psum || !loss_seq || !loss) return EBL_EINVAL;
    if (!aligned4(tile_counts) || !aligned4(tile_psum)) return EBL_EINVAL;
    if ((reinterpret_cast<uintptr_t>(loss_seq) & 7u) || (reinterpret_cast<uintptr_t>(loss) & 7u)) return EBL_EINVAL;
    cudaError_t e = ebl::launch_seq_balance(tile_counts, tile_psum, T, N_r, K, seq_len, alpha, loss_seq, loss,
                                            reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? EBL_OK : cuda_fail("kernel launch", e);
}

int router_forward_logits(const float *logits, const float *bias, int T, int N_r, int K, int32_t *topk_idx,
                          float *gates, int32_t *counts, int32_t *tile_counts, int32_t *status,
                          ebl_stream_t stream) {
    if (check_T(T) || check_topk(N_r, K)) return EBL_EINVAL;
    if (!bias || !counts) return EBL_EINVAL;
    if (T > 0 && (!logits || !topk_idx || !gates)) return EBL_EINVAL;  // T-sized buffers may be NULL when T == 0
    if (!aligned4(logits) || !aligned4(bias) || !aligned4(topk_idx) || !aligned4(gates) || !aligned4(counts))
        return EBL_EINVAL;
    if (tile_counts && !aligned4(tile_counts)) return EBL_EINVAL;
    if (T == 0) return EBL_OK;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    cudaError_t e = ebl::launch_router_logits(logits, bias, T, N_r, K, topk_idx, gates, counts, tile_counts, nullptr,
                                              status ? status : di.internal_status, di.num_sms,
                                              reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? EBL_OK : cuda_fail("kernel launch", e);
}

int router_forward_logits_balance(const float *logits, const float *bias, int T, int N_r, int K, int32_t *topk_idx,
                                  float *gates, int32_t *counts, int32_t *tile_counts, float *tile_psum,
                                  int32_t *status, ebl_stream_t stream) {
    if (check_T(T) || check_topk(N_r, K)) return EBL_EINVAL;
    if (!bias || !counts) return EBL_EINVAL;
    if (T > 0 && (!logits || !topk_idx || !gates || !tile_counts || !tile_psum)) return EBL_EINVAL;
    if (!aligned4(logits) || !aligned4(bias) || !aligned4(topk_idx) || !aligned4(gates) || !aligned4(counts) ||
        !aligned4(tile_counts) || !aligned4(tile_psum))
        return EBL_EINVAL;
    if (T == 0) return EBL_OK;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t *stw = status ? status : di.internal_status;
    cudaError_t e;
    if (ebl::logits_vector_path(logits, N_r)) {
        e = ebl::launch_router_logits(logits, bias, T, N_r, K, topk_idx, gates, counts, tile_counts, tile_psum, stw,
                                      di.num_sms, st);
    } else {  // any N_r and alignment: the row kernel, then the balance statistics as their own pass
        e = ebl::launch_router_logits(logits, bias, T, N_r, K, topk_idx, gates, counts, tile_counts, nullptr, stw,
                                      di.num_sms, st);
        if (e == cudaSuccess) e = ebl::launch_tile_psum_logits(logits, T, N_r, tile_psum, di.num_sms, st);
    }
    return e == cudaSuccess ? EBL_OK : cuda_fail("kernel launch", e);
}

int smebu_step_layers(int32_t *counts, float *bias, float *momentum, int L, int N_r, float lambda, float beta,
                      float kappa, int linear, int reset_counts, float *maxvio_out, int32_t *status,
                      ebl_stream_t stream) {
    if (L < 1 || L > 65535 || N_r < 1 || N_r > EBL_MAX_EXPERTS) return EBL_EINVAL;
    if (!counts || !bias || !momentum) return EBL_EINVAL;
    if (!aligned4(counts) || !aligned4(bias) || !aligned4(momentum)) return EBL_EINVAL;
    if (maxvio_out && !aligned4(maxvio_out)) return EBL_EINVAL;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    cudaError_t e = ebl::launch_smebu(counts, bias, momentum, L, N_r, lambda, beta, kappa, linear, reset_counts,
                                      maxvio_out, status ? status : di.internal_status,
                                      reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? EBL_OK : cuda_fail("kernel launch", e);
}

int smebu_step(int32_t *counts, float *bias, float *momentum, int N_r, float lambda, float beta, float kappa,
               int reset_counts, float *maxvio_out, int32_t *status, ebl_stream_t stream) {
    return smebu_step_layers(counts, bias, momentum, 1, N_r, lambda, beta, kappa, 0, reset_counts, maxvio_out,
                             status, stream);
}

int sign_update_step(int32_t *counts, float *bias, int N_r, float gamma, int reset_counts, float *maxvio_out,
                     int32_t *status, ebl_stream_t stream) {
    if (N_r < 1 || N_r > EBL_MAX_EXPERTS) return EBL_EINVAL;
    if (!counts || !bias || !aligned4(counts) || !aligned4(bias)) return EBL_EINVAL;
    if (maxvio_out && !aligned4(maxvio_out)) return EBL_EINVAL;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    cudaError_t e = ebl::launch_sign_update(counts, bias, N_r, gamma, reset_counts, maxvio_out,
                                            status ? status : di.internal_status,
                                            reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? EBL_OK : cuda_fail("kernel launch", e);
}

size_t ebl_dispatch_workspace_bytes(int T, int N_r) {
    if (T < 0 || N_r < 1 || N_r > EBL_MAX_EXPERTS) return 0;
    return ebl::dispatch_workspace_bytes(T, N_r);
}

int moe_dispatch(const uint16_t *hidden, const int32_t *topk_idx, const int32_t *tile_counts, int T, int d,
                 int N_r, int K, int32_t *offsets, int32_t *perm, int32_t *dest, uint16_t *dispatched,
                 void *workspace, size_t workspace_bytes, int32_t *status, ebl_stream_t stream) {
    if (check_T(T) || check_topk(N_r, K)) return EBL_EINVAL;
    if ((long long)T * K > 2147483647LL) return EBL_EINVAL;
    if (d < 8 || d % 8 != 0 || d > (1 << 24)) return EBL_EINVAL;
    if (!offsets) return EBL_EINVAL;
    if (T > 0 && (!hidden || !topk_idx || !perm || !dest || !dispatched || !workspace)) return EBL_EINVAL;
    if (!aligned16(hidden) || !aligned16(dispatched) || !aligned16(workspace)) return EBL_EINVAL;
    if (!aligned4(topk_idx) || !aligned4(offsets) || !aligned4(perm) || !aligned4(dest)) return EBL_EINVAL;
    if (tile_counts && !aligned4(tile_counts)) return EBL_EINVAL;
    if (workspace_bytes < ebl::dispatch_workspace_bytes(T, N_r)) return EBL_EINVAL;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) {  // offsets of an empty batch are all zero
        cudaError_t e = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (size_t)(N_r + 1), st);
        return e == cudaSuccess ? EBL_OK : cuda_fail("cudaMemsetAsync", e);
    }
    cudaError_t e = ebl::launch_dispatch(hidden, topk_idx, tile_counts, T, d, N_r, K, offsets, perm, dest,
                                         dispatched, workspace, status ? status : di.internal_status, di.num_sms,
                                         st);
    return e == cudaSuccess ? EBL_OK : cuda_fail("kernel launch", e);
}

int moe_combine(const uint16_t *expert_out, const float *gates, const int32_t *dest, int T, int d, int K,
                float *out, int32_t *status, ebl_stream_t stream) {
    if (check_T(T) || K < 1 || K > EBL_MAX_TOPK) return EBL_EINVAL;
    if ((long long)T * K > 2147483647LL) return EBL_EINVAL;
    if (d < 8 || d % 8 != 0 || d > (1 << 24)) return EBL_EINVAL;
    if (T > 0 && (!expert_out || !gates || !dest || !out)) return EBL_EINVAL;
    if (!aligned16(expert_out) || !aligned16(out) || !aligned4(gates) || !aligned4(dest)) return EBL_EINVAL;
    if (T == 0) return EBL_OK;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    cudaError_t e = ebl::launch_combine(expert_out, gates, dest, T, d, K, out,
                                        status ? status : di.internal_status, di.num_sms,
                                        reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? EBL_OK : cuda_fail("kernel launch", e);
}

static int check_finite_call(const void *x, int64_t n, int bf16, int32_t *status, ebl_stream_t stream) {
    if (n < 0 || !status || !aligned4(status)) return EBL_EINVAL;
    if (n > 0 && (!x || (reinterpret_cast<uintptr_t>(x) & (bf16 ? 1u : 3u)))) return EBL_EINVAL;
    if (n == 0) return EBL_OK;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    cudaError_t e = ebl::launch_check_finite(x, n, bf16, status, di.num_sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? EBL_OK : cuda_fail("kernel launch", e);
}

int ebl_check_finite_f32(const float *x, int64_t n, int32_t *status, ebl_stream_t stream) {
    return check_finite_call(x, n, 0, status, stream);
}

int ebl_check_finite_bf16(const uint16_t *x, int64_t n, int32_t *status, ebl_stream_t stream) {
    return check_finite_call(x, n, 1, status, stream);
}

int ebl_read_internal_status(int32_t *out, int clear) {
    if (!out) return EBL_EINVAL;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    cudaError_t e = cudaMemcpy(out, di.internal_status, sizeof(int32_t), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail("cudaMemcpy", e);
    if (clear && (e = cudaMemset(di.internal_status, 0, sizeof(int32_t))) != cudaSuccess) return cuda_fail("cudaMemset", e);
    return EBL_OK;
}

}  // extern "C"
