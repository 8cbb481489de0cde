// launch.h -- host-side launchers of the kernels, shared by the C-ABI layer.
// Every launcher validates nothing (abi.cu does) and returns the CUDA error of
// the launch.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace ebl {

constexpr int kTileTokens = 128;  // router tile: tokens per tile (UMMA M), tile_counts row
constexpr int kMaxExperts = 256;  // N_r limit
constexpr int kMaxTopK = 8;       // K limit

// router_gemm.cu
int router_gemm_w_box_rows(int Nr);  // rows of W per TMA box (N_r / CTAs per MMA)
cudaError_t launch_router_gemm(const CUtensorMap &tmap_h, const CUtensorMap &tmap_w, const float *bias, int T,
                               int d, int Nr, int K, int32_t *topk_idx, float *gates, int32_t *counts,
                               int32_t *tile_counts, double *zloss_sum, float *tile_psum, int32_t *status,
                               int num_sms, cudaStream_t stream);

// router_logits.cu
// tile_psum != NULL (the balance option) needs the vector path: logits_vector_path()
bool logits_vector_path(const float *logits, int Nr);
cudaError_t launch_router_logits(const float *logits, const float *bias, int T, int Nr, int K, int32_t *topk_idx,
                                 float *gates, int32_t *counts, int32_t *tile_counts, float *tile_psum,
                                 int32_t *status, int num_sms, cudaStream_t stream);
cudaError_t launch_score_error(const float *x, int64_t n, float *max_err, float *exact_out, cudaStream_t stream);
cudaError_t launch_check_finite(const void *p, int64_t n, int bf16, int32_t *status, int num_sms,
                                cudaStream_t stream);
float logits_key_error_bound();

// bias_update.cu
cudaError_t launch_smebu(int32_t *counts, float *bias, float *momentum, int L, int Nr, float lambda, float beta,
                         float kappa, int linear, int reset_counts, float *maxvio_out, int32_t *status,
                         cudaStream_t stream);
cudaError_t launch_sign_update(int32_t *counts, float *bias, int Nr, float gamma, int reset_counts,
                               float *maxvio_out, int32_t *status, cudaStream_t stream);

// balance_logits.cu
cudaError_t launch_tile_psum_logits(const float *logits, int T, int Nr, float *tile_psum, int num_sms,
                                    cudaStream_t stream);

// seq_balance.cu
cudaError_t launch_seq_balance(const int32_t *tile_counts, const float *tile_psum, int T, int Nr, int K, int seq_len,
                               float alpha, double *loss_seq, double *loss, cudaStream_t stream);

// dispatch.cu
size_t dispatch_workspace_bytes(int T, int Nr);
cudaError_t launch_dispatch(const uint16_t *hidden, const int32_t *topk_idx, const int32_t *tile_counts, int T,
                            int d, int Nr, int K, int32_t *offsets, int32_t *perm, int32_t *dest,
                            uint16_t *dispatched, void *workspace, int32_t *status, int num_sms,
                            cudaStream_t stream);
cudaError_t launch_combine(const uint16_t *expert_out, const float *gates, const int32_t *dest, int T, int d,
                           int K, float *out, int32_t *status, int num_sms, cudaStream_t stream);

}  // namespace ebl
