// seq_balance.cu -- the sequence-wise balance loss from the router's per-tile
// statistics.
//
// "SMEBU Load Balancing" ("How it works") keeps a small sequence-wise balance
// loss, eqs. (29)-(32), with coefficient alpha (5e-5 on the Large
// checkpoint), beside the bias balancing; the pages do not print it.  It is
// read as the complementary sequence-wise balance loss of auxiliary-loss-free
// balancing: for a sequence of S tokens,
//   f_i = N_r / (K S) * n_i       n_i: the sequence's selections of expert i
//   P_i = (1 / S) * q_i           q_i: sum over its tokens of s_i / sum_j s_j
//   L   = alpha * sum_i f_i P_i = alpha N_r / (K S^2) * sum_i n_i q_i
// and the batch value is the mean of L over the T / S sequences.  The router
// (GEMM mode, balance option) writes n and q per 128-token tile; S is a
// multiple of 128, so each sequence owns S / 128 whole tiles.
//
// Two launches, both deterministic: one CTA per sequence gathers its tiles
// (thread i owns expert i; tiles in order, fp64) and reduces sum_i n_i q_i
// over the experts in a fixed tree; then one CTA averages the sequences in a
// fixed order.  The work is (T / 128) x N_r x 8 bytes of reads: 16 MB at
// T = 2^20, N_r = 256, a few microseconds.

#include "launch.h"

namespace ebl {
namespace {

constexpr int kSeqThreads = 256;  // >= N_r

// Fixed-order sum of one value per thread of the CTA (thread 0 gets the sum).
__device__ __forceinline__ double block_sum(double v, double *red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_down_sync(0xffffffffu, v, off);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    v = 0.0;
    if (warp == 0) {
        if (lane < (int)(blockDim.x >> 5)) v = red[lane];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_down_sync(0xffffffffu, v, off);
    }
    return v;
}

__global__ void __launch_bounds__(kSeqThreads) seq_loss_kernel(const int32_t *__restrict__ tile_counts,
                                                               const float *__restrict__ tile_psum, int Nr,
                                                               int tiles_per_seq, double scale,
                                                               double *__restrict__ loss_seq) {
    __shared__ double red[kSeqThreads / 32];
    const int i = threadIdx.x;
    double nq = 0.0;
    if (i < Nr) {
        const size_t base = (size_t)blockIdx.x * tiles_per_seq * Nr + i;
        long long n = 0;
        double q = 0.0;
        for (int j = 0; j < tiles_per_seq; ++j) {
            n += tile_counts[base + (size_t)j * Nr];
            q += (double)tile_psum[base + (size_t)j * Nr];
        }
        nq = (double)n * q;
    }
    const double sum = block_sum(nq, red);
    if (threadIdx.x == 0) loss_seq[blockIdx.x] = scale * sum;
}

__global__ void __launch_bounds__(kSeqThreads) seq_mean_kernel(const double *__restrict__ loss_seq, int B,
                                                               double *__restrict__ loss) {
    __shared__ double red[kSeqThreads / 32];
    double v = 0.0;
    for (int b = threadIdx.x; b < B; b += kSeqThreads) v += loss_seq[b];
    const double sum = block_sum(v, red);
    if (threadIdx.x == 0) *loss = sum / (double)B;
}

}  // namespace

cudaError_t launch_seq_balance(const int32_t *tile_counts, const float *tile_psum, int T, int Nr, int K, int seq_len,
                               float alpha, double *loss_seq, double *loss, cudaStream_t stream) {
    const int B = T / seq_len;
    const double S = (double)seq_len;
    const double scale = (double)alpha * (double)Nr / ((double)K * S * S);
    seq_loss_kernel<<<B, kSeqThreads, 0, stream>>>(tile_counts, tile_psum, Nr, seq_len / kTileTokens, scale, loss_seq);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    seq_mean_kernel<<<1, kSeqThreads, 0, stream>>>(loss_seq, B, loss);
    return cudaGetLastError();
}

}  // namespace ebl
