// router_logits.cu -- the router's selection stage fed with precomputed fp32
// logits: the bit-exact mode of the library.
//
// Per token: s = (float)(1/(1+exp(-(double)x))), key = s + b (one fp32 add),
// Top-K of key with equal keys going to the lower expert index, gates
// g_k = (float)((double)s_k / sum of (double)s over the selected slots in slot
// order), per-expert counts and per-128-token-tile counts.
// Sources: "Arcee Trinity Large Technical Report" section 2.3; "SMEBU Load
// Balancing" eq. (17).
//
// Layout: one warp per token row; lane l owns experts l, l+32, ... (so each
// load instruction reads 128 contiguous bytes of the row), keeps a running
// Top-K of its own experts, and the warp merges the 32 lists with K rounds of
// a shuffle arg-max under the order (key desc, index asc).  One CTA of 8 warps
// handles a 128-token tile at a time (persistent grid), with a shared-memory
// histogram flushed per tile (tile_counts) and per CTA (counts).

#include "launch.h"
#include "ptx.cuh"
#include "topk.cuh"

namespace ebl {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ float sigmoid_rounded_once(float x) {
    // fp64 evaluation, one rounding to fp32 at the end
    const double e = exp(-(double)x);
    return __double2float_rn(__ddiv_rn(1.0, __dadd_rn(1.0, e)));
}

template <int K>
__global__ void __launch_bounds__(kThreads) router_logits_kernel(const float *__restrict__ logits,
                                                                 const float *__restrict__ bias, int T, int Nr,
                                                                 int32_t *__restrict__ topk_idx,
                                                                 float *__restrict__ gates,
                                                                 int32_t *__restrict__ counts,
                                                                 int32_t *__restrict__ tile_counts) {
    __shared__ float bias_s[kMaxExperts];
    __shared__ int hist_total[kMaxExperts];
    __shared__ int hist_tile[kMaxExperts];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < Nr; i += kThreads) {
        bias_s[i] = bias[i];
        hist_total[i] = 0;
        hist_tile[i] = 0;
    }
    __syncthreads();

    const bool want_tiles = tile_counts != nullptr;
    int *hist = want_tiles ? hist_tile : hist_total;
    const int num_tiles = (T + kTileTokens - 1) / kTileTokens;

    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        for (int r = warp; r < kTileTokens; r += kWarps) {
            const int row = tile * kTileTokens + r;
            if (row >= T) break;
            const float *x = logits + (size_t)row * Nr;

            RowTopK<K> mine;
            mine.init();
            for (int c = lane; c < Nr; c += 32) {
                const float s = sigmoid_rounded_once(__ldcs(x + c));
                mine.push(__fadd_rn(s, bias_s[c]), s, c);
            }

            int sel_i[K];
            float sel_s[K];
#pragma unroll
            for (int k = 0; k < K; ++k) {
                float bk = mine.key[0];
                int bi = mine.idx[0];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const float ok = __shfl_xor_sync(0xffffffffu, bk, off);
                    const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
                    if (ok > bk || (ok == bk && oi < bi)) {
                        bk = ok;
                        bi = oi;
                    }
                }
                const int owner = bi & 31;
                sel_i[k] = bi;
                sel_s[k] = __shfl_sync(0xffffffffu, mine.score[0], owner);
                if (lane == owner) {  // pop the head of the owner's list
#pragma unroll
                    for (int p = 0; p + 1 < K; ++p) {
                        mine.key[p] = mine.key[p + 1];
                        mine.score[p] = mine.score[p + 1];
                        mine.idx[p] = mine.idx[p + 1];
                    }
                    mine.key[K - 1] = -INFINITY;
                    mine.idx[K - 1] = 0x7fffffff;
                }
            }

            if (lane == 0) {
                double sum = 0.0;
#pragma unroll
                for (int k = 0; k < K; ++k) sum = __dadd_rn(sum, (double)sel_s[k]);
                int32_t *oi = topk_idx + (size_t)row * K;
                float *og = gates + (size_t)row * K;
#pragma unroll
                for (int k = 0; k < K; ++k) {
                    oi[k] = sel_i[k];
                    og[k] = __double2float_rn(__ddiv_rn((double)sel_s[k], sum));
                    if ((unsigned)sel_i[k] < (unsigned)Nr) atomicAdd(&hist[sel_i[k]], 1);
                }
            }
        }
        if (want_tiles) {
            __syncthreads();
            for (int e = threadIdx.x; e < Nr; e += kThreads) {
                const int v = hist_tile[e];
                tile_counts[(size_t)tile * Nr + e] = v;
                hist_total[e] += v;
                hist_tile[e] = 0;
            }
            __syncthreads();
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < Nr; e += kThreads)
        if (hist_total[e] != 0) atomicAdd(&counts[e], hist_total[e]);
}

}  // namespace

cudaError_t launch_router_logits(const float *logits, const float *bias, int T, int Nr, int K, int32_t *topk_idx,
                                 float *gates, int32_t *counts, int32_t *tile_counts, int num_sms,
                                 cudaStream_t stream) {
    const int num_tiles = (T + kTileTokens - 1) / kTileTokens;
    int grid = num_sms * 8;
    if (grid > num_tiles) grid = num_tiles;
    switch (K) {
#define EBL_CASE(KK)                                                                                    \
    case KK:                                                                                            \
        router_logits_kernel<KK><<<grid, kThreads, 0, stream>>>(logits, bias, T, Nr, topk_idx, gates, \
                                                                counts, tile_counts);                  \
        break;
        EBL_CASE(1)
        EBL_CASE(2)
        EBL_CASE(3)
        EBL_CASE(4)
        EBL_CASE(5)
        EBL_CASE(6)
        EBL_CASE(7)
        EBL_CASE(8)
#undef EBL_CASE
        default:
            return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace ebl
