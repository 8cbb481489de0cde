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
// Layout: one thread per token row (a CTA of 128 threads takes a 128-token
// tile; persistent grid).  A warp's 32 rows are read together, 32 experts at a
// time: each load instruction fetches 128 contiguous bytes of one row, and the
// 32 x 32 block is transposed through padded shared memory so that every thread
// then walks its own row in increasing expert index.  Each thread keeps a
// running Top-K in registers; visiting experts in increasing index lets a
// strict comparison keep the lower index first on equal keys.  A shared-memory
// histogram is flushed per tile (tile_counts) and per CTA (counts).
//
// The fp64 sigmoid is only evaluated where it can matter.  A first pass ranks
// the experts with an fp32 sigmoid whose distance to the fp64-rounded value
// is bounded (kSigmaErr); its K-th key tau bounds the exact K-th key within
// kSigmaErr plus the rounding of the key add.  Only experts whose approximate
// key is within twice that margin of tau can be in the exact Top-K, so the
// second pass computes the exact score of those candidates alone (usually K or
// K+1 of them) and selects among them: the same result as evaluating every
// expert in fp64.

#include "launch.h"
#include "ptx.cuh"
#include "topk.cuh"

namespace ebl {
namespace {

constexpr int kThreads = kTileTokens;  // one thread per row of a tile

__device__ __forceinline__ float sigmoid_rounded_once(float x) {
    // fp64 evaluation, one rounding to fp32 at the end
    const double e = exp(-(double)x);
    return __double2float_rn(__ddiv_rn(1.0, __dadd_rn(1.0, e)));
}

// fp32 sigmoid from the fast intrinsics: __expf (at most 2 + 1.173|x| ulp off)
// and __fdividef (at most 2 ulp).  Its distance to sigmoid_rounded_once() is
// below 4e-7 for every finite x (the exp error is damped by s(1-s), which
// decays faster than the error grows); kSigmaErr leaves a 10x margin.
__device__ __forceinline__ float sigmoid_fast(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }
constexpr float kSigmaErr = 4.0e-6f;

constexpr int kWarpsPerCta = kThreads / 32;
constexpr int kMaxCand = 8;  // candidates a lane buffers before scoring them exactly

// The K largest values seen so far (with repeats), sorted descending; one
// fmax/fmin pair per slot and value, no branches.  NaN values are dropped.
template <int K>
struct TopValues {
    float v[K];
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int k = 0; k < K; ++k) v[k] = -INFINITY;
    }
    __device__ __forceinline__ void push(float x) {
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const float hi = fmaxf(v[k], x);
            x = fminf(v[k], x);
            v[k] = hi;
        }
    }
};

// The warp's rows row0 .. row0+31 (lane l owns row0 + l): calls f(c, x) for
// each expert c of the lane's row in increasing c, x its logit.  Rows at or
// past T read nothing (x = 0).
template <class F>
__device__ __forceinline__ void warp_rows_each_logit(const float *__restrict__ logits, int row0, int T, int Nr,
                                                     float (*blk)[33], int lane, F &&f) {
    for (int c0 = 0; c0 < Nr; c0 += 32) {
        const int c = c0 + lane;
#pragma unroll 8
        for (int r = 0; r < 32; ++r) {
            const int row = row0 + r;
            blk[r][lane] = (row < T && c < Nr) ? __ldg(logits + (size_t)row * Nr + c) : 0.0f;
        }
        __syncwarp();
        const int cn = min(32, Nr - c0);
        for (int j = 0; j < cn; ++j) f(c0 + j, blk[lane][j]);
        __syncwarp();
    }
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
    __shared__ float blocks[kWarpsPerCta][32][33];  // per-warp transpose buffer (padded: no bank conflicts)
    __shared__ float cand_x[kWarpsPerCta][kMaxCand][32];  // per-lane candidates of pass 2: logit, expert
    __shared__ int cand_c[kWarpsPerCta][kMaxCand][32];

    for (int i = threadIdx.x; i < Nr; i += kThreads) {
        bias_s[i] = bias[i];
        hist_total[i] = 0;
        hist_tile[i] = 0;
    }
    __syncthreads();

    const bool want_tiles = tile_counts != nullptr;
    int *hist = want_tiles ? hist_tile : hist_total;
    const int num_tiles = (T + kTileTokens - 1) / kTileTokens;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    float(*blk)[33] = blocks[warp];

    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        const int row0 = tile * kTileTokens + warp * 32;
        const int row = row0 + lane;
        if (row0 < T) {  // warp-uniform: the whole warp joins the block loads
            // pass 1: approximate keys, their K-th largest
            TopValues<K> approx;
            approx.init();
            warp_rows_each_logit(logits, row0, T, Nr, blk, lane, [&](int c, float xv) {
                approx.push(__fadd_rn(sigmoid_fast(xv), bias_s[c]));
            });
            const float tau = approx.v[K - 1];
            // |approximate key - exact key| <= kSigmaErr + one rounding of each add
            const float lim = tau - 2.0f * (kSigmaErr + 2.384185791015625e-7f * fabsf(tau));
            // pass 2: exact keys of the candidates only.  Candidates are buffered
            // per lane (in increasing expert index) and scored after the scan,
            // so the fp64 work runs in a short loop instead of under a branch
            // that some lane of the warp takes at most experts.
            RowTopK<K> tk;
            tk.init();
            int nc = 0;
            auto flush = [&]() {
                for (int q = 0; q < nc; ++q) {
                    const int c = cand_c[warp][q][lane];
                    const float s = sigmoid_rounded_once(cand_x[warp][q][lane]);
                    tk.push(__fadd_rn(s, bias_s[c]), s, c);
                }
                nc = 0;
            };
            warp_rows_each_logit(logits, row0, T, Nr, blk, lane, [&](int c, float xv) {
                if (__fadd_rn(sigmoid_fast(xv), bias_s[c]) >= lim) {
                    if (nc == kMaxCand) flush();  // many near-equal keys: score what we have first
                    cand_x[warp][nc][lane] = xv;
                    cand_c[warp][nc][lane] = c;
                    ++nc;
                }
            });
            flush();
            if (row < T) {
                double sum = 0.0;
#pragma unroll
                for (int k = 0; k < K; ++k) sum = __dadd_rn(sum, (double)tk.score[k]);
                int32_t *oi = topk_idx + (size_t)row * K;
                float *og = gates + (size_t)row * K;
#pragma unroll
                for (int k = 0; k < K; ++k) {
                    oi[k] = tk.idx[k];
                    og[k] = __double2float_rn(__ddiv_rn((double)tk.score[k], sum));
                    if ((unsigned)tk.idx[k] < (unsigned)Nr) atomicAdd(&hist[tk.idx[k]], 1);
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
    int grid = num_sms * 16;
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
