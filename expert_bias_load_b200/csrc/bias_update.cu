// bias_update.cu -- the once-per-step expert-bias updates and MaxVio.
//
// SMEBU ("SMEBU Load Balancing", "How it works", eqs. (23)-(28); constants in
// "Arcee Trinity Large Technical Report" section 2.3):
//   nbar = sum n / N_r;  v = (nbar - n)/nbar;  db = lambda * tanh(kappa v)
//   db -= mean(db);  m = beta m + (1 - beta) db;  b += m
// Linear ablation (same sources): db = lambda v.
// Sign update of the smaller models (same note, eqs. (20)-(22)):
//   b' = b + gamma sign(nbar - n);  b = b' - mean(b')
// MaxVio ("Arcee Halts 400B Blackwell Model Collapse With Dynamic Router
// Biases", "The MaxVio Metric and the Day-4 Crisis"): max n / min n.
//
// One CTA per MoE layer, one thread per expert.  All arithmetic is fp64 with
// explicitly rounded operations (no contraction into FMA), and the mean is
// summed by one thread in expert order, so the result does not depend on the
// launch shape; the fp32 state is read widened and stored rounded to nearest.

#include "launch.h"
#include "ptx.cuh"

namespace ebl {
namespace {

constexpr int kThreads = kMaxExperts;  // one thread per expert

struct LoadStats {
    long long total;
    int max_n, min_n;
};

// Block reductions of the loads: sum, max, min (threads >= Nr contribute the
// identity).  Every thread receives the result.
__device__ LoadStats load_stats(int n, bool active) {
    __shared__ long long s_sum[kThreads / 32];
    __shared__ int s_max[kThreads / 32], s_min[kThreads / 32];
    __shared__ LoadStats out;
    long long sum = active ? (long long)n : 0;
    int mx = active ? n : INT_MIN;
    int mn = active ? n : INT_MAX;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        sum += __shfl_xor_sync(0xffffffffu, sum, off);
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        s_sum[warp] = sum;
        s_max[warp] = mx;
        s_min[warp] = mn;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        long long a = 0;
        int b = INT_MIN, c = INT_MAX;
        for (int w = 0; w < kThreads / 32; ++w) {
            a += s_sum[w];
            b = max(b, s_max[w]);
            c = min(c, s_min[w]);
        }
        out.total = a;
        out.max_n = b;
        out.min_n = c;
    }
    __syncthreads();
    return out;
}

__device__ __forceinline__ float maxvio_of(int mx, int mn) {
    if (mn == 0) return __int_as_float(0x7f800000);  // +inf: an expert got no load
    return __double2float_rn(__ddiv_rn((double)mx, (double)mn));
}

// mean of v[0..Nr) in fp64, summed in index order by one thread.
__device__ double ordered_mean(const double *v, int Nr) {
    __shared__ double s_mean;
    __syncthreads();
    if (threadIdx.x == 0) {
        double s = 0.0;
        for (int i = 0; i < Nr; ++i) s = __dadd_rn(s, v[i]);
        s_mean = __ddiv_rn(s, (double)Nr);
    }
    __syncthreads();
    return s_mean;
}

__global__ void __launch_bounds__(kThreads) smebu_kernel(int32_t *__restrict__ counts, float *__restrict__ bias,
                                                         float *__restrict__ momentum, int Nr, float lambda_f,
                                                         float beta_f, float kappa_f, int linear, int reset_counts,
                                                         float *__restrict__ maxvio_out,
                                                         int32_t *__restrict__ status) {
    __shared__ double db_s[kThreads];
    const size_t layer = blockIdx.x;
    counts += layer * Nr;
    bias += layer * Nr;
    momentum += layer * Nr;
    const int i = threadIdx.x;
    const bool active = i < Nr;
    const int n = active ? counts[i] : 0;
    const LoadStats st = load_stats(n, active);
    if (active && reset_counts) counts[i] = 0;
    if (i == 0 && maxvio_out) maxvio_out[layer] = maxvio_of(st.max_n, st.min_n);
    if (st.total <= 0) {
        if (i == 0) atomicOr(status, kStEmptyLoad);
        return;
    }
    const double lambda = lambda_f, beta = beta_f, kappa = kappa_f;
    const double nbar = __ddiv_rn((double)st.total, (double)Nr);
    double db = 0.0;
    if (active) {
        const double v = __ddiv_rn(__dsub_rn(nbar, (double)n), nbar);  // eq. (23)
        db = linear ? __dmul_rn(lambda, v)                              // linear ablation
                    : __dmul_rn(lambda, tanh(__dmul_rn(kappa, v)));     // eqs. (24)-(25)
        db_s[i] = db;
    }
    const double mean = ordered_mean(db_s, Nr);  // eq. (26)
    if (active) {
        const double dc = __dsub_rn(db, mean);
        const double m = __dadd_rn(__dmul_rn(beta, (double)momentum[i]), __dmul_rn(__dsub_rn(1.0, beta), dc));
        const double b = __dadd_rn((double)bias[i], m);  // eqs. (27)-(28)
        momentum[i] = __double2float_rn(m);
        bias[i] = __double2float_rn(b);
    }
}

__global__ void __launch_bounds__(kThreads) sign_update_kernel(int32_t *__restrict__ counts,
                                                               float *__restrict__ bias, int Nr, float gamma_f,
                                                               int reset_counts, float *__restrict__ maxvio_out,
                                                               int32_t *__restrict__ status) {
    __shared__ double bp_s[kThreads];
    const int i = threadIdx.x;
    const bool active = i < Nr;
    const int n = active ? counts[i] : 0;
    const LoadStats st = load_stats(n, active);
    if (active && reset_counts) counts[i] = 0;
    if (i == 0 && maxvio_out) *maxvio_out = maxvio_of(st.max_n, st.min_n);
    if (st.total <= 0) {
        if (i == 0) atomicOr(status, kStEmptyLoad);
        return;
    }
    const double gamma = gamma_f;
    const double nbar = __ddiv_rn((double)st.total, (double)Nr);
    double bp = 0.0;
    if (active) {
        const double diff = __dsub_rn(nbar, (double)n);
        const double sgn = diff > 0.0 ? 1.0 : (diff < 0.0 ? -1.0 : 0.0);
        bp = __dadd_rn((double)bias[i], __dmul_rn(gamma, sgn));  // eqs. (20)-(21)
        bp_s[i] = bp;
    }
    const double mean = ordered_mean(bp_s, Nr);  // eq. (22): re-centre after the add
    if (active) bias[i] = __double2float_rn(__dsub_rn(bp, mean));
}

}  // namespace

cudaError_t launch_smebu(int32_t *counts, float *bias, float *momentum, int L, int Nr, float lambda, float beta,
                         float kappa, int linear, int reset_counts, float *maxvio_out, int32_t *status,
                         cudaStream_t stream) {
    smebu_kernel<<<L, kThreads, 0, stream>>>(counts, bias, momentum, Nr, lambda, beta, kappa, linear, reset_counts,
                                             maxvio_out, status);
    return cudaGetLastError();
}

cudaError_t launch_sign_update(int32_t *counts, float *bias, int Nr, float gamma, int reset_counts,
                               float *maxvio_out, int32_t *status, cudaStream_t stream) {
    sign_update_kernel<<<1, kThreads, 0, stream>>>(counts, bias, Nr, gamma, reset_counts, maxvio_out, status);
    return cudaGetLastError();
}

}  // namespace ebl
