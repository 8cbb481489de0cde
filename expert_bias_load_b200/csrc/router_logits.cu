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
// The fp64 sigmoid is only evaluated where it can matter.  An approximate key
// with a bounded distance to the exact one ranks all experts; the K-th largest
// approximate key tau bounds the exact K-th key, and only experts whose
// approximate key is within twice that distance of tau can be in the exact
// Top-K.  Those candidates (K to K+2 per token on most rows) are scored exactly and
// the exact Top-K is taken among them: the same result as scoring every expert
// in fp64.
//
// Two kernels.  The vector kernel (N_r % 4 == 0, 16-byte aligned logits, the
// usual case) gives each token row to 8 lanes: every load instruction fetches
// 128 contiguous bytes of each of 4 rows, a lane's 4*NV logits and their keys
// stay in registers, tau comes from a butterfly over the 8 lanes, and the
// candidates (column and logit) are compacted per row in shared memory, scored
// by the row's 8 lanes and ranked in parallel while the next rows load.  The
// logits are read from HBM exactly once.  With the balance option the same
// pass also writes the per-tile statistics of the sequence-wise balance loss.
// The row kernel (any N_r, 4-byte alignment) gives each row to one thread and
// reads the logits twice.

#include <cfloat>
#include <cstdint>
#include <mutex>

#include "launch.h"
#include "ptx.cuh"
#include "scores.cuh"
#include "topk.cuh"

namespace ebl {
namespace {

constexpr int kThreads = kTileTokens;  // one thread per row of a tile

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
    // Keep the K largest of this lane's list and lane (lane ^ m)'s (K a power
    // of two): the elementwise max of one list and the other reversed is a
    // bitonic sequence holding the K largest of both, which a half-cleaner
    // cascade sorts.
    __device__ __forceinline__ void merge_xor(int m) {
        static_assert((K & (K - 1)) == 0, "bitonic merge needs a power-of-two list");
        float o[K];
#pragma unroll
        for (int k = 0; k < K; ++k) o[k] = __shfl_xor_sync(0xffffffffu, v[k], m);
#pragma unroll
        for (int k = 0; k < K; ++k) v[k] = fmaxf(v[k], o[K - 1 - k]);
#pragma unroll
        for (int h = K / 2; h > 0; h >>= 1) {
#pragma unroll
            for (int i = 0; i < K; ++i) {
                if ((i & h) == 0) {
                    const float a = v[i], b = v[i + h];
                    v[i] = fmaxf(a, b);
                    v[i + h] = fminf(a, b);
                }
            }
        }
    }
    // The Kth largest (1-based) of this lane's list and lane (lane ^ m)'s, both
    // sorted descending, Kth <= P: taking i values from one list and Kth - i
    // from the other, the Kth largest of the union is the largest over i of
    // the smaller of the two lists' last values taken.  Both lanes get it.
    template <int Kth>
    __device__ __forceinline__ float kth_of_merge_xor(int m) const {
        static_assert(Kth >= 1 && Kth <= K, "Kth within the list");
        float o[Kth];
#pragma unroll
        for (int k = 0; k < Kth; ++k) o[k] = __shfl_xor_sync(0xffffffffu, v[k], m);
        float r = fmaxf(v[Kth - 1], o[Kth - 1]);
#pragma unroll
        for (int i = 1; i < Kth; ++i) r = fmaxf(r, fminf(v[i - 1], o[Kth - 1 - i]));
        return r;
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
                                                                 int32_t *__restrict__ tile_counts,
                                                                 int32_t *__restrict__ status) {
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
                    if ((unsigned)tk.idx[k] < (unsigned)Nr)
                        atomicAdd(&hist[tk.idx[k]], 1);
                    else
                        atomicOr(status, kStNonfinite);  // only a NaN or -inf key leaves a slot unfilled
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


// ---------------------------------------------------------------------------
// Vector kernel: 8 lanes per token row, one HBM read of the logits.
// ---------------------------------------------------------------------------

constexpr int kLanesPerRow = 8;
constexpr int kRowsPerGroup = 32 / kLanesPerRow;         // rows a warp takes at once
constexpr int kGroupsPerWarp = 32 / kRowsPerGroup;       // row groups of a warp per tile
constexpr int kWin = 24;                                 // candidates of a row scored per round
constexpr int kWinPad = kWin + 1;                        // odd stride: rows of a group hit different banks

__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// The largest of three values in one three-input max instruction (the keys
// it compares are finite or -inf; inputs are assumed finite).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float y;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
    return y;
}

// Approximate key from hb = fl(0.5 + b): 0.5 tanh(x/2) + 0.5 + b is
// sigmoid(x) + b.  Distance to the exact key fl(fl(sigmoid(x)) + b):
//   0.5 |tanh.approx(x/2) - tanh(x/2)|   about 2^-12 (the documented relative
//                                        error of tanh.approx.f32 is about
//                                        2^-11; ebl_selftest_score_error
//                                        measures the actual one)
//   fl(sigmoid(x)) - sigmoid(x)          <= 2^-25
//   roundings of hb, the fma, the add    <= 2^-24 (|hb| + |key_a| + |key_e|)
//                                        <= 2^-24 (3 |key_e| + 1.5) + O(2^-36)
// (|b| <= |key_e| + 1), so |key_a - key_e| <= kKeyErr + 2^-22 |key_e| with the
// constant part given an 8x margin.
constexpr float kKeyErr = 0x1p-9f;
__device__ __forceinline__ float key_approx(float x, float hb) { return fmaf(0.5f, tanh_approx(0.5f * x), hb); }

// Lower limit on the approximate key of every member of the exact Top-K, from
// tau' <= the K-th largest approximate key.  With E(y) = kKeyErr + 2^-22 |y|:
// the K-th exact key tau_e satisfies tau' <= tau_e + E(tau_e), so
// tau_e >= tau' - kKeyErr - 2^-21 |tau' - kKeyErr|; a member i has
// key_a >= key_e - E(key_e) >= tau_e - E(tau_e).  Together (and with the
// rounding of this fp32 expression) key_a >= tau' - 2 kKeyErr - 2^-19 |tau'|.
// An empty list (tau' = -inf) admits every finite key; padding keys (-inf)
// never pass.
__device__ __forceinline__ float candidate_limit(float tau, float key_err = kKeyErr) {
    return fmaxf(tau - (2.0f * key_err + 0x1p-19f * fabsf(tau)), -FLT_MAX);
}

// An unsigned value that orders like the float f (-inf lowest; f not NaN,
// and +0 for zero, which every key here is: s >= +0 and +0 + -0 = +0).
__device__ __forceinline__ uint32_t order_bits(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ void cp_async_16(void *dst, const void *src, bool pred) {
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(dst));
    const int n = pred ? 16 : 0;  // 0: the 16 bytes are zero-filled and nothing is read
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Lane j of a row owns the row's 4*NV consecutive columns [4*NV*j, 4*NV*(j+1)),
// so the row's candidates come out of a prefix over its lanes already in
// expert order.  In shared memory (the logits stage and the bias table) each
// lane's columns are followed by 16 unused bytes: a lane reads its float4 m at
// 16 (NV + 1) j + 16 m bytes, and NV + 1 odd puts the 8 lanes of a row on 8
// different 16-byte bank groups.  Column c sits at float offset pad_col(c).
template <int NV>
__device__ __forceinline__ int pad_col(int c) {
    return c + 4 * (c / (4 * NV));
}
template <int NV>
__host__ __device__ constexpr int padded_row() {
    return 32 * (NV + 1);  // floats of one row (or the bias table) in shared memory
}

// Dynamic shared memory of the vector kernel: one logits stage per warp (the
// warp's 4 rows of the current item).  The stage is refilled as soon as each
// candidate's logit has been copied out of it, and the candidate stage runs
// while the next item loads; a single stage keeps 7 CTAs (28 warps) resident
// per SM, which measured faster than two stages at 5 CTAs.
template <int NV>
constexpr size_t vec_ring_bytes() {
    return sizeof(float) * kWarpsPerCta * kRowsPerGroup * padded_row<NV>();
}

// Per-warp candidate buffers of the vector kernel (the fast path lists each
// candidate's column in c and its logit in key).  With the balance option a
// warp's column sums (kMaxExperts floats) reuse this space at the end of each
// tile, after the warp's last candidate stage of the tile.
struct WarpCand {
    int c[kRowsPerGroup][kWinPad];  // a round's candidates of each row
    float key[kRowsPerGroup][kWinPad];
    float s[kRowsPerGroup][kWinPad];
};
static_assert(sizeof(WarpCand) >= (kMaxExperts + 32) * sizeof(float), "column sums fit the candidate buffers");

// BAL (the balance option): the approximate key is sigmoid_fast(x) + b instead
// of the tanh form, and the same fast scores give the per-tile statistics of
// the sequence-wise balance loss, tile_psum[j, i] = sum over the tile's rows t
// of s_t,i / sum_l s_t,l.  Each lane keeps the fp32 sums of its 4*NV columns
// over the rows it sees; at the end of a tile the warp folds its four row
// lanes per column with two shuffles and the CTA adds its four warps in
// order, so the sums do not depend on scheduling.
template <int K, int NV, bool FULL, bool BAL>
__device__ __forceinline__ void logits_vec_body(const float *__restrict__ logits, const float *__restrict__ bias,
                                                int T, int Nr, int32_t *__restrict__ topk_idx,
                                                float *__restrict__ gates, int32_t *__restrict__ counts,
                                                int32_t *__restrict__ tile_counts, float *__restrict__ tile_psum,
                                                int32_t *__restrict__ status) {
    // lane-local lists of the approximate pass hold P >= K values (P a power of two)
    constexpr int P = K <= 1 ? 1 : (K <= 2 ? 2 : (K <= 4 ? 4 : 8));
    constexpr int kRow = 32 * NV;  // columns per row in the ring (N_r rounded up, zero-filled)
    constexpr int kRowPad = padded_row<NV>();
    constexpr int kLaneCols = 4 * NV;  // columns a lane owns
    // FULL: N_r == kRow, so every column a lane copies exists (no per-column test)
    static_assert(NV % 2 == 0 && kRow <= kMaxExperts, "a lane holds NV float4 of a row, in pairs");
    // distance of the approximate key to the exact one (see key_approx, sigmoid_fast)
    constexpr float kErr = BAL ? kSigmaErr : kKeyErr;
    extern __shared__ __align__(16) float ring_s[];  // [warp][row of group][kRowPad]
    // tanh form: fl(0.5 + b); balance option: b.  -inf past N_r either way.
    // Padded like a row of the ring.
    __shared__ __align__(16) float hb_s[kMaxExperts + 32];
    __shared__ int hist_total[kMaxExperts];
    __shared__ int hist_tile[kMaxExperts];
    __shared__ __align__(16) WarpCand cand[kWarpsPerCta];
    __shared__ float sel_key[kWarpsPerCta][kRowsPerGroup][2 * K];  // [0,K): the Top-K so far; [K,2K): a later round's
    __shared__ float sel_s[kWarpsPerCta][kRowsPerGroup][2 * K];
    __shared__ int sel_c[kWarpsPerCta][kRowsPerGroup][2 * K];

    for (int i = threadIdx.x; i < kMaxExperts; i += kThreads) {
        hist_total[i] = 0;
        hist_tile[i] = 0;
    }
    for (int i = threadIdx.x; i < kRow; i += kThreads) {
        const bool in = i < Nr;
        const float b = in ? bias[i] : 0.0f;
        hb_s[pad_col<NV>(i)] = in ? (BAL ? b : __fadd_rn(0.5f, b)) : -INFINITY;
    }
    for (int i = threadIdx.x; i < kWarpsPerCta * kRowsPerGroup * 2 * K; i += kThreads) {
        (&sel_key[0][0][0])[i] = -INFINITY;
        (&sel_s[0][0][0])[i] = 0.0f;
        (&sel_c[0][0][0])[i] = 0;
    }
    __syncthreads();

    const bool want_tiles = tile_counts != nullptr;
    int *hist = want_tiles ? hist_tile : hist_total;
    const int num_tiles = (T + kTileTokens - 1) / kTileTokens;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int r = lane >> 3;  // row of the group this lane works on
    const int j = lane & 7;   // lane within the row: it owns columns [4*NV*j, 4*NV*(j+1))
    float *ring = ring_s + (size_t)warp * kRowsPerGroup * kRowPad;
    const float *hbl = hb_s + (kLaneCols + 4) * j;  // this lane's bias values
    int *cc = cand[warp].c[r];
    float *ck = cand[warp].key[r];
    float *cs = cand[warp].s[r];
    float *colsum = reinterpret_cast<float *>(&cand[warp]);  // balance option: the warp's column sums
    float *sk = sel_key[warp][r];
    float *ss = sel_s[warp][r];
    int *sc = sel_c[warp][r];

    // Work item i of this warp: row group i % 8 of tile blockIdx.x + (i / 8) * gridDim.x.
    // Its 4 rows go to the warp's stage; lane j of a row copies float4
    // columns 8m + j (into the owner lane's padded slots), so each copy
    // instruction covers 128 contiguous bytes of each of the 4 rows.  Rows
    // past T are zero-filled without a read.  (Whole
    // tiles per CTA also stream 128 KB of consecutive rows at a time, which
    // measured 2% faster than dealing row groups to all warps in turn.)
    auto item_row = [&](int item) -> int64_t {
        const int64_t tile = (int64_t)blockIdx.x + (int64_t)(item >> 3) * gridDim.x;
        return tile * kTileTokens + warp * 32 + (item & 7) * kRowsPerGroup + r;
    };
    auto issue = [&](int item, int64_t row) {
        const bool rin = row < T;
        const float *src = logits + (rin ? row : 0) * (int64_t)Nr;
        float *dst = ring + r * kRowPad;
#pragma unroll
        for (int m = 0; m < NV; ++m) {
            const int c = 4 * (8 * m + j);
            const bool ok = FULL ? rin : (rin && c < Nr);
            cp_async_16(dst + pad_col<NV>(c), src + (ok ? c : 0), ok);
        }
        cp_async_commit();
    };
    // the row of item + 1 from the row of item (the same tile, or the next tile of this CTA)
    const int64_t tile_jump = (int64_t)gridDim.x * kTileTokens - (kGroupsPerWarp - 1) * kRowsPerGroup;
    auto next_row = [&](int64_t row, int item) { return ((item + 1) & 7) ? row + kRowsPerGroup : row + tile_jump; };

    const int items = num_tiles > (int)blockIdx.x
                          ? ((num_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1) * kGroupsPerWarp
                          : 0;
    float psum[BAL ? NV : 1][4];  // balance option: this lane's column sums over the tile's rows it sees
#pragma unroll
    for (int m = 0; m < (BAL ? NV : 1); ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) psum[m][e] = 0.0f;
    int64_t ahead = item_row(0);  // the row of the most recently issued item
    issue(0, ahead);
    for (int item = 0; item < items; ++item) {
        const int64_t row = ahead;
        ahead = next_row(ahead, item);
        cp_async_wait<0>();
        __syncwarp();
        // this lane's columns of its row; the next item is issued once they are read
        const float *xr = ring + r * kRowPad + (kLaneCols + 4) * j;

        // approximate keys of this lane's 4*NV experts
        float kv[NV][4];
        if constexpr (BAL) {
            // fast scores; their row total over the row's 8 lanes; the lane's
            // column sums gain s / total (0 for a row past T); then the keys
            float rs = 0.0f;
#pragma unroll
            for (int m = 0; m < NV; ++m) {
                const float4 x = *reinterpret_cast<const float4 *>(xr + 4 * m);
                kv[m][0] = sigmoid_fast(x.x);
                kv[m][1] = sigmoid_fast(x.y);
                kv[m][2] = sigmoid_fast(x.z);
                kv[m][3] = sigmoid_fast(x.w);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if constexpr (!FULL)  // padding columns (zero-filled, s = 1/2) add nothing
                        if (kLaneCols * j + 4 * m + e >= Nr) kv[m][e] = 0.0f;
                    rs += kv[m][e];
                }
            }
            rs += __shfl_xor_sync(0xffffffffu, rs, 1);
            rs += __shfl_xor_sync(0xffffffffu, rs, 2);
            rs += __shfl_xor_sync(0xffffffffu, rs, 4);
            const float inv = (row < T && rs > 0.0f) ? __frcp_rn(rs) : 0.0f;
#pragma unroll
            for (int m = 0; m < NV; ++m) {
                const float4 h = *reinterpret_cast<const float4 *>(hbl + 4 * m);
                const float hv[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    psum[m][e] = fmaf(kv[m][e], inv, psum[m][e]);
                    kv[m][e] = __fadd_rn(kv[m][e], hv[e]);  // -inf past N_r
                }
            }
        } else {
            // key_approx on pairs of columns through the packed two-lane fp32
            // instructions (each half rounds like the scalar operation)
            const float2 half = make_float2(0.5f, 0.5f);
#pragma unroll
            for (int m = 0; m < NV; ++m) {
                const float4 x = *reinterpret_cast<const float4 *>(xr + 4 * m);
                const float4 h = *reinterpret_cast<const float4 *>(hbl + 4 * m);
                const float2 xa = __fmul2_rn(half, make_float2(x.x, x.y));
                const float2 xb = __fmul2_rn(half, make_float2(x.z, x.w));
                const float2 ya =
                    __ffma2_rn(half, make_float2(tanh_approx(xa.x), tanh_approx(xa.y)), make_float2(h.x, h.y));
                const float2 yb =
                    __ffma2_rn(half, make_float2(tanh_approx(xb.x), tanh_approx(xb.y)), make_float2(h.z, h.w));
                kv[m][0] = ya.x;
                kv[m][1] = ya.y;
                kv[m][2] = yb.x;
                kv[m][3] = yb.y;
            }
        }
        // tau': the K-th largest of the maxima of groups of 8 keys (each
        // maximum is a key of its own, so tau' is at most the K-th key)
        constexpr int G = NV / 2;  // groups per lane
        float gm[G];
#pragma unroll
        for (int q = 0; q < G; ++q) {
            const float a = fmax3(kv[2 * q][0], kv[2 * q][1], kv[2 * q][2]);
            const float b = fmax3(kv[2 * q][3], kv[2 * q + 1][0], kv[2 * q + 1][1]);
            gm[q] = fmaxf(b, fmax3(kv[2 * q + 1][2], kv[2 * q + 1][3], a));
        }
        TopValues<P> top;
        top.init();
        if constexpr (G <= P) {
            // all of the lane's group maxima fit the list: sort them (network for 1, 2 or 4)
            static_assert(G == 1 || G == 2 || G == 4, "groups per lane");
            auto ce = [](float &hi, float &lo) {
                const float a = hi, b = lo;
                hi = fmaxf(a, b);
                lo = fminf(a, b);
            };
            if constexpr (G == 2) ce(gm[0], gm[1]);
            if constexpr (G == 4 && P == 4) {
                ce(gm[0], gm[1]);
                ce(gm[2], gm[3]);
                const float hi = fmaxf(gm[0], gm[2]);
                gm[1] = fmaxf(fminf(gm[0], gm[2]), fmaxf(gm[1], gm[3]));
                gm[0] = hi;
            } else if constexpr (G == 4) {
                ce(gm[0], gm[1]);
                ce(gm[2], gm[3]);
                ce(gm[0], gm[2]);
                ce(gm[1], gm[3]);
                ce(gm[1], gm[2]);
            }
            if constexpr (G == 4 && P == 4) {
                // K = 3 or 4: the lane's two largest group maxima are enough
                // (the K-th largest of what the row's lanes keep is still at
                // most the K-th key); the list's lower two slots stay -inf
                top.v[0] = gm[0];
                top.v[1] = gm[1];
            } else {
#pragma unroll
                for (int q = 0; q < G; ++q) top.v[q] = gm[q];
            }
        } else {
#pragma unroll
            for (int q = 0; q < G; ++q) top.push(gm[q]);
        }
        top.merge_xor(1);
        top.merge_xor(2);
        const float lim = candidate_limit(top.template kth_of_merge_xor<K>(4), kErr);
        // candidate mask: 4 bits per float4, combined in a tree (a chain of 32
        // dependent ORs measured slower)
        unsigned mb[NV];
#pragma unroll
        for (int m = 0; m < NV; ++m)
            mb[m] = (kv[m][0] >= lim ? 1u : 0u) | (kv[m][1] >= lim ? 2u : 0u) | (kv[m][2] >= lim ? 4u : 0u) |
                    (kv[m][3] >= lim ? 8u : 0u);
#pragma unroll
        for (int w = 1; w < NV; w <<= 1)
#pragma unroll
            for (int m = 0; m + w < NV; m += 2 * w) mb[m] |= mb[m + w] << (4 * w);
        const unsigned mask = row < T ? mb[0] : 0u;

        // candidate offsets within the row: prefix over the row's 8 lanes
        const int n = __popc(mask);
        int incl = n;
#pragma unroll
        for (int d = 1; d < kLanesPerRow; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, d);
            if (j >= d) incl += y;
        }
        const int excl = incl - n;
        const int row_n = __shfl_sync(0xffffffffu, incl, lane | (kLanesPerRow - 1));

        if (__all_sync(0xffffffffu, n <= 8 && row_n <= 2 * kLanesPerRow)) {
            // The usual case, without loops: at most 8 candidates per lane and
            // 16 per row (at most 4 and 8 on most items).  Lane j scores the
            // row's j-th candidate (and its (j+8)-th, if any) and ranks it
            // against the others through shuffles.
            unsigned mm = mask;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int p = __ffs(mm) - 1;
                mm &= mm - 1;
                if (q < n) {
                    cc[excl + q] = kLaneCols * j + p;
                    ck[excl + q] = xr[p];
                }
            }
            if (__any_sync(0xffffffffu, n > 4)) {
#pragma unroll
                for (int q = 4; q < 8; ++q) {
                    const int p = __ffs(mm) - 1;
                    mm &= mm - 1;
                    if (q < n) {
                        cc[excl + q] = kLaneCols * j + p;
                        ck[excl + q] = xr[p];
                    }
                }
            }
            __syncwarp();
            issue(item + 1, ahead);  // every candidate's logit is in ck: the stage is free
            const bool has = j < row_n;
            const int c = has ? cc[j] : 0;
            const float s = sigmoid_rounded_once(ck[has ? j : 0]);
            // The row's list is in expert order, so an equal key ranks above
            // exactly when it sits earlier in the list: lane q < j counts on
            // o_q >= o, i.e. o_q > o - 1.  Keys order as o >= 0x007fffff (-inf);
            // lanes past the list carry 0 and rank below everything.
            const uint32_t o = has ? order_bits(__fadd_rn(s, __ldg(bias + c))) : 0u;
            const int src0 = lane & ~(kLanesPerRow - 1);
            int rank = 0;
            if (!__any_sync(0xffffffffu, row_n > kLanesPerRow)) {
#pragma unroll
                for (int d = 1; d < kLanesPerRow; ++d) {
                    const uint32_t oq = __shfl_sync(0xffffffffu, o, src0 | ((j + d) & (kLanesPerRow - 1)));
                    // (two spellings of one test: each keeps its variant's register count lower)
                    if constexpr (BAL)
                        rank += (oq > o) | ((oq == o) & (j + d >= kLanesPerRow));
                    else
                        rank += oq > (o - (uint32_t)((j + d) >> 3)) ? 1 : 0;
                }
            } else {
                // a second candidate per lane at list position j + 8, after
                // every first one
                const bool has2 = j + kLanesPerRow < row_n;
                const int c2 = has2 ? cc[j + kLanesPerRow] : 0;
                const float s2 = sigmoid_rounded_once(ck[has2 ? j + kLanesPerRow : 0]);
                const uint32_t o2 = has2 ? order_bits(__fadd_rn(s2, __ldg(bias + c2))) : 0u;
                rank = o2 > o ? 1 : 0;
                int rank2 = o >= o2 ? 1 : 0;
#pragma unroll
                for (int d = 1; d < kLanesPerRow; ++d) {
                    const int q = src0 | ((j + d) & (kLanesPerRow - 1));
                    const uint32_t oq = __shfl_sync(0xffffffffu, o, q);
                    const uint32_t oq2 = __shfl_sync(0xffffffffu, o2, q);
                    const uint32_t before = (uint32_t)((j + d) >> 3);  // lane q precedes lane j
                    rank += (oq > o - before ? 1 : 0) + (oq2 > o ? 1 : 0);
                    rank2 += (oq >= o2 ? 1 : 0) + (oq2 > o2 - before ? 1 : 0);
                }
                if (has2 && rank2 < K) {
                    ss[rank2] = s2;
                    sc[rank2] = c2;
                }
            }
            if (has && rank < K) {
                ss[rank] = s;
                sc[rank] = c;
            }
            __syncwarp();
        } else {
            issue(item + 1, ahead);  // this path reads the candidates' logits from global memory (L2)
            const int most = __reduce_max_sync(0xffffffffu, row_n);
            // rounds of up to kWin candidates per row (one round unless many keys tie)
            for (int w0 = 0; w0 < most; w0 += kWin) {
                if (incl > w0 && excl < w0 + kWin) {
                    unsigned mm = mask;
                    int off = excl;
                    while (mm) {
                        const int p = __ffs(mm) - 1;
                        mm &= mm - 1;
                        if (off >= w0 && off < w0 + kWin) cc[off - w0] = kLaneCols * j + p;
                        ++off;
                    }
                }
                __syncwarp();
                const int wn = min(kWin, row_n - w0);
                // exact scores: the row's 8 lanes share the round's candidates;
                // slots [wn, 8) get a sentinel that ranks below everything
                for (int e = j; e < wn; e += kLanesPerRow) {
                    const int c = cc[e];
                    const float s = sigmoid_rounded_once(__ldg(logits + row * (int64_t)Nr + c));
                    cs[e] = s;
                    ck[e] = __fadd_rn(s, __ldg(bias + c));
                }
                if (j >= wn) {
                    ck[j] = -INFINITY;
                    cc[j] = 0x7fffffff;
                }
                __syncwarp();
                // slot of each candidate: its rank under (key desc, index asc)
                const int dst = w0 == 0 ? 0 : K;
                for (int e = j; e < wn; e += kLanesPerRow) {
                    const float ke = ck[e];
                    const int ce = cc[e];
                    int rank = 0;
#pragma unroll
                    for (int q = 0; q < kLanesPerRow; ++q) {
                        const float kq = ck[q];
                        rank += (kq > ke || (kq == ke && cc[q] < ce)) ? 1 : 0;
                    }
                    for (int q = kLanesPerRow; q < wn; ++q) {
                        const float kq = ck[q];
                        rank += (kq > ke || (kq == ke && cc[q] < ce)) ? 1 : 0;
                    }
                    if (rank < K) {
                        sk[dst + rank] = ke;
                        ss[dst + rank] = cs[e];
                        sc[dst + rank] = ce;
                    }
                }
                __syncwarp();
                if (w0 > 0 && j == 0 && wn > 0) {
                    // merge this round's best min(K, wn) into the Top-K so far
                    float mk[K], ms[K];
                    int mc[K];
                    const int nb = min(K, wn);
                    int a = 0, b = 0;
#pragma unroll
                    for (int k = 0; k < K; ++k) {
                        const bool take_b =
                            b < nb && (sk[K + b] > sk[a] || (sk[K + b] == sk[a] && sc[K + b] < sc[a]));
                        const int src = take_b ? K + b : a;
                        mk[k] = sk[src];
                        ms[k] = ss[src];
                        mc[k] = sc[src];
                        b += take_b ? 1 : 0;
                        a += take_b ? 0 : 1;
                    }
#pragma unroll
                    for (int k = 0; k < K; ++k) {
                        sk[k] = mk[k];
                        ss[k] = ms[k];
                        sc[k] = mc[k];
                    }
                }
                __syncwarp();
            }
        }

        // gates (fp64, slot order), outputs, histogram: lane j writes slot j.
        // Slots [0, min(K, row_n)) hold the row's Top-K; fewer than K
        // candidates happen only when NaN or -inf keys leave slots unfilled.
        if (row < T && j < K) {
            double sum = 0.0;
#pragma unroll
            for (int k = 0; k < K; ++k)
                if (k < row_n) sum = __dadd_rn(sum, (double)ss[k]);
            if (j < row_n) {
                const int c = sc[j];
                topk_idx[row * K + j] = c;
                gates[row * K + j] = __double2float_rn(__ddiv_rn((double)ss[j], sum));
                atomicAdd(&hist[c], 1);
            } else {
                topk_idx[row * K + j] = 0x7fffffff;
                gates[row * K + j] = 0.0f;
                atomicOr(status, kStNonfinite);
            }
        }
        __syncwarp();  // the ring stage and the candidate slots are reused

        if (want_tiles && (item & 7) == 7) {
            const int tile = (int)blockIdx.x + (item >> 3) * (int)gridDim.x;
            if constexpr (BAL) {
                // the warp's 32 rows per column: lanes j, j + 8, j + 16, j + 24
                // hold the same columns; fold them (fixed order), lanes 0..7 store
#pragma unroll
                for (int m = 0; m < NV; ++m)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float v = psum[m][e];
                        v += __shfl_xor_sync(0xffffffffu, v, 8);
                        v += __shfl_xor_sync(0xffffffffu, v, 16);
                        if (r == 0) colsum[(kLaneCols + 4) * j + 4 * m + e] = v;  // padded like hb_s
                        psum[m][e] = 0.0f;
                    }
            }
            __syncthreads();
            for (int e = threadIdx.x; e < Nr; e += kThreads) {
                const int v = hist_tile[e];
                tile_counts[(size_t)tile * Nr + e] = v;
                hist_total[e] += v;
                hist_tile[e] = 0;
                if constexpr (BAL) {
                    const float *c0 = reinterpret_cast<const float *>(&cand[0]);
                    const float *c1 = reinterpret_cast<const float *>(&cand[1]);
                    const float *c2 = reinterpret_cast<const float *>(&cand[2]);
                    const float *c3 = reinterpret_cast<const float *>(&cand[3]);
                    const int pe = pad_col<NV>(e);
                    tile_psum[(size_t)tile * Nr + e] = ((c0[pe] + c1[pe]) + c2[pe]) + c3[pe];
                }
            }
            __syncthreads();
        }
    }
    cp_async_wait<0>();  // the zero-fill copies issued past the last item
    __syncthreads();
    for (int e = threadIdx.x; e < Nr; e += kThreads)
        if (hist_total[e] != 0) atomicAdd(&counts[e], hist_total[e]);
}

// Routing alone: the compiler's own register choice (64 at K = 4, N_r = 256)
// gives 8 CTAs per SM.
template <int K, int NV, bool FULL>
__global__ void __launch_bounds__(kThreads) router_logits_vec_kernel(const float *__restrict__ logits,
                                                                     const float *__restrict__ bias, int T, int Nr,
                                                                     int32_t *__restrict__ topk_idx,
                                                                     float *__restrict__ gates,
                                                                     int32_t *__restrict__ counts,
                                                                     int32_t *__restrict__ tile_counts,
                                                                     int32_t *__restrict__ status) {
    logits_vec_body<K, NV, FULL, false>(logits, bias, T, Nr, topk_idx, gates, counts, tile_counts, nullptr, status);
}

// With the balance statistics: the lane's column sums hold 4*NV more
// registers; 96 per thread keep 5 CTAs per SM.
template <int K, int NV, bool FULL>
__global__ void __launch_bounds__(kThreads, 5) router_logits_vec_balance_kernel(
    const float *__restrict__ logits, const float *__restrict__ bias, int T, int Nr, int32_t *__restrict__ topk_idx,
    float *__restrict__ gates, int32_t *__restrict__ counts, int32_t *__restrict__ tile_counts,
    float *__restrict__ tile_psum, int32_t *__restrict__ status) {
    logits_vec_body<K, NV, FULL, true>(logits, bias, T, Nr, topk_idx, gates, counts, tile_counts, tile_psum, status);
}

// max over i of |approximate score - exact score| as the bits of a
// non-negative float (those order like unsigned integers)
__global__ void score_error_kernel(const float *__restrict__ x, int64_t n, unsigned *__restrict__ max_bits,
                                   float *__restrict__ exact_out) {
    float worst = 0.0f;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float e = sigmoid_rounded_once(x[i]);
        worst = fmaxf(worst, fabsf(key_approx(x[i], 0.5f) - e));
        if (exact_out) exact_out[i] = e;
    }
    atomicMax(max_bits, __float_as_uint(worst));
}

}  // namespace

namespace {

// Per (kernel, device): the dynamic shared-memory grant is set once and the
// resident CTAs per SM are measured once (the persistent grid's size).
struct VecSetup {
    const void *kern;
    int device;
    int blocks_per_sm;
};
std::mutex g_vec_mu;
VecSetup g_vec[64];
int g_num_vec = 0;

cudaError_t vec_setup(const void *kern, size_t smem, int *blocks_per_sm) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lock(g_vec_mu);
    for (int i = 0; i < g_num_vec; ++i)
        if (g_vec[i].kern == kern && g_vec[i].device == dev) {
            *blocks_per_sm = g_vec[i].blocks_per_sm;
            return cudaSuccess;
        }
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    int b = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, kThreads, smem);
    if (err != cudaSuccess) return err;
    if (b < 1) b = 1;
    if (g_num_vec < 64) g_vec[g_num_vec++] = {kern, dev, b};
    *blocks_per_sm = b;
    return cudaSuccess;
}

template <int K, int NV, bool FULL, bool BAL>
cudaError_t launch_vec(const float *logits, const float *bias, int T, int Nr, int32_t *topk_idx, float *gates,
                       int32_t *counts, int32_t *tile_counts, float *tile_psum, int32_t *status, int num_sms,
                       cudaStream_t stream) {
    const void *kern = BAL ? reinterpret_cast<const void *>(&router_logits_vec_balance_kernel<K, NV, FULL>)
                           : reinterpret_cast<const void *>(&router_logits_vec_kernel<K, NV, FULL>);
    const size_t smem = vec_ring_bytes<NV>();
    int per_sm = 1;
    cudaError_t err = vec_setup(kern, smem, &per_sm);
    if (err != cudaSuccess) return err;
    const int num_tiles = (T + kTileTokens - 1) / kTileTokens;
    int grid = num_sms * per_sm;
    if (grid > num_tiles) grid = num_tiles;
    if constexpr (BAL)
        router_logits_vec_balance_kernel<K, NV, FULL><<<grid, kThreads, smem, stream>>>(
            logits, bias, T, Nr, topk_idx, gates, counts, tile_counts, tile_psum, status);
    else
        router_logits_vec_kernel<K, NV, FULL><<<grid, kThreads, smem, stream>>>(logits, bias, T, Nr, topk_idx, gates,
                                                                               counts, tile_counts, status);
    return cudaGetLastError();
}

}  // namespace

bool logits_vector_path(const float *logits, int Nr) {
    return Nr % 4 == 0 && (reinterpret_cast<uintptr_t>(logits) & 15) == 0;
}

cudaError_t launch_router_logits(const float *logits, const float *bias, int T, int Nr, int K, int32_t *topk_idx,
                                 float *gates, int32_t *counts, int32_t *tile_counts, float *tile_psum,
                                 int32_t *status, int num_sms, cudaStream_t stream) {
    const int num_tiles = (T + kTileTokens - 1) / kTileTokens;
    if (logits_vector_path(logits, Nr)) {
        // vector kernel: persistent CTAs, as many per SM as fit
        const int nv = Nr <= 64 ? 2 : (Nr <= 128 ? 4 : 8);
        const bool bal = tile_psum != nullptr;
        switch (K * 16 + nv) {
#define EBL_VLAUNCH(KK, NN, F, B) \
    launch_vec<KK, NN, F, B>(logits, bias, T, Nr, topk_idx, gates, counts, tile_counts, tile_psum, status, num_sms, stream)
#define EBL_VCASE(KK, NN)                                                                          \
    case KK * 16 + NN:                                                                             \
        if (bal) return Nr == 32 * NN ? EBL_VLAUNCH(KK, NN, true, true) : EBL_VLAUNCH(KK, NN, false, true); \
        return Nr == 32 * NN ? EBL_VLAUNCH(KK, NN, true, false) : EBL_VLAUNCH(KK, NN, false, false);
#define EBL_VCASES(KK) EBL_VCASE(KK, 2) EBL_VCASE(KK, 4) EBL_VCASE(KK, 8)
            EBL_VCASES(1)
            EBL_VCASES(2)
            EBL_VCASES(3)
            EBL_VCASES(4)
            EBL_VCASES(5)
            EBL_VCASES(6)
            EBL_VCASES(7)
            EBL_VCASES(8)
#undef EBL_VCASES
#undef EBL_VCASE
#undef EBL_VLAUNCH
            default:
                return cudaErrorInvalidValue;
        }
    }
    // row kernel: any N_r and alignment (the balance option runs beside it, as a
    // separate pass: launch_tile_psum_logits)
    if (tile_psum) return cudaErrorInvalidValue;
    int grid = num_sms * 16;
    if (grid > num_tiles) grid = num_tiles;
    switch (K) {
#define EBL_CASE(KK)                                                                                    \
    case KK:                                                                                            \
        router_logits_kernel<KK><<<grid, kThreads, 0, stream>>>(logits, bias, T, Nr, topk_idx, gates, \
                                                                counts, tile_counts, status);          \
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

cudaError_t launch_score_error(const float *x, int64_t n, float *max_err, float *exact_out, cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(max_err, 0, sizeof(float), stream);
    if (e != cudaSuccess) return e;
    if (n == 0) return cudaSuccess;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    score_error_kernel<<<(int)blocks, 256, 0, stream>>>(x, n, reinterpret_cast<unsigned *>(max_err), exact_out);
    return cudaGetLastError();
}

float logits_key_error_bound() { return kKeyErr; }

}  // namespace ebl
