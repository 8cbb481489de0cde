// dispatch.cu -- expert-sorted token dispatch and the gate-weighted combine.
//
// The pages name expert parallelism and no mechanism, so dispatch here is a
// stable counting sort of the (token, slot) pairs by expert id, in pair order
// p = t*K + k:
//   offsets[e] = sum of loads of experts < e;  j = offsets[e] + rank of p among
//   the pairs of expert e;  perm[j] = t;  dest[p] = j;  X[j,:] = hidden[t,:].
// The rank is made deterministic (no atomics decide it) in four passes:
//   1. tile_hist   per 128-token tile, per expert pair counts (skipped when
//                  the router already wrote tile_counts)
//   2. seg_sums    per segment of 32 tiles, per expert sums
//   3. seg_scan    one CTA: expert totals, offsets (exclusive scan over
//                  experts), segment bases (exclusive scan over segments)
//   4. tile_bases  per tile, per expert base = segment base + earlier tiles
// and the copy kernel ranks each tile's pairs in pair order from its tile base
// (warp match on expert ids, 32 pairs at a time) and streams every hidden row
// once from HBM to its K destinations with 16-byte loads and stores.
//
// Combine: out[t,:] = sum_k g[t,k] * Y[dest[t*K+k],:], one warp per token,
// fp32 fma chain in slot order from 0 (deterministic, no atomics).

#include "launch.h"
#include "ptx.cuh"

namespace ebl {
namespace {

constexpr int kSegTiles = 32;
constexpr int kCopyThreads = 256;
constexpr int kCopyWarps = kCopyThreads / 32;

__host__ __device__ inline int num_tiles_of(int T) { return (T + kTileTokens - 1) / kTileTokens; }
__host__ __device__ inline int num_segs_of(int tiles) { return (tiles + kSegTiles - 1) / kSegTiles; }

__global__ void __launch_bounds__(kTileTokens) tile_hist_kernel(const int32_t *__restrict__ topk_idx, int T, int Nr,
                                                                int K, int32_t *__restrict__ tile_counts,
                                                                int32_t *__restrict__ status) {
    __shared__ int h[kMaxExperts];
    for (int e = threadIdx.x; e < Nr; e += kTileTokens) h[e] = 0;
    __syncthreads();
    const int tile = blockIdx.x;
    const int row = tile * kTileTokens + threadIdx.x;
    bool bad = false;
    if (row < T) {
        for (int k = 0; k < K; ++k) {
            const int e = topk_idx[(size_t)row * K + k];
            if ((unsigned)e < (unsigned)Nr)
                atomicAdd(&h[e], 1);
            else
                bad = true;
        }
    }
    if (bad) atomicOr(status, kStBadExpert);
    __syncthreads();
    for (int e = threadIdx.x; e < Nr; e += kTileTokens) tile_counts[(size_t)tile * Nr + e] = h[e];
}

__global__ void __launch_bounds__(kMaxExperts) seg_sums_kernel(const int32_t *__restrict__ tile_counts,
                                                               int num_tiles, int Nr,
                                                               int32_t *__restrict__ seg) {
    const int e = threadIdx.x;
    if (e >= Nr) return;
    const int t0 = blockIdx.x * kSegTiles;
    const int t1 = min(num_tiles, t0 + kSegTiles);
    int s = 0;
    for (int t = t0; t < t1; ++t) s += tile_counts[(size_t)t * Nr + e];
    seg[(size_t)blockIdx.x * Nr + e] = s;
}

__global__ void __launch_bounds__(kMaxExperts) seg_scan_kernel(int32_t *__restrict__ seg, int num_segs, int Nr,
                                                               long long num_pairs, int32_t *__restrict__ offsets,
                                                               int32_t *__restrict__ status) {
    __shared__ int warp_tot[kMaxExperts / 32];
    const int e = threadIdx.x;
    const int lane = e & 31, warp = e >> 5;
    int total = 0;
    if (e < Nr)
        for (int s = 0; s < num_segs; ++s) total += seg[(size_t)s * Nr + e];
    // exclusive scan of the expert totals over e
    int incl = total;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += warp_tot[w];
    const int excl = before + incl - total;
    if (e < Nr) {
        offsets[e] = excl;
        if (e == Nr - 1) {
            offsets[Nr] = excl + total;
            // tile counts that do not add up to T*K cannot come from this topk_idx
            if ((long long)excl + total != num_pairs) atomicOr(status, kStBadCounts);
        }
        int run = excl;
        for (int s = 0; s < num_segs; ++s) {
            const int v = seg[(size_t)s * Nr + e];
            seg[(size_t)s * Nr + e] = run;
            run += v;
        }
    }
}

__global__ void __launch_bounds__(kMaxExperts) tile_bases_kernel(const int32_t *tile_counts,
                                                                 const int32_t *__restrict__ seg, int num_tiles,
                                                                 int Nr, int32_t *bases) {
    const int e = threadIdx.x;
    if (e >= Nr) return;
    const int t0 = blockIdx.x * kSegTiles;
    const int t1 = min(num_tiles, t0 + kSegTiles);
    int run = seg[(size_t)blockIdx.x * Nr + e];
    for (int t = t0; t < t1; ++t) {
        const int v = tile_counts[(size_t)t * Nr + e];  // may alias bases: read before write
        bases[(size_t)t * Nr + e] = run;
        run += v;
    }
}

__global__ void __launch_bounds__(kCopyThreads) rank_copy_kernel(const uint4 *__restrict__ hidden,
                                                                 const int32_t *__restrict__ topk_idx,
                                                                 const int32_t *__restrict__ bases, int T,
                                                                 int d8, int Nr, int K, int32_t *__restrict__ perm,
                                                                 int32_t *__restrict__ dest,
                                                                 uint4 *__restrict__ dispatched,
                                                                 int32_t *__restrict__ status) {
    __shared__ int cnt[kMaxExperts];
    __shared__ int dst_s[kTileTokens * kMaxTopK];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_tiles = num_tiles_of(T);
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        const int row0 = tile * kTileTokens;
        const int rows = min(kTileTokens, T - row0);
        const int np = rows * K;
        const size_t p0 = (size_t)row0 * K;
        for (int e = threadIdx.x; e < Nr; e += kCopyThreads) cnt[e] = bases[(size_t)tile * Nr + e];
        for (int q = threadIdx.x; q < np; q += kCopyThreads) dst_s[q] = topk_idx[p0 + q];
        __syncthreads();
        if (warp == 0) {
            const long long num_rows = (long long)T * K;
            bool bad = false, bad_base = false;
            for (int q0 = 0; q0 < np; q0 += 32) {
                const int q = q0 + lane;
                const bool valid = q < np;
                int e = valid ? dst_s[q] : -1;
                const bool good = valid && (unsigned)e < (unsigned)Nr;
                if (valid && !good) bad = true;
                if (!good) e = -1 - (valid ? 0 : 1);  // invalid lanes never match good ones
                const uint32_t peers = __match_any_sync(0xffffffffu, e);
                int j = -1;
                if (good) j = cnt[e] + __popc(peers & lanemask_lt());
                __syncwarp();
                if (good && lane == __ffs(peers) - 1) cnt[e] += __popc(peers);
                if (good && (unsigned)j >= (unsigned)num_rows) {  // tile counts that disagree with topk_idx
                    bad_base = true;
                    j = -1;
                }
                if (valid) {
                    dst_s[q] = j;
                    dest[p0 + q] = j;
                    if (j >= 0) perm[j] = (row0 + q / K);
                }
                __syncwarp();
            }
            if (bad || bad_base) atomicOr(status, kStBadExpert);
        }
        __syncthreads();
        // stream the rows: warp w copies rows w, w + 8, ...
        for (int r = warp; r < rows; r += kCopyWarps) {
            const uint4 *src = hidden + (size_t)(row0 + r) * d8;
            int dj[kMaxTopK];
#pragma unroll
            for (int k = 0; k < kMaxTopK; ++k) dj[k] = k < K ? dst_s[r * K + k] : -1;
            int c = lane;
            for (; c + 96 < d8; c += 128) {
                const uint4 v0 = __ldcs(src + c), v1 = __ldcs(src + c + 32), v2 = __ldcs(src + c + 64),
                            v3 = __ldcs(src + c + 96);
#pragma unroll
                for (int k = 0; k < kMaxTopK; ++k) {
                    if (dj[k] < 0) continue;
                    uint4 *dst = dispatched + (size_t)dj[k] * d8;
                    __stcs(dst + c, v0);
                    __stcs(dst + c + 32, v1);
                    __stcs(dst + c + 64, v2);
                    __stcs(dst + c + 96, v3);
                }
            }
            for (; c < d8; c += 32) {
                const uint4 v = __ldcs(src + c);
#pragma unroll
                for (int k = 0; k < kMaxTopK; ++k)
                    if (dj[k] >= 0) __stcs(dispatched + (size_t)dj[k] * d8 + c, v);
            }
        }
        __syncthreads();
    }
}

__device__ __forceinline__ void fma_bf16x8(const uint4 v, float g, float (&acc)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fmaf_rn(g, __uint_as_float(w[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = __fmaf_rn(g, __uint_as_float(w[i] & 0xffff0000u), acc[2 * i + 1]);
    }
}

template <int K>
__global__ void __launch_bounds__(256) combine_kernel(const uint4 *__restrict__ Y, const float *__restrict__ gates,
                                                      const int32_t *__restrict__ dest, int T, int d8,
                                                      float4 *__restrict__ out, int32_t *__restrict__ status) {
    const int lane = threadIdx.x & 31;
    const int warps_total = gridDim.x * (blockDim.x >> 5);
    const long long rows_Y = (long long)T * K;
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps_total) {
        int dj[K];
        float g[K];
        bool bad = false;
#pragma unroll
        for (int k = 0; k < K; ++k) {
            dj[k] = dest[(size_t)t * K + k];
            g[k] = gates[(size_t)t * K + k];
            if (dj[k] < 0 || dj[k] >= rows_Y) {
                bad = true;
                dj[k] = -1;
            }
        }
        if (bad && lane == 0) atomicOr(status, kStBadDest);
        float4 *o = out + (size_t)t * d8 * 2;
        for (int c = lane; c < d8; c += 32) {
            uint4 v[K];
#pragma unroll
            for (int k = 0; k < K; ++k)
                v[k] = dj[k] >= 0 ? __ldcs(Y + (size_t)dj[k] * d8 + c) : make_uint4(0, 0, 0, 0);
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < K; ++k)
                if (dj[k] >= 0) fma_bf16x8(v[k], g[k], acc);
            __stcs(o + 2 * c, make_float4(acc[0], acc[1], acc[2], acc[3]));
            __stcs(o + 2 * c + 1, make_float4(acc[4], acc[5], acc[6], acc[7]));
        }
    }
}

}  // namespace

size_t dispatch_workspace_bytes(int T, int Nr) {
    const int tiles = num_tiles_of(T);
    const int segs = num_segs_of(tiles);
    return ((size_t)tiles + (size_t)segs) * (size_t)Nr * sizeof(int32_t);
}

cudaError_t launch_dispatch(const uint16_t *hidden, const int32_t *topk_idx, const int32_t *tile_counts, int T,
                            int d, int Nr, int K, int32_t *offsets, int32_t *perm, int32_t *dest,
                            uint16_t *dispatched, void *workspace, int32_t *status, int num_sms,
                            cudaStream_t stream) {
    const int tiles = num_tiles_of(T);
    const int segs = num_segs_of(tiles);
    int32_t *ws_tiles = static_cast<int32_t *>(workspace);        // [tiles, Nr]: counts, then bases
    int32_t *ws_seg = ws_tiles + (size_t)tiles * Nr;               // [segs, Nr]: sums, then bases
    const int32_t *tc = tile_counts;
    if (tc == nullptr) {
        tile_hist_kernel<<<tiles, kTileTokens, 0, stream>>>(topk_idx, T, Nr, K, ws_tiles, status);
        tc = ws_tiles;
    }
    seg_sums_kernel<<<segs, kMaxExperts, 0, stream>>>(tc, tiles, Nr, ws_seg);
    seg_scan_kernel<<<1, kMaxExperts, 0, stream>>>(ws_seg, segs, Nr, (long long)T * K, offsets, status);
    tile_bases_kernel<<<segs, kMaxExperts, 0, stream>>>(tc, ws_seg, tiles, Nr, ws_tiles);
    int grid = num_sms * 4;
    if (grid > tiles) grid = tiles;
    rank_copy_kernel<<<grid, kCopyThreads, 0, stream>>>(reinterpret_cast<const uint4 *>(hidden), topk_idx,
                                                        ws_tiles, T, d / 8, Nr, K, perm, dest,
                                                        reinterpret_cast<uint4 *>(dispatched), status);
    return cudaGetLastError();
}

cudaError_t launch_combine(const uint16_t *expert_out, const float *gates, const int32_t *dest, int T, int d,
                           int K, float *out, int32_t *status, int num_sms, cudaStream_t stream) {
    const int warps_per_block = 8;
    long long blocks = ((long long)T + warps_per_block - 1) / warps_per_block;
    const long long cap = (long long)num_sms * 8;
    const int grid = (int)(blocks < cap ? blocks : cap);
    const uint4 *Y = reinterpret_cast<const uint4 *>(expert_out);
    float4 *o = reinterpret_cast<float4 *>(out);
    switch (K) {
#define EBL_CASE(KK)                                                                               \
    case KK:                                                                                       \
        combine_kernel<KK><<<grid, warps_per_block * 32, 0, stream>>>(Y, gates, dest, T, d / 8, o, \
                                                                      status);                     \
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
