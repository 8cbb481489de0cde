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
// then rank_kernel ranks each tile's pairs in pair order from its tile base
// (warp match on expert ids, 32 pairs at a time) into dest and perm, and
// copy_kernel streams every hidden row once from HBM to its K destinations
// with TMA bulk copies through a shared-memory ring.
//
// Combine: out[t,:] = sum_k g[t,k] * Y[dest[t*K+k],:], one warp per token,
// fp32 fma chain in slot order from 0 (deterministic, no atomics).

#include <mutex>

#include "launch.h"
#include "ptx.cuh"

namespace ebl {
namespace {

constexpr int kSegTiles = 32;

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

// Rank: one warp per tile ranks the tile's pairs in pair order from the tile's
// bases, 32 pairs at a time (warp match on the expert ids), and writes dest
// and perm.  Expert ids outside [0, N_r) get dest = -1; so do pairs whose
// rank falls outside [0, T*K), which only tile counts that disagree with
// topk_idx can cause.  Both raise EBL_ST_BAD_EXPERT.
constexpr int kRankWarps = 4;

__global__ void __launch_bounds__(kRankWarps * 32) rank_kernel(const int32_t *__restrict__ topk_idx,
                                                               const int32_t *__restrict__ bases, int T, int Nr,
                                                               int K, int32_t *__restrict__ perm,
                                                               int32_t *__restrict__ dest,
                                                               int32_t *__restrict__ status) {
    __shared__ int cnt_s[kRankWarps][kMaxExperts];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tile = blockIdx.x * kRankWarps + warp;
    if (tile >= num_tiles_of(T)) return;  // whole warps only; no CTA barrier below
    int *cnt = cnt_s[warp];
    for (int e = lane; e < Nr; e += 32) cnt[e] = bases[(size_t)tile * Nr + e];
    __syncwarp();
    const int row0 = tile * kTileTokens;
    const int np = min(kTileTokens, T - row0) * K;
    const size_t p0 = (size_t)row0 * K;
    const long long num_pairs = (long long)T * K;
    bool bad = false;
    for (int q0 = 0; q0 < np; q0 += 32) {
        const int q = q0 + lane;
        const bool valid = q < np;
        int e = valid ? topk_idx[p0 + q] : -1;
        const bool good = valid && (unsigned)e < (unsigned)Nr;
        if (valid && !good) bad = true;
        if (!good) e = valid ? -1 : -2;  // never equal to a good id
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        int j = -1;
        if (good) j = cnt[e] + __popc(peers & lanemask_lt());
        __syncwarp();
        if (good && lane == __ffs(peers) - 1) cnt[e] += __popc(peers);
        __syncwarp();
        if (good && (unsigned long long)j >= (unsigned long long)num_pairs) {
            bad = true;
            j = -1;
        }
        if (valid) {
            dest[p0 + q] = j;
            if (j >= 0) perm[j] = row0 + q / K;
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, kStBadExpert);
}

// Copy: TMA bulk copies.  One warp per CTA; lane 0 streams the CTA's rows
// (a contiguous block of tokens) through a ring of shared-memory stages in
// chunks of up to kChunkBytes: one bulk load per chunk, then one bulk store
// per destination row.  kCopyAhead loads are in flight; a stage is refilled
// only after the stores issued kCopyAhead chunks earlier have read it.  The
// lanes hold the dest entries of 32 rows at a time, loaded one batch ahead.
constexpr int kCopyStages = 12;
constexpr int kCopyAhead = kCopyStages / 2;
constexpr int kChunkBytes = 8192;
constexpr size_t kCopySmemBytes = (size_t)kCopyStages * kChunkBytes;

__device__ __forceinline__ void bulk_load(void *smem, const void *gmem, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(smem)),
                 "l"(gmem), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void bulk_store(void *gmem, const void *smem, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gmem), "r"(smem_u32(smem)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(32) copy_kernel(const uint8_t *__restrict__ hidden, const int32_t *__restrict__ dest,
                                                  int T, int row_bytes, int K, uint8_t *__restrict__ dispatched,
                                                  int32_t *__restrict__ status) {
    extern __shared__ __align__(128) uint8_t ring[];  // kCopyStages x kChunkBytes
    __shared__ uint64_t full[kCopyStages];
    __shared__ int abort_flag;
    const int lane = threadIdx.x;
    const int64_t per = ((int64_t)T + gridDim.x - 1) / gridDim.x;
    const int64_t r0 = (int64_t)blockIdx.x * per;
    const int64_t r1 = min((int64_t)T, r0 + per);
    if (r0 >= r1) return;
    if (lane == 0) {
        for (int s = 0; s < kCopyStages; ++s) mbar_init(&full[s], 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncwarp();
    const int cpr = (row_bytes + kChunkBytes - 1) / kChunkBytes;  // chunks per row
    const int64_t U = (r1 - r0) * cpr;
    auto chunk_row = [&](int64_t u) { return r0 + u / cpr; };
    auto chunk_off = [&](int64_t u) { return (int)(u % cpr) * kChunkBytes; };
    auto chunk_bytes = [&](int64_t u) { return (uint32_t)min(kChunkBytes, row_bytes - chunk_off(u)); };
    auto issue_load = [&](int64_t v) {
        const int s = (int)(v % kCopyStages);
        const uint32_t nb = chunk_bytes(v);
        mbar_arrive_expect_tx(&full[s], nb);
        bulk_load(ring + (size_t)s * kChunkBytes, hidden + chunk_row(v) * row_bytes + chunk_off(v), nb, &full[s]);
    };
    auto load_dest = [&](int64_t row, int (&dk)[kMaxTopK]) {
#pragma unroll
        for (int k = 0; k < kMaxTopK; ++k) dk[k] = (k < K && row < r1) ? dest[row * K + k] : -1;
    };

    if (lane == 0)
        for (int64_t v = 0; v < min((int64_t)kCopyAhead, U); ++v) issue_load(v);
    int64_t batch0 = r0;  // lane l holds the dest entries of row batch0 + l in dk
    int dk[kMaxTopK], dn[kMaxTopK];
    load_dest(batch0 + lane, dk);
    load_dest(batch0 + 32 + lane, dn);
    int64_t u = 0;
    for (; u < U; ++u) {
        const int64_t row = chunk_row(u);
        if (row >= batch0 + 32) {  // next batch of 32 rows (warp-uniform)
            batch0 += 32;
#pragma unroll
            for (int k = 0; k < kMaxTopK; ++k) dk[k] = dn[k];
            load_dest(batch0 + 32 + lane, dn);
        }
        const int s = (int)(u % kCopyStages);
        int ok = 1;
        if (lane == 0) {
            const int64_t v = u + kCopyAhead;
            if (v < U) {
                bulk_wait_read<kCopyAhead - 1>();
                issue_load(v);
            }
            ok = mbar_wait(&full[s], (uint32_t)((u / kCopyStages) & 1), &abort_flag) ? 1 : 0;
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        const int src = (int)(row - batch0);
        const int off = chunk_off(u);
        const uint32_t nb = chunk_bytes(u);
#pragma unroll
        for (int k = 0; k < kMaxTopK; ++k) {
            const int j = __shfl_sync(0xffffffffu, dk[k], src);
            if (lane == 0 && k < K && j >= 0)
                bulk_store(dispatched + (int64_t)j * row_bytes + off, ring + (size_t)s * kChunkBytes, nb);
        }
        if (lane == 0) bulk_commit();
    }
    if (lane == 0) {
        if (u < U) {
            // a load never landed: report, then give the loads already issued a
            // bounded time to land before the shared memory goes away.  The
            // iteration that gave up had issued chunk u + kCopyAhead before its
            // wait, so chunks u .. u + kCopyAhead (those below U) are in flight.
            atomicOr(status, kStTimeout);
            const int64_t issued = min(U, u + kCopyAhead + 1);
            for (int64_t w = u; w < issued; ++w)
                mbar_wait(&full[w % kCopyStages], (uint32_t)((w / kCopyStages) & 1), &abort_flag, 100000000ull);
        }
        bulk_wait_all();  // the stores read shared memory until they complete
    }
    __syncwarp();
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

namespace {

// The copy kernel's dynamic shared-memory grant, set once per device.
std::mutex g_copy_mu;
bool g_copy_ready[64] = {};

cudaError_t copy_setup() {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lock(g_copy_mu);
    if (dev >= 0 && dev < 64 && g_copy_ready[dev]) return cudaSuccess;
    err = cudaFuncSetAttribute(reinterpret_cast<const void *>(&copy_kernel),
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kCopySmemBytes);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < 64) g_copy_ready[dev] = true;
    return cudaSuccess;
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
    rank_kernel<<<(tiles + kRankWarps - 1) / kRankWarps, kRankWarps * 32, 0, stream>>>(topk_idx, ws_tiles, T, Nr, K,
                                                                                      perm, dest, status);
    cudaError_t err = copy_setup();
    if (err != cudaSuccess) return err;
    int grid = num_sms * 2;  // two 96 KB rings per SM
    if (grid > T) grid = T;
    copy_kernel<<<grid, 32, kCopySmemBytes, stream>>>(reinterpret_cast<const uint8_t *>(hidden), dest, T, d * 2, K,
                                                      reinterpret_cast<uint8_t *>(dispatched), status);
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
