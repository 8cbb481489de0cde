// router_gemm.cu -- the fused router kernel, GEMM mode (sm_100a).
//
// Per token t (a row of hidden) and expert i (a row of W_router):
//   x = h_t . w_i  (bf16 x bf16 -> fp32 on the 5th-generation tensor cores),
//   s = sigmoid(x), key = s + b_i (bias only inside Top-K), Top-K of key,
//   gates g = s / sum of the selected s (bias-free), per-expert load counts.
// Sources: "Arcee Trinity Large Technical Report" section 2.3 (sigmoid routing
// with normalized scores; Top-K on score plus bias; gates from the scores
// without the bias); "SMEBU Load Balancing" eq. (17).
//
// Design (one persistent CTA per SM, warp-specialised, CTA pairs):
//   pairs       the two CTAs of a 2-CTA cluster form one 256-token tile: each
//               loads its own 128 token rows and half of W, and one
//               tcgen05.mma.cta_group::2 (M=256) covers both, so W crosses
//               L2 -> SM once per 256 tokens (half the L2 traffic and half the
//               shared-memory fill of single-CTA tiles).
//   TMA warp    streams the 128x128 hidden tile and the (N_r/2) x 128 slice of W
//               for each K step (two 64-column boxes each, 128-byte swizzle)
//               into a ring of shared-memory stages.
//   MMA warp    owns TMEM; in the even CTA it issues tcgen05.mma (M=256, N=N_r,
//               K=16, 8 per stage) for the pair into a double-buffered
//               fp32 accumulator (2 x N_r columns per CTA), so the epilogue of
//               tile i overlaps the MMAs of tile i+1.
//   epilogue    G groups of 4 warps (G = 2 when N_r % 64 == 0, else 1).  Warp
//               w reads TMEM lane quadrant w%4 (one token row per thread);
//               group g = w/4 owns the experts [g*N_r/G, (g+1)*N_r/G).  Each
//               thread runs sigmoid, +bias and a running Top-K over its
//               experts; group 1 hands its sorted partial list to group 0
//               through shared memory, and group 0 merges, writes indices and
//               gates, and keeps the load histogram (and, for the z-loss, a
//               running log-sum-exp per row).  Two epilogue warps per SM
//               sub-partition keep up with the MMAs.
//   balance     optionally (for the sequence-wise balance loss) each thread
//               also totals its row's scores; the groups exchange the totals,
//               read the accumulator a second time, and fold the normalised
//               scores s / total of their 32 rows into column sums with warp
//               shuffles; the tile's sums per expert go to tile_psum in a
//               fixed order, so they are deterministic.
// The logits never leave TMEM.  Counts reach global memory with one atomic per
// expert per CTA; tile_counts with one store per expert per tile.  Every
// pipeline wait is bounded (EBL_ST_TIMEOUT, then a clean exit).

#include <mutex>

#include "launch.h"
#include "ptx.cuh"
#include "topk.cuh"

namespace ebl {
namespace {

constexpr int kSubK = 64;               // hidden elements per TMA box: one 128-byte swizzle row
constexpr int kNSub = 2;                // boxes per pipeline stage
constexpr int kBlockK = kSubK * kNSub;  // hidden elements per stage (8 MMAs between barriers)
constexpr int kUmmaK = 16;              // K of one kind::f16 MMA
constexpr int kChunk = 16;              // TMEM columns per epilogue load
constexpr int kMaxStages = 8;           // ring depth cap (shared memory decides: 3 at N_r = 256)
constexpr uint32_t kASubBytes = kTileTokens * kSubK * 2;
constexpr uint32_t kATileBytes = kASubBytes * kNSub;

__host__ __device__ constexpr int threads_of(int G) { return (4 * G + 2) * 32; }

constexpr int kPair = 2;  // CTAs per MMA (cluster size)

// Bytes of this CTA's slice of W per box and per stage (N_r/2 rows of 128 bytes).
__host__ __device__ inline uint32_t b_sub_bytes(int Nr) { return (uint32_t)(Nr / kPair) * kSubK * 2; }
__host__ __device__ inline uint32_t b_tile_bytes(int Nr) { return b_sub_bytes(Nr) * kNSub; }

__host__ __device__ inline uint32_t tmem_columns(int Nr) {
    uint32_t need = 2u * (uint32_t)Nr, c = 32;
    while (c < need) c <<= 1;
    return c;
}

// Kernel options (the E template argument): z-loss statistic, and the
// per-tile statistics of the sequence-wise balance loss.
constexpr int kOptZloss = 1;
constexpr int kOptBalance = 2;

// Shared memory after the stage ring: barriers, then (16-byte aligned) the
// bias, the histograms and the partial-list exchange buffers; with the balance
// option, two more barriers, the per-row score totals of every group and the
// per-warp column sums.
struct Misc {
    size_t bar_off, vec_off, aux_off, total;
};

__host__ __device__ inline Misc misc_layout(int Nr, int K, int G, int stages, int E) {
    Misc m;
    m.bar_off = (size_t)stages * (kATileBytes + b_tile_bytes(Nr));
    // full[S], empty[S], tfull[2], tempty[2], epi_sync, drain, list_full, list_empty; tmem slot, abort flag
    const size_t bars = (size_t)(2 * stages + 8) * 8 + 16;
    m.vec_off = m.bar_off + ((bars + 15) & ~size_t(15));
    const size_t vec = (size_t)4 * Nr * 4 + (size_t)3 * (G - 1) * K * kTileTokens * 4 +
                       (size_t)2 * (G - 1) * kTileTokens * 4;  // partial lists; partial log-sum-exp
    m.aux_off = (m.vec_off + vec + 15) & ~size_t(15);
    m.total = m.aux_off;
    if (E & kOptBalance) m.total += 16 + (size_t)(G * kTileTokens + 4 * Nr) * 4;
    return m;
}

__device__ __forceinline__ bool wait_timed(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_timer_ns() - t0 > kWaitLimitNs) return false;
    return true;
}

// Running log-sum-exp of a row's logits as (max, sum of exp(x - max)).
struct RowLse {
    float m, s;
    __device__ __forceinline__ void init() {
        m = -INFINITY;
        s = 0.0f;
    }
    __device__ __forceinline__ void merge(float m2, float s2) {
        const float nm = fmaxf(m, m2);
        s = s * __expf(m - nm) + s2 * __expf(m2 - nm);
        m = nm;
    }
};

template <int K, bool Z, bool P>
__device__ __forceinline__ void consume_chunk(const uint32_t (&r)[kChunk], const float *__restrict__ bias_s, int c,
                                              RowTopK<K> &tk, RowLse &lse, float &rsum) {
    if constexpr (Z) {  // z-loss: log-sum-exp of the chunk, folded into the row's
        float cm = __uint_as_float(r[0]);
#pragma unroll
        for (int j = 1; j < kChunk; ++j) cm = fmaxf(cm, __uint_as_float(r[j]));
        float cs = 0.0f;
#pragma unroll
        for (int j = 0; j < kChunk; ++j) cs += __expf(__uint_as_float(r[j]) - cm);
        lse.merge(cm, cs);
    }
    const float4 *b4 = reinterpret_cast<const float4 *>(bias_s + c);
#pragma unroll
    for (int q = 0; q < kChunk / 4; ++q) {
        const float4 bb = b4[q];
        const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float x = __uint_as_float(r[4 * q + j]);
            const float s = fast_rcp(1.0f + __expf(-x));
            if constexpr (P) rsum += s;
            tk.push(__fadd_rn(s, bv[j]), s, c + 4 * q + j);
        }
    }
}

// One step of a warp's column sums over its 32 rows: each lane keeps W of its
// 2W values, the half picked by lane bit 2W, and adds the partner's matching
// half (partner = lane ^ 2W).
template <int W>
__device__ __forceinline__ void column_fold(float (&v)[kChunk], int lane) {
    const bool hi = (lane & (2 * W)) != 0;
#pragma unroll
    for (int j = 0; j < W; ++j) {
        const float send = hi ? v[j] : v[j + W];
        const float keep = hi ? v[j + W] : v[j];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, 2 * W);
    }
}

// Sums over the warp's 32 rows of the 16 columns in v (this lane's row):
// lanes 2c and 2c + 1 return the sum of column c.  16 shuffles per 16 columns.
__device__ __forceinline__ float warp_column_sums(float (&v)[kChunk], int lane) {
    column_fold<8>(v, lane);
    column_fold<4>(v, lane);
    column_fold<2>(v, lane);
    column_fold<1>(v, lane);
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// Normalised scores s / total of one 16-column chunk (inv = 1 / total, or 0
// for a row past T), folded into the warp's column sums and stored in pw.
__device__ __forceinline__ void balance_chunk(const uint32_t (&r)[kChunk], float inv, int lane, float *pw) {
    float v[kChunk];
#pragma unroll
    for (int j = 0; j < kChunk; ++j) v[j] = fast_rcp(1.0f + __expf(-__uint_as_float(r[j]))) * inv;
    const float sum = warp_column_sums(v, lane);
    if ((lane & 1) == 0) pw[lane >> 1] = sum;
}

template <int K, int G, int E>
__global__ void __launch_bounds__(threads_of(G), 1)
    router_gemm_kernel(const __grid_constant__ CUtensorMap tmap_h, const __grid_constant__ CUtensorMap tmap_w,
                       const float *__restrict__ bias, int T, int d, int Nr, int stages,
                       int32_t *__restrict__ topk_idx, float *__restrict__ gates, int32_t *__restrict__ counts,
                       int32_t *__restrict__ tile_counts, double *__restrict__ zloss_sum,
                       float *__restrict__ tile_psum, int32_t *__restrict__ status) {
    constexpr bool Z = (E & kOptZloss) != 0;
    constexpr bool P = (E & kOptBalance) != 0;
    constexpr int kEpiWarps = 4 * G;
    constexpr int kProducerWarp = 4 * G;
    constexpr int kMmaWarp = 4 * G + 1;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const Misc ml = misc_layout(Nr, K, G, stages, E);
    const uint32_t b_bytes = b_tile_bytes(Nr);
    uint8_t *smA = smem;
    uint8_t *smB = smem + (size_t)stages * kATileBytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + ml.bar_off);
    uint64_t *empty = full + stages;
    uint64_t *tfull = empty + stages;
    uint64_t *tempty = tfull + 2;
    uint64_t *epi_sync = tempty + 2;
    uint64_t *drain = epi_sync + 1;
    uint64_t *list_full = drain + 1;
    uint64_t *list_empty = list_full + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(list_empty + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *bias_s = reinterpret_cast<float *>(smem + ml.vec_off);
    int *hist_total = reinterpret_cast<int *>(bias_s + Nr);
    int *hist_tile = hist_total + Nr;  // [2][Nr]
    float *pl_key = reinterpret_cast<float *>(hist_tile + 2 * Nr);  // [G-1][K][128]
    float *pl_s = pl_key + (G - 1) * K * kTileTokens;
    int *pl_idx = reinterpret_cast<int *>(pl_s + (G - 1) * K * kTileTokens);
    float *pl_zm = reinterpret_cast<float *>(pl_idx + (G - 1) * K * kTileTokens);  // [G-1][128]
    float *pl_zs = pl_zm + (G - 1) * kTileTokens;
    uint64_t *rows_ready = reinterpret_cast<uint64_t *>(smem + ml.aux_off);  // balance option only
    uint64_t *cols_ready = rows_ready + 1;
    float *row_total = reinterpret_cast<float *>(cols_ready + 1);  // [G][128]
    float *col_part = row_total + G * kTileTokens;                 // [4][Nr]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // CTA `rank` of a cluster pair owns 128-token tile 2*p + rank of pair
    // tile p; the even CTA (rank 0) issues the MMAs for both.
    const uint32_t rank = cluster_ctarank();
    const int unit = (int)blockIdx.x / kPair;       // cluster index
    const int num_units = (int)gridDim.x / kPair;   // clusters in the grid
    const int num_tiles = (T + kTileTokens - 1) / kTileTokens;   // 128-token tiles
    const int num_work = (num_tiles + kPair - 1) / kPair;        // 256-token pair tiles
    const int num_kb = (d + kBlockK - 1) / kBlockK;  // a last half stage reads zeros past d
    const uint32_t tcols = tmem_columns(Nr);

    for (int i = threadIdx.x; i < Nr; i += threads_of(G)) {
        bias_s[i] = bias[i];
        hist_total[i] = 0;
        hist_tile[i] = 0;
        hist_tile[Nr + i] = 0;
    }
    if (warp == kProducerWarp && lane == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], kPair * kEpiWarps);  // one arrival per epilogue warp of the pair
        }
        mbar_init(epi_sync, 128);
        mbar_init(drain, 1);
        mbar_init(list_full, (G - 1) * 128 > 0 ? (G - 1) * 128 : 1);
        mbar_init(list_empty, 128);
        if constexpr (P) {
            mbar_init(rows_ready, kEpiWarps * 32);
            mbar_init(cols_ready, kEpiWarps * 32);
        }
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap_h);
        prefetch_tmap(&tmap_w);
    }
    if (warp == kMmaWarp) {  // same warp id in both CTAs, as the pair allocation requires
        tmem_alloc_pair(tmem_slot, tcols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the peer's barriers exist before anyone signals them
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == kProducerWarp) {
        if (lane == 0) {
            const uint64_t pol_h = l2_policy_evict_first();  // hidden: read once
            const uint64_t pol_w = l2_policy_evict_last();   // W_router: re-read by every tile
            const int w_row0 = (int)rank * (Nr / kPair);     // this CTA's slice of W
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int wk = unit; wk < num_work && ok; wk += num_units) {
                const int tile = wk * kPair + (int)rank;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    // both CTAs' loads complete on the even CTA's barrier, which the
                    // even CTA arms with the bytes of the whole pair
                    const uint32_t bar0 = map_to_cta(smem_u32(&full[s]), 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)kPair * (kATileBytes + b_bytes));
                    for (int u = 0; u < kNSub; ++u) {
                        tma_load_2d_pair(smA + (size_t)s * kATileBytes + u * kASubBytes, &tmap_h, bar0,
                                         kb * kBlockK + u * kSubK, tile * kTileTokens, pol_h);
                        tma_load_2d_pair(smB + (size_t)s * b_bytes + u * b_sub_bytes(Nr), &tmap_w, bar0,
                                         kb * kBlockK + u * kSubK, w_row0, pol_w);
                    }
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok) {
                atomicOr(status, kStTimeout);
                *abort_flag = 1;
                // the pair's loads signal the even CTA: give loads in flight a
                // fixed grace period to land instead of waiting on a barrier
                const uint64_t t0 = global_timer_ns();
                while (global_timer_ns() - t0 < 2000000ull) {
                }
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0 && rank == 0) {
            const uint32_t idesc = idesc_bf16_f32(kTileTokens * kPair, (uint32_t)Nr);
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            int it = 0;
            for (int wk = unit; wk < num_work && ok; wk += num_units, ++it) {
                const int acc = it & 1;
                const uint32_t use = (uint32_t)(it >> 1);
                if (!mbar_wait(&tempty[acc], (use & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * Nr);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&full[s], ph, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smA + (size_t)s * kATileBytes);
                    const uint32_t b0 = smem_u32(smB + (size_t)s * b_bytes);
#pragma unroll
                    for (int kk = 0; kk < kBlockK / kUmmaK; ++kk) {
                        const int u = kk / (kSubK / kUmmaK), w = kk % (kSubK / kUmmaK);
                        const uint64_t ad = smem_desc_sw128_kmajor(a0 + u * kASubBytes + w * kUmmaK * 2);
                        const uint64_t bd = smem_desc_sw128_kmajor(b0 + u * b_sub_bytes(Nr) + w * kUmmaK * 2);
                        umma_bf16_pair(d_tmem, ad, bd, idesc, (uint32_t)(kb | kk));
                    }
                    // free the stage (in both CTAs) once these MMAs have read it
                    umma_commit_pair_mc(&empty[s], 0x3);
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                // accumulator complete (in both CTAs)
                umma_commit_pair_mc(&tfull[acc], 0x3);
            }
            if (!ok) {
                atomicOr(status, kStTimeout);
                *abort_flag = 1;
            }
            // every MMA this thread issued has finished once `drain` completes
            umma_commit_pair(drain);
            wait_timed(drain, 0);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quad = warp & 3;
        const int group = warp >> 2;
        const int rloc = quad * 32 + lane;  // row within the tile = TMEM lane
        const int cpg = Nr / G;             // experts per group (a multiple of 32)
        const int c0 = group * cpg;
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        const bool want_tiles = tile_counts != nullptr;
        uint32_t sync_ph = 0, aux_ph = 0;
        bool ok = true;
        int it = 0;
        float zacc = 0.0f;  // this thread's rows: sum of log-sum-exp squared
        for (int wk = unit; wk < num_work; wk += num_units, ++it) {
            const int tile = wk * kPair + (int)rank;
            const int acc = it & 1;
            const uint32_t use = (uint32_t)(it >> 1);
            if (!mbar_wait(&tfull[acc], use & 1u, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();

            RowTopK<K> tk;
            tk.init();
            RowLse lse;
            lse.init();
            float rsum = 0.0f;
            const uint32_t taddr = tmem_base + lane_base + (uint32_t)(acc * Nr + c0);
            uint32_t ra[kChunk], rb[kChunk];
            __syncwarp();
            tmem_ld_32x32b_x16(taddr, ra);
            tmem_ld_wait_x16(ra);
            for (int c = 0; c < cpg; c += 2 * kChunk) {  // cpg % 32 == 0: chunks come in pairs
                __syncwarp();
                tmem_ld_32x32b_x16(taddr + (uint32_t)(c + kChunk), rb);
                consume_chunk<K, Z, P>(ra, bias_s, c0 + c, tk, lse, rsum);
                __syncwarp();
                tmem_ld_wait_x16(rb);
                const bool more = c + 2 * kChunk < cpg;
                if (more) tmem_ld_32x32b_x16(taddr + (uint32_t)(c + 2 * kChunk), ra);
                consume_chunk<K, Z, P>(rb, bias_s, c0 + c + kChunk, tk, lse, rsum);
                __syncwarp();
                if (more) tmem_ld_wait_x16(ra);
            }
            if constexpr (P) {
                // the row's total over all experts (groups in order, the same sum
                // in every group), then a second pass over this group's columns
                row_total[group * kTileTokens + rloc] = rsum;
                mbar_arrive(rows_ready);
                if (!mbar_wait(rows_ready, aux_ph, abort_flag)) {
                    ok = false;
                    break;
                }
                float total = 0.0f;
#pragma unroll
                for (int g = 0; g < G; ++g) total += row_total[g * kTileTokens + rloc];
                const float inv = (tile * kTileTokens + rloc < T && total > 0.0f) ? __frcp_rn(total) : 0.0f;
                float *pw = col_part + quad * Nr + c0;
                __syncwarp();
                tmem_ld_32x32b_x16(taddr, ra);
                tmem_ld_wait_x16(ra);
                for (int c = 0; c < cpg; c += 2 * kChunk) {
                    __syncwarp();
                    tmem_ld_32x32b_x16(taddr + (uint32_t)(c + kChunk), rb);
                    balance_chunk(ra, inv, lane, pw + c);
                    __syncwarp();
                    tmem_ld_wait_x16(rb);
                    const bool more = c + 2 * kChunk < cpg;
                    if (more) tmem_ld_32x32b_x16(taddr + (uint32_t)(c + 2 * kChunk), ra);
                    balance_chunk(rb, inv, lane, pw + c + kChunk);
                    __syncwarp();
                    if (more) tmem_ld_wait_x16(ra);
                }
                mbar_arrive(cols_ready);
            }
            // this warp is done with the accumulator: hand it back to the MMA warp
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(map_to_cta(smem_u32(&tempty[acc]), 0));
            if constexpr (P) {
                // the tile's column sums: the four row quadrants in order
                if (!mbar_wait(cols_ready, aux_ph, abort_flag)) {
                    ok = false;
                    break;
                }
                aux_ph ^= 1u;
                if (tile < num_tiles)
                    for (int e = (int)threadIdx.x; e < Nr; e += kEpiWarps * 32)
                        tile_psum[(size_t)tile * Nr + e] =
                            ((col_part[e] + col_part[Nr + e]) + col_part[2 * Nr + e]) + col_part[3 * Nr + e];
            }

            if (group > 0) {
                // publish the sorted partial list for group 0
                if (!mbar_wait(list_empty, (uint32_t)(it & 1) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                const int base = (group - 1) * K * kTileTokens + rloc;
#pragma unroll
                for (int k = 0; k < K; ++k) {
                    pl_key[base + k * kTileTokens] = tk.key[k];
                    pl_s[base + k * kTileTokens] = tk.score[k];
                    pl_idx[base + k * kTileTokens] = tk.idx[k];
                }
                if constexpr (Z) {
                    pl_zm[(group - 1) * kTileTokens + rloc] = lse.m;
                    pl_zs[(group - 1) * kTileTokens + rloc] = lse.s;
                }
                mbar_arrive(list_full);
                continue;
            }

            if (G > 1) {
                // merge the partial lists in group order: every expert of a later
                // group has a higher index, and each list is sorted by (key desc,
                // index asc), so pushes keep the tie rule
                if (!mbar_wait(list_full, (uint32_t)(it & 1), abort_flag)) {
                    ok = false;
                    break;
                }
                for (int g = 1; g < G; ++g) {
                    const int base = (g - 1) * K * kTileTokens + rloc;
#pragma unroll
                    for (int k = 0; k < K; ++k) {
                        const float kv = pl_key[base + k * kTileTokens];
                        if (!(kv > tk.key[K - 1])) break;
                        tk.push(kv, pl_s[base + k * kTileTokens], pl_idx[base + k * kTileTokens]);
                    }
                    if constexpr (Z) lse.merge(pl_zm[(g - 1) * kTileTokens + rloc], pl_zs[(g - 1) * kTileTokens + rloc]);
                }
                mbar_arrive(list_empty);
            }

            const int row = tile * kTileTokens + rloc;
            int *hist = want_tiles ? hist_tile + (it & 1) * Nr : hist_total;
            if constexpr (Z) {
                if (row < T) {
                    const float l = lse.m + logf(lse.s);
                    zacc += l * l;
                }
            }
            if (row < T) {
                float sum = 0.0f;
#pragma unroll
                for (int k = 0; k < K; ++k) sum += tk.score[k];
                const float inv = 1.0f / sum;
                int32_t *oi = topk_idx + (size_t)row * K;
                float *og = gates + (size_t)row * K;
                if constexpr (K % 4 == 0) {
#pragma unroll
                    for (int k = 0; k < K; k += 4) {
                        *reinterpret_cast<int4 *>(oi + k) = make_int4(tk.idx[k], tk.idx[k + 1], tk.idx[k + 2],
                                                                      tk.idx[k + 3]);
                        *reinterpret_cast<float4 *>(og + k) =
                            make_float4(tk.score[k] * inv, tk.score[k + 1] * inv, tk.score[k + 2] * inv,
                                        tk.score[k + 3] * inv);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < K; ++k) {
                        oi[k] = tk.idx[k];
                        og[k] = tk.score[k] * inv;
                    }
                }
                bool unfilled = false;
#pragma unroll
                for (int k = 0; k < K; ++k) {  // only a NaN or -inf key can leave a slot unfilled
                    if ((unsigned)tk.idx[k] < (unsigned)Nr)
                        atomicAdd(&hist[tk.idx[k]], 1);
                    else
                        unfilled = true;
                }
                if (unfilled) atomicOr(status, kStNonfinite);
            }
            if (want_tiles) {
                mbar_arrive(epi_sync);
                if (!mbar_wait(epi_sync, sync_ph, abort_flag)) {
                    ok = false;
                    break;
                }
                sync_ph ^= 1u;
                const bool real_tile = tile < num_tiles;  // a pair's odd tile can lie past T
                for (int e = rloc; e < Nr; e += 128) {
                    const int v = hist[e];
                    if (real_tile) tile_counts[(size_t)tile * Nr + e] = v;
                    hist_total[e] += v;
                    hist[e] = 0;
                }
            }
        }
        if (group == 0) {
            if (ok) {
                mbar_arrive(epi_sync);
                ok = mbar_wait(epi_sync, sync_ph, abort_flag);
            }
            if (ok) {
                for (int e = rloc; e < Nr; e += 128)
                    if (hist_total[e] != 0) atomicAdd(&counts[e], hist_total[e]);
                if constexpr (Z) {  // one fp64 atomic per warp
                    double z = (double)zacc;
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
                    if (lane == 0) atomicAdd(zloss_sum, z);
                }
            }
        }
        if (!ok) {
            atomicOr(status, kStTimeout);
            *abort_flag = 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // neither CTA leaves while the pair may still touch it
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, tcols);
    }
}

// Epilogue groups: 2 (8 warps, 2 per SM sub-partition) whenever the experts split
// into 32-column halves.  Measured on the tie workload, 8 epilogue warps keep up
// with the MMAs and leave more issue slots to the TMA and MMA warps than 16.
int groups_for(int Nr) { return (Nr % 64 == 0) ? 2 : 1; }

int stages_for(int Nr, int K, int G, int E) {
    const size_t budget = 232448;  // max dynamic shared memory per CTA on sm_100
    int s = kMaxStages;
    while (s > 2 && 1024 + misc_layout(Nr, K, G, s, E).total > budget) --s;
    return s;
}

// Per device and kernel instantiation: the largest dynamic shared-memory size
// granted so far (the attribute is a limit, so it only ever grows), and per
// shared-memory size the number of co-resident clusters.  Set up on first use
// only, so that later launches (for instance inside a CUDA graph capture)
// issue nothing but the launch itself.
struct SmemGrant {
    const void *kern;
    int device;
    size_t smem;
};
struct ClusterFit {
    const void *kern;
    int device;
    size_t smem;
    int clusters;
};
std::mutex g_setup_mu;
SmemGrant g_grant[128];
int g_num_grant = 0;
ClusterFit g_fit[256];
int g_num_fit = 0;

cudaError_t launch_setup(const void *kern, size_t smem, cudaLaunchConfig_t *cfg, int *clusters) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    int gi = -1;
    for (int i = 0; i < g_num_grant; ++i)
        if (g_grant[i].kern == kern && g_grant[i].device == dev) gi = i;
    if (gi < 0 || g_grant[gi].smem < smem) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        if (gi >= 0)
            g_grant[gi].smem = smem;
        else if (g_num_grant < 128)
            g_grant[g_num_grant++] = {kern, dev, smem};
    }
    for (int i = 0; i < g_num_fit; ++i)
        if (g_fit[i].kern == kern && g_fit[i].device == dev && g_fit[i].smem == smem) {
            *clusters = g_fit[i].clusters;
            return cudaSuccess;
        }
    int active = 0;  // clusters that fit on the device at once
    if (cudaOccupancyMaxActiveClusters(&active, kern, cfg) != cudaSuccess) active = 0;
    (void)cudaGetLastError();
    if (g_num_fit < 256) g_fit[g_num_fit++] = {kern, dev, smem, active};
    *clusters = active;
    return cudaSuccess;
}

template <int K, int G>
cudaError_t launch_kg(const CUtensorMap &th, const CUtensorMap &tw, const float *bias, int T, int d, int Nr,
                      int32_t *idx, float *gates, int32_t *counts, int32_t *tile_counts, double *zloss_sum,
                      float *tile_psum, int32_t *status, int num_sms, cudaStream_t stream) {
    const int E = (zloss_sum ? kOptZloss : 0) | (tile_psum ? kOptBalance : 0);
    void (*kern)(CUtensorMap, CUtensorMap, const float *, int, int, int, int, int32_t *, float *, int32_t *,
                 int32_t *, double *, float *, int32_t *);
    switch (E) {
        case kOptZloss: kern = router_gemm_kernel<K, G, kOptZloss>; break;
        case kOptBalance: kern = router_gemm_kernel<K, G, kOptBalance>; break;
        case kOptZloss | kOptBalance: kern = router_gemm_kernel<K, G, kOptZloss | kOptBalance>; break;
        default: kern = router_gemm_kernel<K, G, 0>; break;
    }
    const int stages = stages_for(Nr, K, G, E);
    const size_t smem = 1024 + misc_layout(Nr, K, G, stages, E).total;
    const int num_tiles = (T + kTileTokens - 1) / kTileTokens;
    const int num_work = (num_tiles + kPair - 1) / kPair;
    int units = num_sms / kPair;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kPair;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.blockDim = dim3(threads_of(G), 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.gridDim = dim3(kPair * units, 1, 1);
    int active = 0;
    cudaError_t err = launch_setup(reinterpret_cast<const void *>(kern), smem, &cfg, &active);
    if (err != cudaSuccess) return err;
    if (active > 0 && active < units) units = active;
    if (units > num_work) units = num_work;
    cfg.gridDim = dim3(kPair * units, 1, 1);
    err = cudaLaunchKernelEx(&cfg, kern, th, tw, bias, T, d, Nr, stages, idx, gates, counts, tile_counts, zloss_sum,
                             tile_psum, status);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

template <int K>
cudaError_t launch_k(const CUtensorMap &th, const CUtensorMap &tw, const float *bias, int T, int d, int Nr,
                     int32_t *idx, float *gates, int32_t *counts, int32_t *tile_counts, double *zl, float *psum,
                     int32_t *status, int num_sms, cudaStream_t stream) {
    switch (groups_for(Nr)) {
        case 2:
            return launch_kg<K, 2>(th, tw, bias, T, d, Nr, idx, gates, counts, tile_counts, zl, psum, status, num_sms,
                                   stream);
        default:
            return launch_kg<K, 1>(th, tw, bias, T, d, Nr, idx, gates, counts, tile_counts, zl, psum, status, num_sms,
                                   stream);
    }
}

}  // namespace

int router_gemm_w_box_rows(int Nr) { return Nr / kPair; }

cudaError_t launch_router_gemm(const CUtensorMap &tmap_h, const CUtensorMap &tmap_w, const float *bias, int T,
                               int d, int Nr, int K, int32_t *topk_idx, float *gates, int32_t *counts,
                               int32_t *tile_counts, double *zloss_sum, float *tile_psum, int32_t *status,
                               int num_sms, cudaStream_t stream) {
    switch (K) {
#define EBL_CASE(KK) \
    case KK:         \
        return launch_k<KK>(tmap_h, tmap_w, bias, T, d, Nr, topk_idx, gates, counts, tile_counts, zloss_sum, \
                             tile_psum, status, num_sms, stream);
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
}

}  // namespace ebl
