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
// Design (one persistent CTA per SM, warp-specialised):
//   warp 4      TMA producer: 128x64 hidden tile + N_r x 64 W tile per stage,
//               128-byte swizzle, into a ring of `stages` shared-memory slots.
//   warp 5      TMEM owner and MMA issuer: tcgen05.mma M=128, N=N_r, K=16,
//               fp32 accumulator in TMEM, two accumulator buffers so the
//               epilogue of tile i overlaps the MMAs of tile i+1.
//   warps 0-3   epilogue: warp q reads TMEM lanes 32q..32q+31 (one token row
//               per thread) 32 columns at a time, and runs sigmoid, +bias,
//               Top-K, gates, output stores and a shared-memory histogram.
// The logits never leave TMEM.  Counts reach global memory with one atomic per
// expert per CTA at the end; tile_counts with one store per expert per tile.
// Every pipeline wait is bounded (EBL_ST_TIMEOUT, then a clean exit).

#include "launch.h"
#include "ptx.cuh"
#include "topk.cuh"

namespace ebl {
namespace {

constexpr int kBlockK = 64;  // hidden elements per stage: one 128-byte swizzle row
constexpr int kUmmaK = 16;   // K of one kind::f16 MMA
constexpr int kEpiWarps = 4;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 192;
constexpr int kMaxStages = 8;
constexpr uint32_t kATileBytes = kTileTokens * kBlockK * 2;  // 16 KiB

__host__ __device__ inline uint32_t b_tile_bytes(int Nr) { return (uint32_t)Nr * kBlockK * 2; }

__host__ __device__ inline uint32_t tmem_columns(int Nr) {
    uint32_t need = 2u * (uint32_t)Nr, c = 32;
    while (c < need) c <<= 1;
    return c;
}

// Byte offset of the small-object region (barriers, flags, bias, histograms).
__host__ __device__ inline size_t misc_offset(int Nr, int stages) {
    return (size_t)stages * (kATileBytes + b_tile_bytes(Nr));
}

__host__ __device__ inline size_t misc_bytes(int Nr, int stages) {
    // full[S], empty[S], tfull[2], tempty[2], epi_sync, drain (8 B each);
    // tmem slot + abort flag + pad (16 B); bias, hist_total, hist_tile[2] (4 Nr each)
    return (size_t)(2 * stages + 6) * 8 + 16 + (size_t)4 * Nr * 4;
}

__device__ __forceinline__ bool wait_timed(uint64_t *bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_timer_ns() - t0 > kWaitLimitNs) return false;
    return true;
}

// tcgen05.wait::ld, with the loaded registers tied to it so that no use of
// them can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld_wait_regs(uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;"
        : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
          "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
          "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]),
          "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
          "+r"(r[30]), "+r"(r[31])
        :
        : "memory");
}

template <int K>
__device__ __forceinline__ void consume_chunk(const uint32_t (&r)[32], const float *__restrict__ bias_s, int c,
                                              RowTopK<K> &tk) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const float x = __uint_as_float(r[j]);
        const float s = fast_rcp(1.0f + __expf(-x));
        const float kv = __fadd_rn(s, bias_s[c + j]);
        tk.push(kv, s, c + j);
    }
}

template <int K>
__global__ void __launch_bounds__(kThreads, 1)
    router_gemm_kernel(const __grid_constant__ CUtensorMap tmap_h, const __grid_constant__ CUtensorMap tmap_w,
                       const float *__restrict__ bias, int T, int d, int Nr, int stages,
                       int32_t *__restrict__ topk_idx, float *__restrict__ gates, int32_t *__restrict__ counts,
                       int32_t *__restrict__ tile_counts, int32_t *__restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const uint32_t b_bytes = b_tile_bytes(Nr);
    uint8_t *smA = smem;
    uint8_t *smB = smem + (size_t)stages * kATileBytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + misc_offset(Nr, stages));
    uint64_t *empty = full + stages;
    uint64_t *tfull = empty + stages;
    uint64_t *tempty = tfull + 2;
    uint64_t *epi_sync = tempty + 2;
    uint64_t *drain = epi_sync + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *bias_s = reinterpret_cast<float *>(tmem_slot + 4);
    int *hist_total = reinterpret_cast<int *>(bias_s + Nr);
    int *hist_tile = hist_total + Nr;  // [2][Nr]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_tiles = (T + kTileTokens - 1) / kTileTokens;
    const int num_kb = d / kBlockK;
    const uint32_t tcols = tmem_columns(Nr);

    for (int i = threadIdx.x; i < Nr; i += kThreads) {
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
            mbar_init(&tempty[a], kEpiWarps * 32);
        }
        mbar_init(epi_sync, kEpiWarps * 32);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap_h);
        prefetch_tmap(&tmap_w);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, tcols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == kProducerWarp) {
        if (lane == 0) {
            const uint64_t pol_h = l2_policy_evict_first();  // hidden: read once
            const uint64_t pol_w = l2_policy_evict_last();   // W_router: re-read by every tile
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued = 0, issued_ph = 0;  // per stage: ever issued, parity of last issue
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], kATileBytes + b_bytes);
                    tma_load_2d(smA + (size_t)s * kATileBytes, &tmap_h, &full[s], kb * kBlockK, tile * kTileTokens,
                                pol_h);
                    tma_load_2d(smB + (size_t)s * b_bytes, &tmap_w, &full[s], kb * kBlockK, 0, pol_w);
                    issued |= 1u << s;
                    issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok) {
                atomicOr(status, kStTimeout);
                *abort_flag = 1;
                // let the loads already in flight land before the CTA exits
                for (int t = 0; t < stages; ++t)
                    if (issued & (1u << t)) wait_timed(&full[t], (issued_ph >> t) & 1u);
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kTileTokens, (uint32_t)Nr);
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            int it = 0;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
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
                        umma_bf16(d_tmem, smem_desc_sw128_kmajor(a0 + kk * kUmmaK * 2),
                                  smem_desc_sw128_kmajor(b0 + kk * kUmmaK * 2), idesc, (uint32_t)(kb | kk));
                    }
                    umma_commit(&empty[s]);  // frees the stage once these MMAs have read it
                    if (++s == stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(&tfull[acc]);  // accumulator complete
            }
            if (!ok) {
                atomicOr(status, kStTimeout);
                *abort_flag = 1;
            }
            // every MMA this thread issued has finished once `drain` completes
            umma_commit(drain);
            wait_timed(drain, 0);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const bool want_tiles = tile_counts != nullptr;
        uint32_t sync_ph = 0;
        bool ok = true;
        int it = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
            const int acc = it & 1;
            const uint32_t use = (uint32_t)(it >> 1);
            if (!mbar_wait(&tfull[acc], use & 1u, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();

            RowTopK<K> tk;
            tk.init();
            const uint32_t taddr = tmem_base + lane_base + (uint32_t)(acc * Nr);
            uint32_t ra[32], rb[32];
            __syncwarp();
            tmem_ld_32x32b_x32(taddr, ra);
            tmem_ld_wait_regs(ra);
            for (int c = 0; c < Nr; c += 64) {
                const bool has_b = c + 32 < Nr;
                __syncwarp();
                if (has_b) tmem_ld_32x32b_x32(taddr + (uint32_t)(c + 32), rb);
                consume_chunk<K>(ra, bias_s, c, tk);
                if (has_b) {
                    __syncwarp();
                    tmem_ld_wait_regs(rb);
                    const bool has_a = c + 64 < Nr;
                    if (has_a) tmem_ld_32x32b_x32(taddr + (uint32_t)(c + 64), ra);
                    consume_chunk<K>(rb, bias_s, c + 32, tk);
                    __syncwarp();
                    if (has_a) tmem_ld_wait_regs(ra);
                }
            }
            // accumulator fully read: hand it back to the MMA warp
            tc_fence_before();
            mbar_arrive(&tempty[acc]);

            const int row = tile * kTileTokens + warp * 32 + lane;
            int *hist = want_tiles ? hist_tile + (it & 1) * Nr : hist_total;
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
#pragma unroll
                for (int k = 0; k < K; ++k)  // a non-finite row can leave a slot unfilled
                    if ((unsigned)tk.idx[k] < (unsigned)Nr) atomicAdd(&hist[tk.idx[k]], 1);
            }
            if (want_tiles) {
                mbar_arrive(epi_sync);
                if (!mbar_wait(epi_sync, sync_ph, abort_flag)) {
                    ok = false;
                    break;
                }
                sync_ph ^= 1u;
                for (int e = threadIdx.x; e < Nr; e += kEpiWarps * 32) {
                    const int v = hist[e];
                    tile_counts[(size_t)tile * Nr + e] = v;
                    hist_total[e] += v;
                    hist[e] = 0;
                }
            }
        }
        if (ok) {
            mbar_arrive(epi_sync);
            ok = mbar_wait(epi_sync, sync_ph, abort_flag);
        }
        if (ok) {
            for (int e = threadIdx.x; e < Nr; e += kEpiWarps * 32)
                if (hist_total[e] != 0) atomicAdd(&counts[e], hist_total[e]);
        } else {
            atomicOr(status, kStTimeout);
            *abort_flag = 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tcols);
    }
}

template <int K>
cudaError_t launch_k(const CUtensorMap &th, const CUtensorMap &tw, const float *bias, int T, int d, int Nr,
                     int32_t *idx, float *gates, int32_t *counts, int32_t *tile_counts, int32_t *status,
                     int num_sms, cudaStream_t stream) {
    const int stages = router_gemm_stages(Nr);
    const size_t smem = router_gemm_smem_bytes(Nr, stages);
    cudaError_t err =
        cudaFuncSetAttribute(router_gemm_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const int num_tiles = (T + kTileTokens - 1) / kTileTokens;
    const int grid = num_tiles < num_sms ? num_tiles : num_sms;
    router_gemm_kernel<K><<<grid, kThreads, smem, stream>>>(th, tw, bias, T, d, Nr, stages, idx, gates, counts,
                                                           tile_counts, status);
    return cudaGetLastError();
}

}  // namespace

int router_gemm_stages(int Nr) {
    const size_t budget = 232448;  // max dynamic shared memory per CTA on sm_100
    int s = kMaxStages;
    while (s > 2 && router_gemm_smem_bytes(Nr, s) > budget) --s;
    return s;
}

size_t router_gemm_smem_bytes(int Nr, int stages) {
    return 1024 /* alignment slack */ + misc_offset(Nr, stages) + misc_bytes(Nr, stages);
}

cudaError_t launch_router_gemm(const CUtensorMap &tmap_h, const CUtensorMap &tmap_w, const float *bias, int T,
                               int d, int Nr, int K, int32_t *topk_idx, float *gates, int32_t *counts,
                               int32_t *tile_counts, int32_t *status, int num_sms, cudaStream_t stream) {
    switch (K) {
#define EBL_CASE(KK) \
    case KK:         \
        return launch_k<KK>(tmap_h, tmap_w, bias, T, d, Nr, topk_idx, gates, counts, tile_counts, status, num_sms, stream);
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
