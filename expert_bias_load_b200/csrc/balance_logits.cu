// balance_logits.cu -- the per-tile statistics of the sequence-wise balance
// loss in logits mode:
//   tile_psum[j, i] = sum over tokens t of tile j (128 tokens, t < T) of
//                     s_t,i / sum_l s_t,l
// with s the logits-mode score, fp64 sigmoid rounded once to fp32 (the value
// router_forward_logits ranks and gates with).  The pages name the loss
// ("SMEBU Load Balancing", "How it works", eqs. (29)-(32)) but do not print
// it; it is read as the complementary sequence-wise balance loss of
// auxiliary-loss-free balancing, whose P_i needs these sums.
//
// One pass over the logits per tile, in four parts of 32 rows: the warps score
// the part's rows (row-major, coalesced; each lane scores its up to 8 columns
// together), keep the scores in shared memory and total each row in fp64
// (fixed lane order, then a fixed shuffle tree); then thread i walks the
// part's rows in order and adds s_t,i / total_t in fp64.
// The fp64 sums are rounded once to fp32 on the way out, so each output is
// within an fp32 rounding of the exact sum.  Deterministic.  The cost is the
// fp64 sigmoid of every score (the logits-mode router evaluates it only for
// the few candidates of each row), not the HBM read.

#include "launch.h"
#include "scores.cuh"

namespace ebl {
namespace {

constexpr int kBalThreads = 256;  // >= N_r: one thread per expert in the column pass
constexpr int kPartRows = 32;  // rows scored per pass; 32 KB of scores at N_r = 256

__global__ void __launch_bounds__(kBalThreads) tile_psum_logits_kernel(const float *__restrict__ logits, int T,
                                                                       int Nr, float *__restrict__ tile_psum) {
    extern __shared__ float s_sm[];  // [kPartRows][Nr] scores of the current part of the tile
    __shared__ double inv_sm[kPartRows];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_tiles = (T + kTileTokens - 1) / kTileTokens;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        double acc = 0.0;  // thread i: expert i
        for (int part = 0; part < kTileTokens / kPartRows; ++part) {
            const int r0 = tile * kTileTokens + part * kPartRows;
            for (int r = warp; r < kPartRows; r += kBalThreads / 32) {
                const int row = r0 + r;
                double tot = 0.0;
                if (row < T) {
                    // the lane's (up to 8) columns are loaded and scored together,
                    // so their fp64 exponentials overlap
                    const float *x = logits + (size_t)row * Nr;
                    float xv[kMaxExperts / 32];
#pragma unroll
                    for (int k = 0; k < kMaxExperts / 32; ++k) {
                        const int c = lane + 32 * k;
                        xv[k] = c < Nr ? x[c] : 0.0f;
                    }
                    const int chunks = (Nr + 31) / 32;  // warp-uniform
                    float sv[kMaxExperts / 32];
#pragma unroll
                    for (int k = 0; k < kMaxExperts / 32; ++k) sv[k] = k < chunks ? sigmoid_rounded_once(xv[k]) : 0.0f;
#pragma unroll
                    for (int k = 0; k < kMaxExperts / 32; ++k) {
                        const int c = lane + 32 * k;
                        if (c < Nr) {
                            s_sm[r * Nr + c] = sv[k];
                            tot += (double)sv[k];
                        }
                    }
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, off);
                if (lane == 0) inv_sm[r] = (row < T && tot > 0.0) ? 1.0 / tot : 0.0;
            }
            __syncthreads();
            const int rows = min(kPartRows, T - r0);
            if ((int)threadIdx.x < Nr)
                for (int r = 0; r < rows; ++r) acc += (double)s_sm[r * Nr + threadIdx.x] * inv_sm[r];
            __syncthreads();
        }
        if ((int)threadIdx.x < Nr) tile_psum[(size_t)tile * Nr + threadIdx.x] = (float)acc;
    }
}

}  // namespace

cudaError_t launch_tile_psum_logits(const float *logits, int T, int Nr, float *tile_psum, int num_sms,
                                    cudaStream_t stream) {
    const int num_tiles = (T + kTileTokens - 1) / kTileTokens;
    const size_t smem = (size_t)kPartRows * Nr * sizeof(float);  // at most 32 KB
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tile_psum_logits_kernel, kBalThreads, smem) !=
            cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    (void)cudaGetLastError();
    int grid = num_sms * per_sm;
    if (grid > num_tiles) grid = num_tiles;
    tile_psum_logits_kernel<<<grid, kBalThreads, smem, stream>>>(logits, T, Nr, tile_psum);
    return cudaGetLastError();
}

}  // namespace ebl
