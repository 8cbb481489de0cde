/*
 * ebl.h -- C ABI of libebl.so: the MoE router step with aux-loss-free
 * expert-bias balancing (SMEBU), hand-written CUDA for sm_100a (B200).
 *
 * The method (page titles, sections and equations):
 *   "Arcee Trinity Large Technical Report", section 2.3 "Mixture-of-Experts":
 *     sigmoid routing with normalized scores; Top-K on routing score plus
 *     expert bias; gates from the routing scores without the bias; SMEBU
 *     with lambda = 5e-4, beta = 0.5, kappa = 2; the sign update of the
 *     smaller models; a linear unclamped update as an ablation.
 *   "SMEBU Load Balancing" (study note), "How it works": eq. (17) bias only
 *     inside Top-K; eqs. (20)-(22) sign update with re-centred bias;
 *     eqs. (23)-(28) normalised violation, tanh clamp, scaled and re-centred
 *     step, momentum, bias add; the sequence-wise balance loss, eqs.
 *     (29)-(32), with alpha = 5e-5 (named, not printed: see
 *     router_forward_balance for the reading).
 *   "Arcee Halts 400B Blackwell Model Collapse With Dynamic Router Biases",
 *     "The MaxVio Metric and the Day-4 Crisis": MaxVio, the ratio of the most-
 *     to the least-routed expert's load; and the stabilization table of
 *     "Precision Fallbacks, Loss Stabilization, and MaxVio as Data Telemetry":
 *     the z-loss log^2 sum_i e^{x_i}, an auxiliary balance loss per sequence.
 *
 * Conventions shared by every entry point:
 *   - Pointers marked "device" are CUDA device pointers (or managed memory) on
 *     the current device.  The caller owns every buffer; the library keeps no
 *     pointer after a call returns and allocates no device memory.
 *   - bf16 data is passed as uint16_t bit patterns (IEEE binary32 upper half).
 *   - All arrays are dense row-major, innermost index last.
 *   - Every call is asynchronous on `stream` (NULL = legacy default stream)
 *     and never synchronises.  Host-side argument checks run before anything
 *     is launched; a call that returns an error launched nothing, except
 *     EBL_ECUDA, which reports a launch failure.
 *   - Return value: EBL_OK (0) or a negative error code (ebl_strerror()).
 *   - T == 0 (no tokens) is a no-op that launches nothing (moe_dispatch zeroes
 *     offsets); the buffers whose size is proportional to T may then be NULL.
 *   - Errors only visible on the device (an expert id out of range, a sum of
 *     loads of zero, a pipeline wait that ran out) are OR-ed into the optional
 *     device word `status` as EBL_ST_* bits; kernels never trap.  With
 *     status == NULL they go to a library-owned device word that
 *     ebl_read_internal_status() reads.
 */
#ifndef EBL_H
#define EBL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st *ebl_stream_t;

/* Return codes. */
#define EBL_OK 0
#define EBL_EINVAL (-1)       /* null pointer, bad shape or size, misaligned pointer */
#define EBL_EUNSUPPORTED (-2) /* valid request this build does not implement (e.g. N_r % 32 != 0 in GEMM mode) */
#define EBL_ECUDA (-3)        /* a CUDA runtime/driver call failed; the CUDA error is cleared */
#define EBL_EDATA (-4)        /* reserved for data errors reported synchronously */

/* Bits of the device status word. */
#define EBL_ST_BAD_EXPERT 1   /* an expert id outside [0, N_r) was seen; that pair was skipped */
#define EBL_ST_BAD_DEST 2     /* a dest index outside [0, T*K) was seen; that slot was skipped */
#define EBL_ST_EMPTY_LOAD 4   /* sum of loads was 0: bias/momentum left untouched */
#define EBL_ST_TIMEOUT 8      /* a pipeline wait (router kernel, dispatch copy) ran out; outputs invalid */
#define EBL_ST_BAD_COUNTS 16  /* dispatch: tile_counts do not add up to T*K (they do not match topk_idx) */
#define EBL_ST_NONFINITE 32   /* ebl_check_finite_*: a NaN or infinity was found; routers: a Top-K slot
                                 stayed unfilled (only a NaN or -inf key can cause that) */

#define EBL_MAX_EXPERTS 256   /* N_r limit of every entry point */
#define EBL_MAX_TOPK 8        /* K limit */

/* Human-readable text for a return code. Never NULL. */
const char *ebl_strerror(int code);

/* Library version, major*10000 + minor*100 + patch. */
int ebl_version(void);

/* The last CUDA failure behind an EBL_ECUDA return on the calling thread, as
 * "call: reason" text ("none" if there was none).  Never NULL; valid until the
 * next library call on this thread. */
const char *ebl_last_cuda_error(void);

/* Tokens per router tile: the row count of one tile_counts row (128). */
int ebl_tile_tokens(void);

/*
 * router_forward -- one router pass in GEMM mode.
 * Passage: "Arcee Trinity Large Technical Report" 2.3 (sigmoid routing with
 * normalized scores; Top-K on score plus bias; gates without the bias) and
 * "SMEBU Load Balancing" eq. (17).
 *
 * For every token t < T:
 *   x_{t,i}  = sum_k hidden[t,k] * W_router[i,k]     bf16 x bf16, fp32 accumulate (tensor cores)
 *   s_{t,i}  = 1 / (1 + exp(-x_{t,i}))               fp32
 *   key      = s_{t,i} + bias[i]                      fp32, bias used only here
 *   topk_idx[t, 0..K-1] = the K experts of largest key; equal keys go to the
 *                         lower expert index; slots sorted by (key desc, index asc)
 *   gates[t,k] = s_{t,idx_k} / sum_k' s_{t,idx_k'}   (bias-free, sums to 1)
 *   counts[i] += #{(t,k) : topk_idx[t,k] == i}        ACCUMULATED: the caller zeroes
 *                                                     counts once per optimizer step
 *   tile_counts[j, i] = the same count over tokens [128 j, 128 j + 128)  (overwritten)
 *
 * hidden       device, bf16 [T, d]; 16-byte aligned.
 * W_router     device, bf16 [N_r, d] (expert-major, i.e. K-major for the MMA); 16-byte aligned.
 * bias         device, fp32 [N_r].
 * T            tokens, 0 <= T <= 2^31 - 2^8.  T == 0 is a no-op.
 * d            hidden size, d % 64 == 0, 64 <= d <= 2^20.
 * N_r          routed experts, N_r % 32 == 0, 32 <= N_r <= 256 (else EBL_EUNSUPPORTED).
 * K            experts per token, 1 <= K <= min(8, N_r).
 * topk_idx     device, int32 [T, K], written.
 * gates        device, fp32 [T, K], written.
 * counts       device, int32 [N_r], accumulated with one atomic per expert per CTA.
 * tile_counts  device, int32 [ceil(T/128), N_r], written; or NULL to skip.
 * status       device int32 or NULL; EBL_ST_TIMEOUT if the pipeline stalled.
 * Inputs are assumed finite (ebl_check_finite_* can vouch for them).  If a
 * NaN logit or a -inf bias leaves fewer than K experts with a key above -inf,
 * the unfilled slots get expert id 0x7fffffff, add no load, and
 * EBL_ST_NONFINITE is raised in status.  Deterministic: the outputs do not depend on
 * scheduling (integer histogram, per-row arithmetic in a fixed order).
 */
int router_forward(const uint16_t *hidden, const uint16_t *W_router, const float *bias,
                   int T, int d, int N_r, int K,
                   int32_t *topk_idx, float *gates, int32_t *counts, int32_t *tile_counts,
                   int32_t *status, ebl_stream_t stream);

/*
 * router_forward_zloss -- router_forward that also accumulates the router
 * z-loss statistic  zloss_sum += sum_{t<T} (log sum_i exp(x_{t,i}))^2  into a
 * caller-zeroed fp64 device scalar (one atomic per epilogue warp per CTA).
 * The z-loss, L_z = log^2 sum_i e^{x_i} per token, is named in "Arcee Halts
 * 400B Blackwell Model Collapse With Dynamic Router Biases" ("Precision
 * Fallbacks, Loss Stabilization, and MaxVio as Data Telemetry", stabilization
 * table); "Arcee Trinity Large Technical Report" section 6 gives its weight
 * (1e-4 intended, 1e-6 effective).  The mean z-loss is zloss_sum / T.  The
 * log-sum-exp is formed from the fp32 logits around the row maximum (no
 * overflow).  zloss_sum: device, 8-byte aligned, not NULL.  The per-warp
 * partial sums meet in fp64 atomics, so the last bits of zloss_sum can vary
 * between runs with the order in which CTAs finish; indices, gates and counts
 * stay deterministic.  Other arguments and outputs as router_forward.
 */
int router_forward_zloss(const uint16_t *hidden, const uint16_t *W_router, const float *bias,
                         int T, int d, int N_r, int K,
                         int32_t *topk_idx, float *gates, int32_t *counts, int32_t *tile_counts,
                         double *zloss_sum, int32_t *status, ebl_stream_t stream);

/*
 * router_forward_balance -- router_forward that also writes the per-tile
 * statistics of the sequence-wise balance loss (and, if zloss_sum is not
 * NULL, accumulates the z-loss statistic as router_forward_zloss does):
 *   tile_psum[j, i] = sum over tokens t in [128 j, 128 j + 128), t < T, of
 *                     s_{t,i} / sum_l s_{t,l}       (all N_r experts, no bias)
 * next to tile_counts[j, i] (required here).  "SMEBU Load Balancing" ("How it
 * works") keeps a small sequence-wise balance loss, eqs. (29)-(32), with
 * coefficient alpha; the pages do not print it, and it is read as the
 * complementary sequence-wise balance loss of auxiliary-loss-free balancing
 * (see seq_balance_loss).  The sums run in fp32 over the fp32 scores of the
 * epilogue in a fixed order (deterministic); rows past T add nothing.
 * tile_counts  device, int32 [ceil(T/128), N_r], written, not NULL.
 * tile_psum    device, fp32 [ceil(T/128), N_r], written, not NULL.
 * zloss_sum    device fp64 scalar (8-byte aligned, accumulated) or NULL.
 * Other arguments and outputs as router_forward.
 */
int router_forward_balance(const uint16_t *hidden, const uint16_t *W_router, const float *bias,
                           int T, int d, int N_r, int K,
                           int32_t *topk_idx, float *gates, int32_t *counts, int32_t *tile_counts,
                           float *tile_psum, double *zloss_sum, int32_t *status, ebl_stream_t stream);

/*
 * balance_stats_logits -- the per-tile statistics of the sequence-wise balance
 * loss in logits mode (a separate pass over the logits):
 *   tile_psum[j, i] = sum over tokens t in [128 j, 128 j + 128), t < T, of
 *                     s_{t,i} / sum_l s_{t,l}
 * with s = (float)(1 / (1 + exp(-(double)x))), the logits-mode score of
 * router_forward_logits.  Row totals and the sums run in fp64 in a fixed
 * order and are rounded once to fp32, so each output is within one fp32
 * rounding of the exact value.  Pair it with the tile_counts of
 * router_forward_logits and call seq_balance_loss.  Passage as for
 * router_forward_balance.
 * logits     device, fp32 [T, N_r], 4-byte aligned (assumed finite).
 * T          tokens, 0 <= T <= 2^31 - 2^8; T == 0 is a no-op.
 * N_r        1 <= N_r <= 256.
 * tile_psum  device, fp32 [ceil(T/128), N_r], written.
 */
int balance_stats_logits(const float *logits, int T, int N_r, float *tile_psum, ebl_stream_t stream);

/*
 * seq_balance_loss -- the sequence-wise balance loss from the per-tile
 * statistics of router_forward_balance (GEMM mode) or of
 * router_forward_logits and balance_stats_logits (logits mode).  For each sequence b of seq_len
 * consecutive tokens (B = T / seq_len sequences, S = seq_len):
 *   f_i = N_r / (K S) * (selections of expert i in the sequence)
 *   P_i = (1 / S) * sum_t s_{t,i} / sum_l s_{t,l}
 *   loss_seq[b] = alpha * sum_i f_i P_i           fp64
 *   *loss = (1 / B) * sum_b loss_seq[b]           fp64, the batch value
 * Passage: "SMEBU Load Balancing", "How it works" (the loss, eqs. (29)-(32),
 * alpha = 5e-5 on the Large checkpoint); "Arcee Halts 400B Blackwell Model
 * Collapse With Dynamic Router Biases", stabilization table (balancing
 * evaluated per sequence).  The formula is a reading: the complementary
 * sequence-wise balance loss published with auxiliary-loss-free balancing.
 * Only the forward value is computed.
 * tile_counts, tile_psum  device, [T/128, N_r] as router_forward_balance wrote them.
 * T           tokens, a multiple of seq_len; T == 0 is a no-op.
 * N_r, K      as for the router call that produced the statistics.
 * seq_len     tokens per sequence, a positive multiple of 128.
 * alpha       the coefficient (finite).
 * loss_seq    device, fp64 [B], written (8-byte aligned).
 * loss        device, fp64 scalar, written (8-byte aligned).
 * Deterministic (fixed-order sums).  Two launches on `stream`.
 */
int seq_balance_loss(const int32_t *tile_counts, const float *tile_psum, int T, int N_r, int K, int seq_len,
                     float alpha, double *loss_seq, double *loss, ebl_stream_t stream);

/*
 * router_forward_logits -- the same selection, gates and counts from
 * precomputed fp32 logits.  This is the bit-exact mode: each value that
 * decides a selection has one defined rounding,
 *   s   = (float)(1 / (1 + exp(-(double)x)))        fp64 evaluation, rounded once
 *   key = s + bias[i]                                one fp32 add, round to nearest
 *   g_k = (float)((double)s_k / sum_k' (double)s_k')  fp64, slot order, rounded once
 * so indices, counts and tile_counts match any implementation of these
 * formulas exactly (up to a last-ulp difference between two fp64 exp
 * implementations, about one value in 2^28).
 *
 * logits  device, fp32 [T, N_r], 4-byte aligned.  With N_r % 4 == 0 and a
 *         16-byte aligned base the logits are read from HBM once; otherwise
 *         a slower kernel reads them twice (same results).
 * N_r     1 <= N_r <= 256 (any value).  K: 1 <= K <= min(8, N_r).
 * Other arguments as router_forward.  Logits and bias are assumed finite;
 * a Top-K slot that no key fills is reported as for router_forward
 * (id 0x7fffffff, no load, EBL_ST_NONFINITE).
 */
int router_forward_logits(const float *logits, const float *bias, int T, int N_r, int K,
                          int32_t *topk_idx, float *gates, int32_t *counts, int32_t *tile_counts,
                          int32_t *status, ebl_stream_t stream);

/*
 * router_forward_logits_balance -- router_forward_logits that also writes the
 * per-tile statistics of the sequence-wise balance loss in the same pass over
 * the logits (read from HBM once):
 *   tile_psum[j, i] = sum over tokens t in [128 j, 128 j + 128), t < T, of
 *                     s_{t,i} / sum_l s_{t,l}       (all N_r experts, no bias)
 * next to tile_counts (required here); pair them with seq_balance_loss.
 * Passage and reading as for router_forward_balance.  Indices, gates, counts
 * and tile_counts are those of router_forward_logits, bit for bit.  The
 * statistics use the fast fp32 score 1 / (1 + exp(-x)) (hardware exp2 and
 * reciprocal approximations), not the rounded-once score that decides the
 * selection: the loss is a training signal, not a selection, so one defined
 * rounding is not needed there.  Each output is within 2^-16 relative (plus
 * 2^-60 absolute) of the exact sums of the rounded-once scores for
 * |x| <= 40; the sums run in a fixed order, so they are deterministic.  With
 * N_r % 4 != 0 or a base address that is not 16-byte aligned, the routing
 * runs in the row kernel and the statistics in a second pass that uses the
 * fp64 score of balance_stats_logits (same tolerance or better).
 * tile_counts  device, int32 [ceil(T/128), N_r], written, not NULL.
 * tile_psum    device, fp32 [ceil(T/128), N_r], written, not NULL.
 * Other arguments as router_forward_logits.
 */
int router_forward_logits_balance(const float *logits, const float *bias, int T, int N_r, int K,
                                  int32_t *topk_idx, float *gates, int32_t *counts, int32_t *tile_counts,
                                  float *tile_psum, int32_t *status, ebl_stream_t stream);

/*
 * smebu_step -- one SMEBU update of the expert bias, once per optimizer step.
 * Passage: "SMEBU Load Balancing", "How it works", eqs. (23)-(28).
 *   nbar = sum_j n_j / N_r
 *   v_i  = (nbar - n_i) / nbar;  db_i = lambda * tanh(kappa * v_i)
 *   db_i -= (1/N_r) sum_j db_j      (summed in index order)
 *   m_i  = beta * m_i + (1 - beta) * db_i;  b_i += m_i
 * Arithmetic is fp64 with IEEE rounding and no contraction; bias and momentum
 * are fp32 state, read widened and stored rounded to nearest.
 *
 * counts       device, int32 [N_r]: the loads n_i of this step (router_forward output).
 * bias         device, fp32 [N_r], updated in place.
 * momentum     device, fp32 [N_r], updated in place (persistent buffer, starts at 0).
 * lambda, beta, kappa   5e-4, 0.5, 2 in the report.
 * reset_counts nonzero: counts is zeroed after it is read, ready for the next step.
 * maxvio_out   device fp32 scalar or NULL: MaxVio = max_i n_i / min_i n_i (+inf if min is 0).
 * status       device int32 or NULL: EBL_ST_EMPTY_LOAD if sum n = 0 (state untouched).
 * One CTA; N_r in [1, 256].
 */
int smebu_step(int32_t *counts, float *bias, float *momentum, int N_r,
               float lambda, float beta, float kappa, int reset_counts,
               float *maxvio_out, int32_t *status, ebl_stream_t stream);

/*
 * smebu_step_layers -- smebu_step for L independent MoE layers in one launch
 * (one bias and momentum vector per layer: "SMEBU Load Balancing" writes b as
 * a vector in R^{N_r} per layer).  counts, bias, momentum are [L, N_r];
 * maxvio_out is [L] or NULL.  linear != 0 selects the linear, unclamped
 * ablation db_i = lambda * v_i ("Arcee Trinity Large Technical Report" 2.3;
 * "SMEBU Load Balancing", last paragraph of "How it works"); kappa is then
 * ignored.  One CTA per layer.
 */
int smebu_step_layers(int32_t *counts, float *bias, float *momentum, int L, int N_r,
                      float lambda, float beta, float kappa, int linear, int reset_counts,
                      float *maxvio_out, int32_t *status, ebl_stream_t stream);

/*
 * sign_update_step -- the aux-loss-free sign update used for the smaller models.
 * Passage: "SMEBU Load Balancing", eqs. (20)-(22).
 *   db_i = gamma * sign(nbar - n_i)   (sign(0) = 0)
 *   b'_i = b_i + db_i;  b_i = b'_i - (1/N_r) sum_j b'_j   (re-centred after the add)
 * fp64 arithmetic on fp32 state.  Arguments as smebu_step.
 */
int sign_update_step(int32_t *counts, float *bias, int N_r, float gamma, int reset_counts,
                     float *maxvio_out, int32_t *status, ebl_stream_t stream);

/*
 * moe_dispatch -- expert-sorted, deterministic token dispatch.
 * The pages name expert parallelism but give no mechanism; this is the plain
 * stable counting sort of the (token, slot) pairs by expert.
 *   pairs p = t*K + k, expert e = topk_idx[t,k]
 *   offsets[0] = 0, offsets[e+1] = offsets[e] + n_e                (int32 [N_r+1])
 *   j = offsets[e] + #{p' < p : topk_idx flat[p'] == e}             (stable, by p)
 *   perm[j] = t;  dest[p] = j;  dispatched[j, :] = hidden[t, :]     (bit copy)
 *
 * hidden       device, bf16 [T, d], 16-byte aligned, d % 8 == 0.
 * topk_idx     device, int32 [T, K].
 * tile_counts  device int32 [ceil(T/128), N_r] from the same router pass, or
 *              NULL (the per-tile histogram is then computed here).
 * offsets      device int32 [N_r + 1]; perm, dest device int32 [T*K];
 * dispatched   device bf16 [T*K, d], 16-byte aligned.
 * workspace    device scratch of at least ebl_dispatch_workspace_bytes(T, N_r)
 *              bytes, 16-byte aligned; contents on entry are ignored.
 * status       EBL_ST_BAD_EXPERT if an id is outside [0, N_r): that pair is
 *              skipped and its dest is -1.  EBL_ST_BAD_COUNTS if the given
 *              tile_counts do not add up to T*K; destinations that would fall
 *              outside [0, T*K) are then skipped (dest -1), others are not
 *              meaningful.  EBL_ST_TIMEOUT if a row copy did not complete
 *              within the bounded wait (dispatched rows are then not valid).
 *              Nothing is written outside the output buffers.
 * The rows move by TMA bulk copies through shared memory (one read of each
 * hidden row, one write per destination).  T*K <= 2^31 - 1.
 */
size_t ebl_dispatch_workspace_bytes(int T, int N_r);
int moe_dispatch(const uint16_t *hidden, const int32_t *topk_idx, const int32_t *tile_counts,
                 int T, int d, int N_r, int K,
                 int32_t *offsets, int32_t *perm, int32_t *dest, uint16_t *dispatched,
                 void *workspace, size_t workspace_bytes, int32_t *status, ebl_stream_t stream);

/*
 * moe_dispatch_static -- moe_dispatch without a workspace argument; it
 * allocates nothing.  The pages have no counterpart to this entry point: it
 * exists for callers that cannot call cudaMalloc to provide the dispatch
 * scratch, for example a plugin whose host framework owns every device byte
 * through its own memory pool and gives the plugin no allocator, or a runtime
 * that forbids device allocation once it has started serving.
 *
 * The scratch lives in one library-owned device array of
 * EBL_DISPATCH_STATIC_SCRATCH_BYTES (4 MiB), which every GPU that loads the
 * library holds until the process exits.  A problem fits when
 * ebl_dispatch_workspace_bytes(T, N_r) <= 4 MiB, i.e. T <= 508288 tokens at
 * N_r = 256 or T <= 2033536 at N_r = 64; larger problems return EBL_EINVAL
 * and launch nothing (use moe_dispatch with a caller workspace for them).
 *
 * All calls share that one array.  Calls whose kernels overlap on the GPU
 * (different streams, or different host threads on one device) race on it
 * and corrupt each other's results; serialise them on one stream.  The array
 * keeps the last call's contents, which the next call overwrites before
 * reading, so no clearing is needed between calls.
 *
 * The first call on each device does a one-time set-up with that device
 * current (it looks up the array's device address); make that first call
 * before any stream capture.  The call makes no cudaMalloc, cudaFree or other
 * allocating call.
 *
 * Arguments, outputs and status bits are those of moe_dispatch.  With
 * status == NULL, device-side error bits go to a library word nobody reads.
 */
#define EBL_DISPATCH_STATIC_SCRATCH_BYTES (4u << 20)
int moe_dispatch_static(const uint16_t *hidden, const int32_t *topk_idx, const int32_t *tile_counts,
                        int T, int d, int N_r, int K,
                        int32_t *offsets, int32_t *perm, int32_t *dest, uint16_t *dispatched,
                        int32_t *status, ebl_stream_t stream);

/*
 * moe_combine -- gate-weighted un-permute of the expert outputs.
 *   out[t, :] = sum_{k=0..K-1} gates[t,k] * expert_out[dest[t*K+k], :]
 * accumulated in fp32 in slot order as acc = fmaf(g, (float)y, acc) from 0,
 * so the result is deterministic (no atomics) and bit-reproducible.
 *
 * expert_out   device, bf16 [T*K, d], 16-byte aligned, d % 8 == 0.
 * gates        device, fp32 [T, K];  dest device, int32 [T*K] (moe_dispatch output).
 * out          device, fp32 [T, d], 16-byte aligned, overwritten.
 * status       EBL_ST_BAD_DEST if a dest is outside [0, T*K): that slot adds nothing.
 */
int moe_combine(const uint16_t *expert_out, const float *gates, const int32_t *dest,
                int T, int d, int K, float *out, int32_t *status, ebl_stream_t stream);

/*
 * ebl_selftest_wait_timeout -- failure-detection self-test.  Launches one
 * thread that waits, through the same bounded mbarrier wait the router kernel
 * uses for its pipeline, on a barrier nothing ever arrives on.  After
 * limit_us microseconds (1 .. 1e6) the wait gives up and EBL_ST_TIMEOUT is
 * OR-ed into *status (device int32); the kernel then returns and the CUDA
 * context stays usable.  No counterpart on the pages: it exists so that the
 * timeout path is exercised without faulting or hanging a GPU.
 */
int ebl_selftest_wait_timeout(int32_t *status, unsigned int limit_us, ebl_stream_t stream);

/*
 * ebl_selftest_score_error -- checks the approximation router_forward_logits
 * ranks with.  That mode scores every expert with an approximate sigmoid
 * (0.5 + 0.5 tanh(x/2), one tanh.approx.f32) and evaluates the exact score
 * only for experts whose approximate key is within a bound of the K-th
 * largest; the bound must exceed the approximation's error.  This call writes
 *   *max_err = max_i | approx(x_i) - (float)(1 / (1 + exp(-(double)x_i))) |
 * (device fp32, 4-byte aligned) and, if bound is not NULL, the absolute error
 * bound the ranking assumes to *bound (host).  If exact_out is not NULL
 * (device fp32 [n]) it receives the exact scores (float)(1/(1+exp(-(double)x_i)))
 * as this library computes them, so that they can be compared with another
 * fp64 implementation.  x: device fp32 [n], n >= 0.
 * No counterpart on the pages: it tests an implementation assumption.
 */
int ebl_selftest_score_error(const float *x, int64_t n, float *max_err, float *bound, float *exact_out,
                             ebl_stream_t stream);

/*
 * ebl_check_finite_f32 / ebl_check_finite_bf16 -- input validation.  The
 * router assumes finite logits, hidden states and bias; these scan n values
 * (device, 4-byte aligned for fp32, 2-byte for bf16) and OR EBL_ST_NONFINITE
 * into *status (device int32, not NULL) if any is NaN or +-inf.  One read of
 * the buffer; asynchronous on the stream.  No counterpart on the pages.
 */
int ebl_check_finite_f32(const float *x, int64_t n, int32_t *status, ebl_stream_t stream);
int ebl_check_finite_bf16(const uint16_t *x, int64_t n, int32_t *status, ebl_stream_t stream);

/*
 * ebl_read_internal_status -- copy the library-owned status word (used when a
 * call passed status == NULL) of the current device to *out, and clear it if
 * `clear` is nonzero.  Synchronous (waits for the device).
 */
int ebl_read_internal_status(int32_t *out, int clear);

#ifdef __cplusplus
}
#endif

#endif /* EBL_H */
