/*
 * ebl_oracle.c -- TEST INFRASTRUCTURE, not part of the product.
 *
 * A plain, slow, single-purpose CPU statement of the MoE router step with
 * aux-loss-free expert-bias balancing and the SMEBU bias update, written from
 * the pages that describe the method so that the CUDA library can be checked
 * against it.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg load this code.  It shares nothing with the CUDA library: no
 * header, no helper, no table.  Its only common ground with that library is
 * the seeded input data the tests hand to both.
 *
 * Arithmetic is fp64 unless a function says otherwise.  Loops run in the
 * obvious order; the only concession to speed is an OpenMP pragma over
 * independent tokens (the per-token arithmetic is unchanged by it).
 *
 * Sources (page title, section / equation):
 *   [TR]    "Arcee Trinity Large Technical Report" (paper summary),
 *           section 2.3 "Mixture-of-Experts": sigmoid routing with normalized
 *           scores; Top-K on routing score plus expert bias; gates from the
 *           routing scores without the bias; lambda=5e-4, beta=0.5, kappa=2.
 *   [SN]    "SMEBU Load Balancing" (study note), "How it works":
 *           eq. (17) bias only inside Top-K; eqs. (20)-(22) sign update with
 *           re-centred b; eqs. (23)-(24) normalised violation and tanh clamp;
 *           eqs. (25)-(28) scaled step, re-centred step, momentum, bias add.
 *   [TALK]  "Arcee Halts 400B Blackwell Model Collapse With Dynamic Router
 *           Biases", section "The MaxVio Metric and the Day-4 Crisis":
 *           MaxVio = load of the most-routed expert / load of the least-routed.
 *   [BLOG]  "trinity-large-moe-routing-load-balancing" (blog post), section on
 *           sigmoid routing and Top-K: scores are per-expert dot products
 *           u_t . e_i passed through a sigmoid.
 *
 * Readings taken where the pages are silent or disagree (each also listed in
 * the design notes):
 *   - the bias is added to the sigmoid score, not to the logit ([SN] eq. 17
 *     writes s_{i,t}+b_i; [BLOG] says otherwise and is not followed);
 *   - ties in Top-K go to the lower expert index; output slots are in the
 *     order (key descending, index ascending);
 *   - gates are g = s / (sum of s over the selected experts), scale 1;
 *   - a "load" n_i counts (token, slot) assignments, so sum n = K*T;
 *   - the sign update re-centres b after adding the step;
 *   - MaxVio is +inf when some expert received no load;
 *   - the sequence-wise balance loss, which the pages name but do not print,
 *     is the complementary sequence-wise loss of auxiliary-loss-free
 *     balancing (four equations, as the pages' numbering (29)-(32) suggests),
 *     averaged over the sequences of a batch.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EINVAL (-1)
#define ORC_EDATA (-4)

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static double bf16_to_f64(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* sum_k a[k] * b[k * b_stride] over k < d, exact bf16 products summed in fp64. */
static double dot_bf16(const uint16_t *a, const uint16_t *b, int64_t b_stride, int d)
{
    double acc = 0.0;
    for (int k = 0; k < d; ++k) acc += bf16_to_f64(a[k]) * bf16_to_f64(b[k * b_stride]);
    return acc;
}

/* The sigmoid router score s = 1 / (1 + exp(-x))  ([TR] 2.3; [BLOG]). */
static double sigmoid_f64(double x)
{
    return 1.0 / (1.0 + exp(-x));
}

/*
 * Top-K under the total order "larger key first, lower index first on equal
 * keys".  Plain repeated selection of the best remaining expert: K passes over
 * the n keys.  `taken` is caller scratch of n bytes.
 */
static void topk_f64(const double *key, int n, int K, unsigned char *taken, int32_t *out)
{
    memset(taken, 0, (size_t)n);
    for (int k = 0; k < K; ++k) {
        int best = -1;
        for (int i = 0; i < n; ++i) {
            if (taken[i]) continue;
            if (best < 0 || key[i] > key[best]) best = i; /* equal keys keep the lower index */
        }
        taken[best] = 1;
        out[k] = best;
    }
}

static void topk_f32(const float *key, int n, int K, unsigned char *taken, int32_t *out)
{
    memset(taken, 0, (size_t)n);
    for (int k = 0; k < K; ++k) {
        int best = -1;
        for (int i = 0; i < n; ++i) {
            if (taken[i]) continue;
            if (best < 0 || key[i] > key[best]) best = i;
        }
        taken[best] = 1;
        out[k] = best;
    }
}

/*
 * Router step, GEMM mode, in fp64.
 *   x_{t,i} = sum_k h_{t,k} W_{i,k}   (router projection, u_t . e_i)
 *   s_{t,i} = sigmoid(x_{t,i})
 *   key     = s_{t,i} + b_i            (bias only inside Top-K, [SN] eq. 17)
 *   idx     = Top-K of key
 *   g_{t,k} = s_{t,idx_k} / sum_k' s_{t,idx_k'}   (bias-free, [TR] 2.3)
 *   n_i    += number of (t,k) with idx_{t,k} = i
 *
 * hidden: bf16 bits [T,d] row-major; W: bf16 bits [Nr,d] row-major;
 * bias: fp32 [Nr].  Outputs: idx int32 [T,K]; gates fp64 [T,K];
 * counts int64 [Nr] (ACCUMULATED); optional: logits fp64 [T,Nr], scores fp64
 * [T,Nr], gap fp64 [T] = key of slot K minus best unselected key (+inf when
 * K == Nr).
 */
int orc_router_gemm(const uint16_t *hidden, const uint16_t *W, const float *bias,
                    int64_t T, int d, int Nr, int K,
                    int32_t *idx, double *gates, int64_t *counts,
                    double *logits_out, double *scores_out, double *gap_out)
{
    if (T < 0 || d <= 0 || Nr <= 0 || K <= 0 || K > Nr) return ORC_EINVAL;
#pragma omp parallel
    {
        double *x = (double *)malloc(sizeof(double) * (size_t)Nr);
        double *s = (double *)malloc(sizeof(double) * (size_t)Nr);
        double *key = (double *)malloc(sizeof(double) * (size_t)Nr);
        unsigned char *taken = (unsigned char *)malloc((size_t)Nr);
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            const uint16_t *h = hidden + t * (int64_t)d;
            for (int i = 0; i < Nr; ++i) {
                x[i] = dot_bf16(h, W + (int64_t)i * d, 1, d); /* u_t . e_i */
                s[i] = sigmoid_f64(x[i]);
                key[i] = s[i] + (double)bias[i];
            }
            int32_t *sel = idx + t * K;
            topk_f64(key, Nr, K, taken, sel);
            double sum = 0.0;
            for (int k = 0; k < K; ++k) sum += s[sel[k]];
            for (int k = 0; k < K; ++k) gates[t * K + k] = s[sel[k]] / sum;
            if (gap_out) {
                double best_rest = -INFINITY;
                for (int i = 0; i < Nr; ++i)
                    if (!taken[i] && key[i] > best_rest) best_rest = key[i];
                gap_out[t] = (K == Nr) ? INFINITY : key[sel[K - 1]] - best_rest;
            }
            if (logits_out) memcpy(logits_out + t * Nr, x, sizeof(double) * (size_t)Nr);
            if (scores_out) memcpy(scores_out + t * Nr, s, sizeof(double) * (size_t)Nr);
        }
        free(x);
        free(s);
        free(key);
        free(taken);
    }
    for (int64_t p = 0; p < T * K; ++p) counts[idx[p]] += 1;
    return ORC_OK;
}

/*
 * Router step, logits mode (the bit-exact contract).  The input is fp32
 * logits; every value that decides a selection is fixed to one rounding:
 *   s_f32   = (float)(1 / (1 + exp(-(double)x)))   (fp64, rounded once)
 *   key_f32 = s_f32 + b_f32                         (one fp32 add, nearest)
 *   g       = (float)((double)s_k / sum_k' (double)s_k')  sum in slot order
 * Outputs as in orc_router_gemm, but gates are fp32; optional scores fp32
 * [T,Nr] and tile_counts int32 [ceil(T/tile), Nr] (tile = tile_tokens rows).
 */
int orc_router_logits(const float *logits, const float *bias, int64_t T, int Nr, int K,
                      int32_t *idx, float *gates, int64_t *counts,
                      float *scores_out, int32_t *tile_counts, int tile_tokens)
{
    if (T < 0 || Nr <= 0 || K <= 0 || K > Nr) return ORC_EINVAL;
#pragma omp parallel
    {
        float *s = (float *)malloc(sizeof(float) * (size_t)Nr);
        float *key = (float *)malloc(sizeof(float) * (size_t)Nr);
        unsigned char *taken = (unsigned char *)malloc((size_t)Nr);
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            const float *x = logits + t * Nr;
            for (int i = 0; i < Nr; ++i) {
                s[i] = (float)sigmoid_f64((double)x[i]);
                key[i] = s[i] + bias[i]; /* one binary32 add, nearest */
            }
            int32_t *sel = idx + t * K;
            topk_f32(key, Nr, K, taken, sel);
            double sum = 0.0;
            for (int k = 0; k < K; ++k) sum += (double)s[sel[k]];
            for (int k = 0; k < K; ++k) gates[t * K + k] = (float)((double)s[sel[k]] / sum);
            if (scores_out) memcpy(scores_out + t * Nr, s, sizeof(float) * (size_t)Nr);
        }
        free(s);
        free(key);
        free(taken);
    }
    for (int64_t p = 0; p < T * K; ++p) counts[idx[p]] += 1;
    if (tile_counts && tile_tokens > 0) {
        int64_t tiles = (T + tile_tokens - 1) / tile_tokens;
        memset(tile_counts, 0, sizeof(int32_t) * (size_t)(tiles * Nr));
        for (int64_t p = 0; p < T * K; ++p) tile_counts[(p / K / tile_tokens) * Nr + idx[p]] += 1;
    }
    return ORC_OK;
}

/*
 * Router z-loss statistic: sum over tokens of (log sum_i exp(x_{t,i}))^2, the
 * per-token term of L_z = log^2 sum_i e^{x_i} ([TALK], "Precision Fallbacks,
 * Loss Stabilization, and MaxVio as Data Telemetry", stabilization table;
 * weights in [TR] section 6).  fp64; the log-sum-exp is taken around the row
 * maximum so that large logits do not overflow.  Same inputs as
 * orc_router_gemm.
 */
double orc_router_zloss(const uint16_t *hidden, const uint16_t *W, int64_t T, int d, int Nr)
{
    double total = 0.0;
    double *x = (double *)malloc(sizeof(double) * (size_t)Nr);
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t *h = hidden + t * (int64_t)d;
        double mx = -INFINITY;
        for (int i = 0; i < Nr; ++i) {
            const double xi = dot_bf16(h, W + (int64_t)i * d, 1, d);
            x[i] = xi;
            if (xi > mx) mx = xi;
        }
        double sum = 0.0;
        for (int i = 0; i < Nr; ++i) sum += exp(x[i] - mx);
        const double lse = mx + log(sum);
        total += lse * lse;
    }
    free(x);
    return total;
}

/*
 * Sequence-wise balance loss, the small auxiliary term kept beside the bias
 * balancing.  [SN] "How it works" names it (eqs. (29)-(32), coefficient
 * alpha, 5e-5 on the Large checkpoint) and calls it a within-sequence nudge;
 * [TALK]'s stabilization table describes it as auxiliary load balancing
 * evaluated per sequence.  The pages do not print the four equations.
 * Reading: the complementary sequence-wise balance loss published with
 * auxiliary-loss-free balancing (DeepSeek-V3 technical report, section
 * 2.1.2), whose four equations are, for one sequence of S tokens:
 *   f_i    = N_r / (K * S) * #{(t,k) in the sequence : idx_{t,k} = i}
 *   s'_t,i = s_t,i / sum_j s_t,j        (all N_r experts, no bias)
 *   P_i    = (1 / S) * sum_t s'_t,i
 *   L      = alpha * sum_i f_i * P_i
 * A batch of T tokens holds T / S consecutive sequences; its value is the
 * mean of their L.
 * scores: fp64 [T,Nr], the sigmoid scores of the router step; idx: int32
 * [T,K].  Optional outputs f [B,Nr], P [B,Nr], loss_seq [B]; *loss the mean.
 */
int orc_seq_balance(const double *scores, const int32_t *idx, int64_t T, int Nr, int K, int64_t S,
                    double alpha, double *f_out, double *p_out, double *loss_seq, double *loss)
{
    if (T <= 0 || Nr <= 0 || K <= 0 || K > Nr || S <= 0 || T % S != 0) return ORC_EINVAL;
    for (int64_t p = 0; p < T * K; ++p)
        if (idx[p] < 0 || idx[p] >= Nr) return ORC_EDATA;
    const int64_t B = T / S;
    double *f = (double *)malloc(sizeof(double) * (size_t)Nr);
    double *P = (double *)malloc(sizeof(double) * (size_t)Nr);
    double total = 0.0;
    for (int64_t b = 0; b < B; ++b) {
        for (int i = 0; i < Nr; ++i) {
            f[i] = 0.0;
            P[i] = 0.0;
        }
        for (int64_t t = b * S; t < (b + 1) * S; ++t) {
            for (int k = 0; k < K; ++k) f[idx[t * K + k]] += 1.0;
            const double *s = scores + t * Nr;
            double row = 0.0;
            for (int j = 0; j < Nr; ++j) row += s[j];
            for (int i = 0; i < Nr; ++i) P[i] += s[i] / row;
        }
        double l = 0.0;
        for (int i = 0; i < Nr; ++i) {
            f[i] *= (double)Nr / ((double)K * (double)S);
            P[i] /= (double)S;
            l += f[i] * P[i];
        }
        l *= alpha;
        if (f_out) memcpy(f_out + b * Nr, f, sizeof(double) * (size_t)Nr);
        if (p_out) memcpy(p_out + b * Nr, P, sizeof(double) * (size_t)Nr);
        if (loss_seq) loss_seq[b] = l;
        total += l;
    }
    free(f);
    free(P);
    *loss = total / (double)B;
    return ORC_OK;
}

/*
 * The per-tile pieces of the same loss, for tiles of `tile` consecutive tokens
 * (the last one ragged): psum[j,i] = sum over the tile's tokens t of
 * s_t,i / sum_l s_t,l.
 */
int orc_tile_psum(const double *scores, int64_t T, int Nr, int tile, double *psum)
{
    if (T < 0 || Nr <= 0 || tile <= 0) return ORC_EINVAL;
    const int64_t tiles = (T + tile - 1) / tile;
    memset(psum, 0, sizeof(double) * (size_t)(tiles * Nr));
    for (int64_t t = 0; t < T; ++t) {
        const double *s = scores + t * Nr;
        double row = 0.0;
        for (int l = 0; l < Nr; ++l) row += s[l];
        for (int i = 0; i < Nr; ++i) psum[(t / tile) * Nr + i] += s[i] / row;
    }
    return ORC_OK;
}

/*
 * The loss from per-tile loads and per-tile sums of normalised scores
 * (tile_counts [T/tile, Nr] as the router writes them, psum as above), with
 * S a multiple of tile: the same f_i, P_i and L as orc_seq_balance, each
 * sequence's loads and sums gathered from its S / tile tiles.
 */
int orc_seq_balance_tiles(const int32_t *tile_counts, const double *psum, int64_t T, int Nr, int K, int64_t S,
                          int tile, double alpha, double *loss_seq, double *loss)
{
    if (T <= 0 || Nr <= 0 || K <= 0 || K > Nr || S <= 0 || tile <= 0 || T % S != 0 || S % tile != 0)
        return ORC_EINVAL;
    const int64_t B = T / S, per = S / tile;
    double total = 0.0;
    for (int64_t b = 0; b < B; ++b) {
        double l = 0.0;
        for (int i = 0; i < Nr; ++i) {
            double n = 0.0, q = 0.0;
            for (int64_t j = b * per; j < (b + 1) * per; ++j) {
                n += (double)tile_counts[j * Nr + i];
                q += psum[j * Nr + i];
            }
            const double fi = (double)Nr / ((double)K * (double)S) * n;
            const double Pi = q / (double)S;
            l += fi * Pi;
        }
        l *= alpha;
        if (loss_seq) loss_seq[b] = l;
        total += l;
    }
    *loss = total / (double)B;
    return ORC_OK;
}

/*
 * MaxVio ([TALK]): load of the most-routed expert divided by the load of the
 * least-routed one, in fp64.  +inf when the least-routed expert got nothing.
 */
double orc_maxvio(const int64_t *counts, int Nr, int64_t *max_out, int64_t *min_out)
{
    int64_t mx = counts[0], mn = counts[0];
    for (int i = 1; i < Nr; ++i) {
        if (counts[i] > mx) mx = counts[i];
        if (counts[i] < mn) mn = counts[i];
    }
    if (max_out) *max_out = mx;
    if (min_out) *min_out = mn;
    if (mn == 0) return INFINITY;
    return (double)mx / (double)mn;
}

/*
 * SMEBU, one optimizer step ([SN] eqs. (23)-(28); constants from [TR] 2.3).
 *   nbar   = (sum_j n_j) / Nr
 *   v_i    = (nbar - n_i) / nbar                       (23)
 *   vt_i   = tanh(kappa * v_i)                          (24)
 *   db_i   = lambda * vt_i                              (25)
 *   db_i  -= (1/Nr) sum_j db_j   (sum in index order)   (26)
 *   m_i    = beta * m_i + (1 - beta) * db_i             (27)
 *   b_i    = b_i + m_i                                  (28)
 * The state b, m is fp32 (read as fp64, the step done in fp64, stored rounded
 * to nearest).  Hyper-parameters arrive as fp32 and are widened exactly.
 * Returns ORC_EDATA and leaves the state untouched when sum n == 0.
 * maxvio_out (may be NULL) receives MaxVio of the counts, rounded to fp32.
 */
int orc_smebu(const int64_t *counts, float *bias, float *momentum, int Nr,
              float lambda_f, float beta_f, float kappa_f, float *maxvio_out)
{
    if (Nr <= 0) return ORC_EINVAL;
    const double lambda = lambda_f, beta = beta_f, kappa = kappa_f;
    int64_t total = 0;
    for (int i = 0; i < Nr; ++i) total += counts[i];
    if (maxvio_out) *maxvio_out = (float)orc_maxvio(counts, Nr, NULL, NULL);
    if (total <= 0) return ORC_EDATA;
    const double nbar = (double)total / (double)Nr;
    double *db = (double *)malloc(sizeof(double) * (size_t)Nr);
    for (int i = 0; i < Nr; ++i) {
        double v = (nbar - (double)counts[i]) / nbar;
        double vt = tanh(kappa * v);
        db[i] = lambda * vt;
    }
    double sum = 0.0;
    for (int i = 0; i < Nr; ++i) sum += db[i];
    const double mean = sum / (double)Nr;
    for (int i = 0; i < Nr; ++i) {
        double d = db[i] - mean;
        double m = beta * (double)momentum[i] + (1.0 - beta) * d;
        double b = (double)bias[i] + m;
        momentum[i] = (float)m;
        bias[i] = (float)b;
    }
    free(db);
    return ORC_OK;
}

/*
 * Linear, unclamped variant mentioned as an ablation ([TR] 2.3, [SN] last
 * paragraph of "How it works"): db_i = lambda * v_i instead of
 * lambda * tanh(kappa * v_i); the rest of (26)-(28) is unchanged.
 */
int orc_smebu_linear(const int64_t *counts, float *bias, float *momentum, int Nr,
                     float lambda_f, float beta_f, float *maxvio_out)
{
    if (Nr <= 0) return ORC_EINVAL;
    const double lambda = lambda_f, beta = beta_f;
    int64_t total = 0;
    for (int i = 0; i < Nr; ++i) total += counts[i];
    if (maxvio_out) *maxvio_out = (float)orc_maxvio(counts, Nr, NULL, NULL);
    if (total <= 0) return ORC_EDATA;
    const double nbar = (double)total / (double)Nr;
    double *db = (double *)malloc(sizeof(double) * (size_t)Nr);
    for (int i = 0; i < Nr; ++i) db[i] = lambda * ((nbar - (double)counts[i]) / nbar);
    double sum = 0.0;
    for (int i = 0; i < Nr; ++i) sum += db[i];
    const double mean = sum / (double)Nr;
    for (int i = 0; i < Nr; ++i) {
        double m = beta * (double)momentum[i] + (1.0 - beta) * (db[i] - mean);
        double b = (double)bias[i] + m;
        momentum[i] = (float)m;
        bias[i] = (float)b;
    }
    free(db);
    return ORC_OK;
}

/*
 * Aux-loss-free sign update of the smaller models ([SN] eqs. (20)-(22)):
 *   db_i = gamma * sign(nbar - n_i)          sign(0) = 0
 *   b'_i = b_i + db_i
 *   b_i  = b'_i - (1/Nr) sum_j b'_j          (re-centred after the add)
 * fp64 arithmetic on the fp32 state, stored rounded to nearest.
 */
int orc_sign_update(const int64_t *counts, float *bias, int Nr, float gamma_f, float *maxvio_out)
{
    if (Nr <= 0) return ORC_EINVAL;
    const double gamma = gamma_f;
    int64_t total = 0;
    for (int i = 0; i < Nr; ++i) total += counts[i];
    if (maxvio_out) *maxvio_out = (float)orc_maxvio(counts, Nr, NULL, NULL);
    if (total <= 0) return ORC_EDATA;
    const double nbar = (double)total / (double)Nr;
    double *bp = (double *)malloc(sizeof(double) * (size_t)Nr);
    for (int i = 0; i < Nr; ++i) {
        double diff = nbar - (double)counts[i];
        double sgn = (diff > 0.0) ? 1.0 : ((diff < 0.0) ? -1.0 : 0.0);
        bp[i] = (double)bias[i] + gamma * sgn;
    }
    double sum = 0.0;
    for (int i = 0; i < Nr; ++i) sum += bp[i];
    const double mean = sum / (double)Nr;
    for (int i = 0; i < Nr; ++i) bias[i] = (float)(bp[i] - mean);
    free(bp);
    return ORC_OK;
}

/*
 * Expert-sorted dispatch.  The T*K (token, slot) pairs p = t*K + k are
 * grouped by expert, stably in p order:
 *   offsets[0] = 0, offsets[e+1] = offsets[e] + n_e
 *   walking p = 0 .. T*K-1:  j = offsets[e] + (pairs of expert e seen so far)
 *   perm[j] = t,  dest[p] = j
 * Returns ORC_EDATA if some expert id is outside [0, Nr).
 */
int orc_dispatch(const int32_t *idx, int64_t T, int K, int Nr,
                 int32_t *offsets, int32_t *perm, int32_t *dest)
{
    const int64_t P = T * K;
    for (int64_t p = 0; p < P; ++p)
        if (idx[p] < 0 || idx[p] >= Nr) return ORC_EDATA;
    int64_t *fill = (int64_t *)calloc((size_t)Nr, sizeof(int64_t));
    for (int64_t p = 0; p < P; ++p) fill[idx[p]] += 1;
    offsets[0] = 0;
    for (int e = 0; e < Nr; ++e) offsets[e + 1] = offsets[e] + (int32_t)fill[e];
    memset(fill, 0, sizeof(int64_t) * (size_t)Nr);
    for (int64_t p = 0; p < P; ++p) {
        int e = idx[p];
        int64_t j = offsets[e] + fill[e];
        fill[e] += 1;
        perm[j] = (int32_t)(p / K);
        dest[p] = (int32_t)j;
    }
    free(fill);
    return ORC_OK;
}

/* The gathered rows: X[j,:] = hidden[perm[j],:], bit for bit. */
void orc_gather_rows(const uint16_t *hidden, const int32_t *perm, int64_t rows, int d, uint16_t *X)
{
    for (int64_t j = 0; j < rows; ++j)
        memcpy(X + j * d, hidden + (int64_t)perm[j] * d, sizeof(uint16_t) * (size_t)d);
}

/*
 * Combine: out[t,:] = sum_k g_{t,k} * Y[dest[t*K+k],:].
 *   out64 (may be NULL): the sum in fp64, k in slot order.
 *   out32 (may be NULL): the fp32 statement, acc = 0; acc = fmaf(g, y, acc)
 *   for k = 0..K-1, i.e. one rounding per slot.
 */
int orc_combine(const uint16_t *Y, const float *gates, const int32_t *dest,
                int64_t T, int d, int K, int64_t rows_Y, double *out64, float *out32)
{
    for (int64_t p = 0; p < T * K; ++p)
        if (dest[p] < 0 || dest[p] >= rows_Y) return ORC_EDATA;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int c = 0; c < d; ++c) {
            double a64 = 0.0;
            float a32 = 0.0f;
            for (int k = 0; k < K; ++k) {
                const int64_t row = dest[t * K + k];
                const double y = bf16_to_f64(Y[row * d + c]);
                const float g = gates[t * K + k];
                a64 += (double)g * y;
                a32 = fmaf(g, (float)y, a32);
            }
            if (out64) out64[t * d + c] = a64;
            if (out32) out32[t * d + c] = a32;
        }
    }
    return ORC_OK;
}
