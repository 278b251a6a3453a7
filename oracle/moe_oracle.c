/*
 * moe_oracle.c -- TEST INFRASTRUCTURE, NOT PRODUCT CODE.
 *
 * A plain, slow, obviously-correct CPU restatement of the LongCat-Flash MoE layer with
 * zero-computation experts, in fp64 on exactly-widened bf16 inputs.  Only the test suite,
 * the smoke check and the benchmark's CPU-baseline / reference leg may load this library.
 * It shares no code, header, table or helper with the CUDA library; neither includes the other.
 *
 * Pages cited (title, then section):
 *   P1 = "衝上熱搜！美團大模型，靠「快」火了" (dhxrcw.cn news article)
 *   P2 = CSDN codearts article on LongCat-Flash, sections "一、架构设计" and "二、训练优化"
 *   P4 = "美团的 LongCat-Flash：用 27B 激活算力跑起一个 560B 模型"
 *   P5 = "美团LongCat-Flash：算力调度新纪元", section "技术创新" (figure caption (b))
 *
 * What the layer computes (P1 §零計算專家; the displayed formula itself is missing from the
 * extracted page, so the glossary under it and the prose around it are what we follow):
 *   - the expert pool holds N ordinary FFN experts plus Z zero-computation experts;
 *   - R is a softmax router over the whole pool; b_i is a per-expert bias; K experts are
 *     selected per token;
 *   - the bias steers selection only and stays decoupled from the model's objective, so the
 *     gate weights are the router's softmax outputs, not the biased scores;
 *   - a zero-computation expert returns its input unchanged;
 *   - y_t = sum over the K selected experts of g_i * E_i(x_t).
 * Readings where the pages are silent:
 *   - bias added to the softmax probability p_i (not to the logit); ties -> lower index;
 *   - gates are NOT renormalised over the selected set (renormalisation is an option:
 *     oracle_renormalize_gates);
 *   - an FFN expert is SwiGLU: E(x) = W_d (silu(W_g x) * (W_u x)), silu(z) = z / (1 + e^-z);
 *   - the PID law acts on the mean number of FFN experts per token (see oracle_pid_step),
 *     optionally followed by the per-expert balancing term (oracle_balance_step);
 *   - FP8 (optional): E4M3 weights in 128 x 128 blocks, and optionally E4M3 activations in
 *     1 x 128 blocks, each block with a power-of-two scale (see the FP8 section).
 *
 * Arithmetic: every floating-point step is fp64 except the PID controller, which is fp32 by
 * definition of its state; compile with -ffp-contract=off so no FMA contraction changes it.
 * There is no blocking, fusion or reordering beyond the definition; OpenMP only splits the
 * independent per-token (or per-row) work across threads, which cannot change any result.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* A bf16 bit pattern is the top 16 bits of an IEEE binary32; widening is exact. */
static double bf16_to_f64(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------------------------
 * Router R and biased top-K selection (P1 §零計算專家, glossary under the MoE formula).
 *
 *   l_i = sum_j x_j * W_r[i, j]               (router logits over all E = N + Z experts)
 *   p_i = exp(l_i - max l) / sum_k exp(l_k - max l)     (softmax router R)
 *   s_i = p_i + b_i                           (bias shifts the selection score only)
 *   TopK = K largest s_i; on an exact tie the lower index wins
 *   g_i  = p_i for i in TopK                  (gate = router output, unbiased, unrenormalised)
 *   gap  = s_(K) - s_(K+1)                    (K-th largest minus (K+1)-th largest score)
 *
 * Outputs per token t: topk_idx[t*K + k] in ascending expert id, topk_gate likewise,
 * gap[t] (+INFINITY when E == K), and optionally the full p (probs, T*E) and s (scores, T*E).
 * Selection is K passes of "pick the largest unchosen score, scanning ids upward", i.e.
 * selection sort, kept for its obviousness.
 * ---------------------------------------------------------------------------------------- */
void oracle_router(int64_t T, int64_t d, int64_t E, int64_t K,
                   const uint16_t *x, const uint16_t *W_r, const float *b,
                   int32_t *topk_idx, double *topk_gate, double *gap,
                   double *probs, double *scores)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < T; ++t) {
        double *l = (double *)malloc(sizeof(double) * (size_t)E);
        double *p = (double *)malloc(sizeof(double) * (size_t)E);
        double *s = (double *)malloc(sizeof(double) * (size_t)E);
        char *chosen = (char *)calloc((size_t)E, 1);
        const uint16_t *xt = x + t * d;

        for (int64_t i = 0; i < E; ++i) {
            const uint16_t *wi = W_r + i * d;
            double acc = 0.0;
            for (int64_t j = 0; j < d; ++j)
                acc += bf16_to_f64(xt[j]) * bf16_to_f64(wi[j]);
            l[i] = acc;
        }
        double lmax = l[0];
        for (int64_t i = 1; i < E; ++i)
            if (l[i] > lmax) lmax = l[i];
        double z = 0.0;
        for (int64_t i = 0; i < E; ++i) {
            p[i] = exp(l[i] - lmax);
            z += p[i];
        }
        for (int64_t i = 0; i < E; ++i) {
            p[i] = p[i] / z;
            s[i] = p[i] + (double)b[i];
        }

        /* K passes of selection sort over the biased scores. */
        double kth = INFINITY;
        for (int64_t k = 0; k < K; ++k) {
            int64_t best = -1;
            for (int64_t i = 0; i < E; ++i) {
                if (chosen[i]) continue;
                if (best < 0 || s[i] > s[best]) best = i; /* strict '>' keeps the lower id */
            }
            chosen[best] = 1;
            kth = s[best];
        }
        double next = -INFINITY; /* the (K+1)-th largest score */
        for (int64_t i = 0; i < E; ++i)
            if (!chosen[i] && s[i] > next) next = s[i];
        if (gap) gap[t] = (K < E) ? (kth - next) : INFINITY;

        int64_t k = 0;
        for (int64_t i = 0; i < E; ++i) {
            if (!chosen[i]) continue;
            topk_idx[t * K + k] = (int32_t)i;
            topk_gate[t * K + k] = p[i];
            ++k;
        }
        if (probs)
            for (int64_t i = 0; i < E; ++i) probs[t * E + i] = p[i];
        if (scores)
            for (int64_t i = 0; i < E; ++i) scores[t * E + i] = s[i];
        free(l);
        free(p);
        free(s);
        free(chosen);
    }
}

/* ------------------------------------------------------------------------------------------
 * Dispatch: group the FFN slots by expert (P1 §零計算專家: zero experts need no computation,
 * so only slots with expert id < N are routed to an FFN).  Stable counting sort with key
 * (expert id ascending, then token ascending).
 *
 *   counts[e]        number of slots (t, k) with topk_idx == e, for all E experts
 *   offsets[e]       exclusive prefix of counts over the FFN experts, offsets[N] = A
 *   perm_tok[r]      token of the r-th row of the grouped order, r < A
 *   slot_pos[t*K+k]  row r of that slot, or -1 for a zero-expert slot
 * ---------------------------------------------------------------------------------------- */
void oracle_dispatch(int64_t T, int64_t K, int64_t N, int64_t E, const int32_t *topk_idx,
                     int32_t *counts, int32_t *offsets, int32_t *perm_tok, int32_t *slot_pos)
{
    for (int64_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t k = 0; k < K; ++k) counts[topk_idx[t * K + k]] += 1;
    offsets[0] = 0;
    for (int64_t e = 0; e < N; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1));
    for (int64_t e = 0; e < N; ++e) cursor[e] = offsets[e];
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t k = 0; k < K; ++k) {
            int32_t e = topk_idx[t * K + k];
            if (e < N) {
                int32_t r = cursor[e]++;
                perm_tok[r] = (int32_t)t;
                slot_pos[t * K + k] = r;
            } else {
                slot_pos[t * K + k] = -1;
            }
        }
    }
    free(cursor);
}

static void fp8_round_trip_row(int64_t n, double *v);

/* ------------------------------------------------------------------------------------------
 * One FFN expert on R input rows (P1 §零計算專家 calls them standard FFN experts; the
 * SwiGLU form is the reading taken here):
 *   a = W_g x, u = W_u x        (W_g, W_u: I x d, row-major)
 *   h_f = silu(a_f) * u_f,  silu(z) = z / (1 + exp(-z))
 *   E(x) = W_d h                (W_d: d x I, row-major)
 * ---------------------------------------------------------------------------------------- */
static void swiglu_row(int64_t d, int64_t I, const uint16_t *xr, const uint16_t *W_g,
                       const uint16_t *W_u, const uint16_t *W_d, double *h, double *out)
{
    for (int64_t f = 0; f < I; ++f) {
        double a = 0.0, u = 0.0;
        const uint16_t *wg = W_g + f * d;
        const uint16_t *wu = W_u + f * d;
        for (int64_t j = 0; j < d; ++j) {
            double xj = bf16_to_f64(xr[j]);
            a += bf16_to_f64(wg[j]) * xj;
            u += bf16_to_f64(wu[j]) * xj;
        }
        h[f] = (a / (1.0 + exp(-a))) * u;
    }
    for (int64_t j = 0; j < d; ++j) {
        const uint16_t *wd = W_d + j * I;
        double acc = 0.0;
        for (int64_t f = 0; f < I; ++f) acc += bf16_to_f64(wd[f]) * h[f];
        out[j] = acc;
    }
}

/* The same expert with FP8 activations (an optional variant, used with FP8 weights; see the
 * FP8 section below): the token row is quantised in 1 x 128 blocks and the values q * 2^e enter
 * the up-projection; h is quantised the same way before the down projection.  Everything else
 * is as in swiglu_row, in fp64.  xv holds d doubles of scratch. */
static void swiglu_row_fp8act(int64_t d, int64_t I, const uint16_t *xr, const uint16_t *W_g,
                              const uint16_t *W_u, const uint16_t *W_d, double *xv, double *h,
                              double *out)
{
    for (int64_t j = 0; j < d; ++j) xv[j] = bf16_to_f64(xr[j]);
    fp8_round_trip_row(d, xv);
    for (int64_t f = 0; f < I; ++f) {
        double a = 0.0, u = 0.0;
        const uint16_t *wg = W_g + f * d;
        const uint16_t *wu = W_u + f * d;
        for (int64_t j = 0; j < d; ++j) {
            a += bf16_to_f64(wg[j]) * xv[j];
            u += bf16_to_f64(wu[j]) * xv[j];
        }
        h[f] = (a / (1.0 + exp(-a))) * u;
    }
    fp8_round_trip_row(I, h);
    for (int64_t j = 0; j < d; ++j) {
        const uint16_t *wd = W_d + j * I;
        double acc = 0.0;
        for (int64_t f = 0; f < I; ++f) acc += bf16_to_f64(wd[f]) * h[f];
        out[j] = acc;
    }
}

static void expert_rows(int64_t d, int64_t I, int64_t R, const uint16_t *xrows,
                        const uint16_t *W_g, const uint16_t *W_u, const uint16_t *W_d,
                        double *out, int fp8act)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < R; ++r) {
        double *h = (double *)malloc(sizeof(double) * (size_t)I);
        double *xv = (double *)malloc(sizeof(double) * (size_t)d);
        if (fp8act)
            swiglu_row_fp8act(d, I, xrows + r * d, W_g, W_u, W_d, xv, h, out + r * d);
        else
            swiglu_row(d, I, xrows + r * d, W_g, W_u, W_d, h, out + r * d);
        free(xv);
        free(h);
    }
}

void oracle_swiglu_expert(int64_t d, int64_t I, int64_t R, const uint16_t *xrows,
                          const uint16_t *W_g, const uint16_t *W_u, const uint16_t *W_d,
                          double *out)
{
    expert_rows(d, I, R, xrows, W_g, W_u, W_d, out, 0);
}

/* d and I multiples of 128. */
void oracle_swiglu_expert_fp8act(int64_t d, int64_t I, int64_t R, const uint16_t *xrows,
                                 const uint16_t *W_g, const uint16_t *W_u, const uint16_t *W_d,
                                 double *out)
{
    expert_rows(d, I, R, xrows, W_g, W_u, W_d, out, 1);
}

/* ------------------------------------------------------------------------------------------
 * The whole layer for tokens whose routing is already known (P1 §零計算專家):
 *   y_t = sum_{k < K} g_{t,k} * E_{i_{t,k}}(x_t),   E_i(x) = x for a zero expert (i >= N).
 * Slots are summed in the order given (ascending expert id from oracle_router).
 * Weights are the natural per-expert layouts: W_g, W_u [N][I][d]; W_d [N][d][I].
 * Only tokens listed in `tokens` (n_tok of them) are computed; y has n_tok rows.
 * ---------------------------------------------------------------------------------------- */
static void combine_tokens(int64_t d, int64_t N, int64_t K, int64_t I, int64_t n_tok,
                           const int64_t *tokens, const uint16_t *x, const int32_t *topk_idx,
                           const double *topk_gate, const uint16_t *W_g, const uint16_t *W_u,
                           const uint16_t *W_d, double *y, int fp8act)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n = 0; n < n_tok; ++n) {
        double *h = (double *)malloc(sizeof(double) * (size_t)I);
        double *ffn = (double *)malloc(sizeof(double) * (size_t)d);
        double *xv = (double *)malloc(sizeof(double) * (size_t)d);
        int64_t t = tokens[n];
        const uint16_t *xt = x + t * d;
        double *yt = y + n * d;
        for (int64_t j = 0; j < d; ++j) yt[j] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            int32_t i = topk_idx[t * K + k];
            double g = topk_gate[t * K + k];
            if (i >= N) { /* zero-computation expert: E_i(x) = x */
                for (int64_t j = 0; j < d; ++j) yt[j] += g * bf16_to_f64(xt[j]);
            } else if (fp8act) {
                swiglu_row_fp8act(d, I, xt, W_g + (int64_t)i * I * d, W_u + (int64_t)i * I * d,
                                  W_d + (int64_t)i * d * I, xv, h, ffn);
                for (int64_t j = 0; j < d; ++j) yt[j] += g * ffn[j];
            } else {
                swiglu_row(d, I, xt, W_g + (int64_t)i * I * d, W_u + (int64_t)i * I * d,
                           W_d + (int64_t)i * d * I, h, ffn);
                for (int64_t j = 0; j < d; ++j) yt[j] += g * ffn[j];
            }
        }
        free(xv);
        free(h);
        free(ffn);
    }
}

void oracle_combine_tokens(int64_t d, int64_t N, int64_t K, int64_t I, int64_t n_tok,
                           const int64_t *tokens, const uint16_t *x, const int32_t *topk_idx,
                           const double *topk_gate, const uint16_t *W_g, const uint16_t *W_u,
                           const uint16_t *W_d, double *y)
{
    combine_tokens(d, N, K, I, n_tok, tokens, x, topk_idx, topk_gate, W_g, W_u, W_d, y, 0);
}

/* The same with FP8 activations in the FFN experts (zero experts still return x_t unchanged:
 * no product, nothing to quantise).  d and I multiples of 128. */
void oracle_combine_tokens_fp8act(int64_t d, int64_t N, int64_t K, int64_t I, int64_t n_tok,
                                  const int64_t *tokens, const uint16_t *x,
                                  const int32_t *topk_idx, const double *topk_gate,
                                  const uint16_t *W_g, const uint16_t *W_u, const uint16_t *W_d,
                                  double *y)
{
    combine_tokens(d, N, K, I, n_tok, tokens, x, topk_idx, topk_gate, W_g, W_u, W_d, y, 1);
}

/* ------------------------------------------------------------------------------------------
 * The weighted sum alone, for given expert outputs (P1 §零計算專家):
 *   y_t = sum_{k < K} ( i_{t,k} < N ? rows[slot_pos[t,k]] : g_{t,k} * x_t )
 * where rows[r] already holds g * E_i(x) for grouped row r (the FFN terms arrive gated), and
 * slot_pos maps slot (t, k) to its grouped row.  Slots summed in order, fp64.
 * ---------------------------------------------------------------------------------------- */
void oracle_combine_rows(int64_t T, int64_t d, int64_t N, int64_t K, const uint16_t *x,
                         const int32_t *topk_idx, const double *topk_gate,
                         const int32_t *slot_pos, const double *rows, double *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double *yt = y + t * d;
        for (int64_t j = 0; j < d; ++j) yt[j] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            int32_t i = topk_idx[t * K + k];
            if (i >= N) {
                double g = topk_gate[t * K + k];
                for (int64_t j = 0; j < d; ++j) yt[j] += g * bf16_to_f64(x[t * d + j]);
            } else {
                const double *r = rows + (int64_t)slot_pos[t * K + k] * d;
                for (int64_t j = 0; j < d; ++j) yt[j] += r[j];
            }
        }
    }
}

/* Router, then the layer, for all T tokens. */
void oracle_forward(int64_t T, int64_t d, int64_t N, int64_t Z, int64_t K, int64_t I,
                    const uint16_t *x, const uint16_t *W_r, const float *b, const uint16_t *W_g,
                    const uint16_t *W_u, const uint16_t *W_d, double *y, int32_t *topk_idx,
                    double *topk_gate, double *gap)
{
    int64_t E = N + Z;
    oracle_router(T, d, E, K, x, W_r, b, topk_idx, topk_gate, gap, NULL, NULL);
    int64_t *tokens = (int64_t *)malloc(sizeof(int64_t) * (size_t)(T > 0 ? T : 1));
    for (int64_t t = 0; t < T; ++t) tokens[t] = t;
    oracle_combine_tokens(d, N, K, I, T, tokens, x, topk_idx, topk_gate, W_g, W_u, W_d, y);
    free(tokens);
}

/* ------------------------------------------------------------------------------------------
 * PID controller on the expert biases (P1 §零計算專家, last paragraph: the update rule is a
 * PID controller that tunes the expert biases in real time so the activated parameters per
 * token stay near the ~27B average; P2 §二、训练优化 and P4 §关键要点 say the same;
 * P5 §技术创新 caption (b): the activated experts settle around 8).  The pages give no
 * equation, so this is the plain reading: a single PID loop on the mean number of FFN
 * experts per token, m, against a set-point m*, whose output shifts every FFN expert's bias
 * by the same amount (zero-expert biases stay fixed; only relative scores matter):
 *
 *   m        = (sum_{i<N} counts_i) / T
 *   e        = (m* - m) / K
 *   integral = integral + e
 *   u        = kp*e + ki*integral + kd*(e - e_prev)      (summed left to right)
 *   e_prev   = e
 *   b_i      = b_i + u  for every FFN expert i < N
 *
 * fp32 throughout, one rounding per operation in the order written; state = {integral,
 * e_prev}.  T == 0 leaves everything unchanged.
 * ---------------------------------------------------------------------------------------- */
void oracle_pid_step(int64_t N, int64_t K, int64_t T, const int32_t *counts, float *b,
                     float *state, float target, float kp, float ki, float kd)
{
    if (T <= 0) return;
    int64_t total = 0;
    for (int64_t i = 0; i < N; ++i) total += counts[i];
    float m = (float)total / (float)T;
    float e = (target - m) / (float)K;
    float integral = state[0] + e;
    float p_term = kp * e;
    float i_term = ki * integral;
    float d_term = kd * (e - state[1]);
    float u = (p_term + i_term) + d_term;
    state[0] = integral;
    state[1] = e;
    for (int64_t i = 0; i < N; ++i) b[i] = b[i] + u;
}

/* ------------------------------------------------------------------------------------------
 * Gate renormalisation over the selected set (an optional variant; the layer's default keeps
 * the unrenormalised softmax gate, P1 §零計算專家).  Per token t:
 *
 *   g_k = g_k / sum_{j < K} g_j        (fp64, sum in slot order)
 *
 * The sum runs over all K selected experts, zero-computation ones included, so the weights
 * of every y_t term (identity terms too) add up to one.
 * ---------------------------------------------------------------------------------------- */
void oracle_renormalize_gates(int64_t T, int64_t K, double *topk_gate)
{
    for (int64_t t = 0; t < T; ++t) {
        double sum = 0.0;
        for (int64_t k = 0; k < K; ++k) sum += topk_gate[t * K + k];
        for (int64_t k = 0; k < K; ++k) topk_gate[t * K + k] = topk_gate[t * K + k] / sum;
    }
}

/* ------------------------------------------------------------------------------------------
 * Per-expert balancing term of the aux-loss-free bias scheme that the PID controller
 * modifies (P1 §零計算專家: the expert-specific bias is adjusted from recent expert usage).
 * The pages name the scheme without its rule; this is its published form: after a step,
 * every FFN expert's bias moves by a fixed amount gamma toward the mean load,
 *
 *   c_mean = (sum_{i<N} counts_i) / N
 *   b_i    = b_i + gamma * sign(c_mean - counts_i)     for i < N   (sign(0) = 0)
 *
 * The sign is taken exactly, from the integers: sign(c_mean - c_i) = sign(total - N*c_i).
 * gamma * (+1 | 0 | -1) is exact, so the only rounding is the fp32 add.  Zero-expert biases
 * are unchanged.  When combined with the PID step, the PID step is applied first.
 * ---------------------------------------------------------------------------------------- */
void oracle_balance_step(int64_t N, const int32_t *counts, float *b, float gamma)
{
    int64_t total = 0;
    for (int64_t i = 0; i < N; ++i) total += counts[i];
    for (int64_t i = 0; i < N; ++i) {
        const int64_t diff = total - N * (int64_t)counts[i];
        const float s = diff > 0 ? 1.0f : (diff < 0 ? -1.0f : 0.0f);
        b[i] = b[i] + gamma * s;
    }
}

/* ------------------------------------------------------------------------------------------
 * FP8 block-quantised expert weights (an optional variant).  P1 §系統級優化 says LongCat-Flash
 * quantises with the same fine-grained block-wise scheme as DeepSeek-V3, i.e. one scale per
 * 128 x 128 block of a weight matrix.  Readings taken here (the page gives no format details): the element format is E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
 * no infinities; S.1111.111 is NaN; largest finite 448); each block's scale is the smallest
 * power of two 2^e with max|w| <= 448 * 2^e (a power of two keeps q * 2^e exact in bf16);
 * q = E4M3(w / 2^e) rounded to nearest, ties to even mantissa, saturating at +-448.
 * By default activations stay bf16 (weight-only quantisation).  The FP8-activation variant
 * quantises the inputs of both expert GEMMs too -- the token row x_t and h -- at the activation
 * granularity of the DeepSeek-V3 scheme the page names: one scale per token per 128 consecutive
 * channels (a 1 x 128 block), with the same format and scale rule (reading: the page names the
 * scheme only).
 * ---------------------------------------------------------------------------------------- */
double oracle_e4m3_decode(uint8_t code)
{
    const int s = code >> 7, E = (code >> 3) & 15, M = code & 7;
    if (E == 15 && M == 7) return NAN;
    double v = (E == 0) ? ldexp((double)M, -9) : ldexp(1.0 + M / 8.0, E - 7);
    return s ? -v : v;
}

uint8_t oracle_e4m3_encode(double v)
{
    if (isnan(v)) return 0x7F;
    const uint8_t s = signbit(v) ? 0x80 : 0x00;
    const double a = fabs(v);
    if (a >= 448.0) return (uint8_t)(s | 0x7E);
    if (a < ldexp(1.0, -6)) {                   /* subnormal grid: multiples of 2^-9 */
        const double q = nearbyint(ldexp(a, 9)); /* ties to even under the default mode */
        return (uint8_t)(s | (uint8_t)q);        /* q == 8 is the smallest normal, code 8 */
    }
    int x;
    (void)frexp(a, &x);                          /* a = f * 2^x, f in [0.5, 1) */
    int e = x - 1;                               /* a = m * 2^e, m in [1, 2) */
    double mq = nearbyint((ldexp(a, -e) - 1.0) * 8.0);
    if (mq == 8.0) { mq = 0.0; e += 1; }
    return (uint8_t)(s | (uint8_t)(((e + 7) << 3) | (int)mq));
}

/* The exponent e of a block's scale 2^e: the smallest integer with amax <= 448 * 2^e, at least
 * -126; 0 for an all-zero block. */
static int fp8_scale_exponent(double amax)
{
    int e = 0;
    if (amax > 0.0) {
        e = ilogb(amax) - 8;
        while (amax > ldexp(448.0, e)) ++e;
        while (amax <= ldexp(448.0, e - 1)) --e;
        if (e < -126) e = -126;
    }
    return e;
}

/* Round-to-nearest-even conversion of a double that is exact in fp32 to bf16 bits. */
static uint16_t f64_to_bf16_rne(double v)
{
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40); /* NaN */
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* w: G matrices of [R][C] bf16 (R, C multiples of 128) -> q [G][R][C] E4M3 codes and
 * scale [G][R/128][C/128] fp32 (= 2^e). */
void oracle_quantize_fp8_blocks(int64_t G, int64_t R, int64_t C, const uint16_t *w, uint8_t *q,
                                float *scale)
{
    const int64_t RB = R / 128, CB = C / 128;
#pragma omp parallel for schedule(static)
    for (int64_t gb = 0; gb < G * RB; ++gb) {
        const int64_t g = gb / RB, rb = gb % RB;
        for (int64_t cb = 0; cb < CB; ++cb) {
            double amax = 0.0;
            for (int64_t r = 0; r < 128; ++r)
                for (int64_t c = 0; c < 128; ++c) {
                    const double a = fabs(bf16_to_f64(w[(g * R + rb * 128 + r) * C + cb * 128 + c]));
                    if (a > amax) amax = a;
                }
            const int e = fp8_scale_exponent(amax);
            scale[(g * RB + rb) * CB + cb] = (float)ldexp(1.0, e);
            for (int64_t r = 0; r < 128; ++r)
                for (int64_t c = 0; c < 128; ++c) {
                    const int64_t i = (g * R + rb * 128 + r) * C + cb * 128 + c;
                    q[i] = oracle_e4m3_encode(ldexp(bf16_to_f64(w[i]), -e));
                }
        }
    }
}

/* The weights the FP8 variant computes with: q * scale of its block, as bf16 bits (exact
 * unless the product underflows bf16). */
void oracle_dequantize_fp8_blocks(int64_t G, int64_t R, int64_t C, const uint8_t *q,
                                  const float *scale, uint16_t *w)
{
    const int64_t RB = R / 128, CB = C / 128;
    for (int64_t g = 0; g < G; ++g)
        for (int64_t r = 0; r < R; ++r)
            for (int64_t c = 0; c < C; ++c) {
                const int64_t i = (g * R + r) * C + c;
                const double s = (double)scale[(g * RB + r / 128) * CB + c / 128];
                w[i] = f64_to_bf16_rne(oracle_e4m3_decode(q[i]) * s);
            }
}

/* FP8 activations: v [R][C] (C a multiple of 128) -> q [R][C] E4M3 codes and scale
 * [R][C/128] fp32 (= 2^e), one scale per 1 x 128 block of a row, by the weights' rule. */
void oracle_quantize_fp8_rows(int64_t R, int64_t C, const double *v, uint8_t *q, float *scale)
{
    const int64_t CB = C / 128;
    for (int64_t r = 0; r < R; ++r)
        for (int64_t cb = 0; cb < CB; ++cb) {
            const double *blk = v + r * C + cb * 128;
            double amax = 0.0;
            for (int64_t c = 0; c < 128; ++c)
                if (fabs(blk[c]) > amax) amax = fabs(blk[c]);
            const int e = fp8_scale_exponent(amax);
            scale[r * CB + cb] = (float)ldexp(1.0, e);
            for (int64_t c = 0; c < 128; ++c)
                q[r * C + cb * 128 + c] = oracle_e4m3_encode(ldexp(blk[c], -e));
        }
}

/* v [n] (n a multiple of 128) replaced in place by its FP8-activation value q * 2^e. */
static void fp8_round_trip_row(int64_t n, double *v)
{
    uint8_t *q = (uint8_t *)malloc((size_t)n);
    float *s = (float *)malloc(sizeof(float) * (size_t)(n / 128 > 0 ? n / 128 : 1));
    oracle_quantize_fp8_rows(1, n, v, q, s);
    for (int64_t i = 0; i < n; ++i) v[i] = oracle_e4m3_decode(q[i]) * (double)s[i / 128];
    free(s);
    free(q);
}
