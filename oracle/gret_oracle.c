/*
 * gret_oracle.c -- plain, slow, fp64 CPU oracle for multi-head Gated Retention (gRet).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls this file:
 * only the tests, the smoke check and the benchmark's CPU-baseline leg use it.  It shares no
 * code, header, table or constant with the CUDA library, and it includes nothing from it.
 *
 * Sources (web pages on YOCO; cited by page title and section):
 *   [P1] "YOCO 完全拆解：Decoder-Decoder 架构如何让 KV Cache 只存一次"
 *        (pinghaoyang.com.cn/aigc/posts/yoco/)
 *        - section "路线二：Multi-Head Gated Retention": per-head scalar gate gamma_n from a
 *          learned projection and a temperature tau that keeps gamma near 1; the recurrence
 *          S_n = gamma_n S_{n-1} + K_n^T V_n, O_n = Q_n S_n; the unrolled form in which the
 *          contribution of position m to position n carries the product of the gates strictly
 *          after m up to and including n; per-head GroupNorm followed by swish(X W_G).
 *        - section "Prefill 与 Decode 为什么使用两种计算形态": the chunkwise form (inner
 *          + cross-chunk terms, chunk-end state passed on, cumulative in-chunk decay) and the
 *          statement that parallel, recurrent and chunkwise forms are re-associations of one
 *          formula.
 *        - section "单 token Decode 的实现骨架": the decode update multiplies the old state by
 *          exp(gate) and adds outer(k, v); the gate logit is divided by 16; K is scaled by
 *          d_h^{-1/2}.
 *        - section "路线一：滑动窗口注意力": the other Self-Decoder mixer, softmax attention in
 *          which position i sees only the most recent C positions (C = 1024 in the page's
 *          scaling runs).
 *        - the same "路线二" section weighs an element-wise gate against the head-wise one.
 *   The display formulas of [P1] were stripped when the page was extracted to text; the
 *   readings taken where the page is silent are listed with each function.
 *
 * Parity pins (tests/test_oracle_pins.py): brute-force parallel form, gamma==1 (causal linear
 * attention), gamma==0 (current token only), a hand-worked example in tests/golden/, chunkwise
 * re-association at many chunk sizes, split prefill, decode-after-prefill, linearity, and the
 * GroupNorm moments; for the per-channel gate, reduction to the head-wise recurrence, the
 * brute-force product form, a one-hot query row and closed gates; for sliding-window
 * attention, the explicit-mask matrix form, window 1, a wide window against causal attention
 * and zero queries.
 *
 * Layout used by every function here (the test harness converts to it):
 *   q, k  : [T][H][dk]   (token-major, contiguous, fp64)
 *   v, o  : [T][H][dv]
 *   g     : [T][H]       gate logits
 *   state : [n_seqs][H][dk][dv]
 *   cu_seqlens : [n_seqs+1] int64, sequence s owns tokens cu[s] .. cu[s+1]-1
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* log(sigmoid(x)) evaluated without overflow: min(x,0) - log(1 + exp(-|x|)). */
static double logsigmoid(double x) {
    double m = x < 0.0 ? x : 0.0;
    return m - log1p(exp(-fabs(x)));
}

/* Log of the per-token decay.  [P1, "路线二"] gives gamma = sigmoid(x W_gamma)^(1/tau); the
 * decode section of [P1] says the official code divides the gate logit by 16.  Reading: the
 * library receives the logit g = x W_gamma, and log(gamma) = logsigmoid(g) / tau. */
double oracle_log_gamma(double g, double tau) { return logsigmoid(g) / tau; }

static int check_seqs(const int64_t* cu, int n_seqs, int64_t T) {
    if (n_seqs < 0 || cu == NULL) return -1;
    if (cu[0] != 0 || cu[n_seqs] != T) return -1;
    for (int s = 0; s < n_seqs; ++s)
        if (cu[s + 1] < cu[s]) return -1;
    return 0;
}

/*
 * Recurrent form, [P1, "路线二"] and [P1, "单 token Decode 的实现骨架"]:
 *   S <- gamma_t * S + (k_scale * K_t)^T V_t      (decay first, then add the current token)
 *   O_t <- Q_t S                                  (the output reads the updated state)
 * per sequence and head, starting from state_in (or zero).  state_out receives the final S.
 * state_out may alias state_in.  Returns 0, or -1 on inconsistent sequence offsets.
 */
int oracle_gret_recurrent(const double* q, const double* k, const double* v, const double* g,
                          double tau, double k_scale, int64_t T, int H, int dk, int dv,
                          const int64_t* cu_seqlens, int n_seqs, const double* state_in,
                          double* state_out, double* o) {
    if (check_seqs(cu_seqlens, n_seqs, T)) return -1;
    int64_t units = (int64_t)n_seqs * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
        int s = (int)(u / H), h = (int)(u % H);
        double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
        if (state_in)
            memcpy(S, state_in + u * dk * dv, sizeof(double) * (size_t)dk * dv);
        else
            memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (int64_t t = cu_seqlens[s]; t < cu_seqlens[s + 1]; ++t) {
            const double* qt = q + (t * H + h) * dk;
            const double* kt = k + (t * H + h) * dk;
            const double* vt = v + (t * H + h) * dv;
            double gamma = exp(oracle_log_gamma(g[t * H + h], tau));
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    S[i * dv + j] = gamma * S[i * dv + j] + (k_scale * kt[i]) * vt[j];
            double* ot = o + (t * H + h) * dv;
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += qt[i] * S[i * dv + j];
                ot[j] = acc;
            }
        }
        if (state_out) memcpy(state_out + u * dk * dv, S, sizeof(double) * (size_t)dk * dv);
        free(S);
    }
    return 0;
}

/*
 * Parallel (unrolled) form by brute force, [P1, "路线二"]: the recurrence unrolled gives
 *   O_n = sum_{m<=n} D_{nm} (Q_n . K_m) V_m  +  D_{n,a-1} Q_n S_0,
 *   D_{nm} = prod_{m<k<=n} gamma_k  (an empty product is 1),
 * where a is the first token of the sequence and S_0 the entry state.  The products are
 * formed term by term, not from cumulative sums, so this is an independent route to the same
 * numbers.  O(N^2 (dk+dv)) per head: tiny inputs only.  state_out (optional) is
 *   S_N = D_{N,a-1} S_0 + sum_m D_{Nm} K_m^T V_m.
 */
int oracle_gret_parallel(const double* q, const double* k, const double* v, const double* g,
                         double tau, double k_scale, int64_t T, int H, int dk, int dv,
                         const int64_t* cu_seqlens, int n_seqs, const double* state_in,
                         double* state_out, double* o) {
    if (check_seqs(cu_seqlens, n_seqs, T)) return -1;
    int64_t units = (int64_t)n_seqs * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
        int s = (int)(u / H), h = (int)(u % H);
        int64_t a = cu_seqlens[s], b = cu_seqlens[s + 1];
        const double* S0 = state_in ? state_in + u * dk * dv : NULL;
        for (int64_t n = a; n < b; ++n) {
            double* on = o + (n * H + h) * dv;
            const double* qn = q + (n * H + h) * dk;
            for (int j = 0; j < dv; ++j) on[j] = 0.0;
            for (int64_t m = a; m <= n; ++m) {
                double D = 1.0;
                for (int64_t kk = m + 1; kk <= n; ++kk) D *= exp(oracle_log_gamma(g[kk * H + h], tau));
                const double* km = k + (m * H + h) * dk;
                const double* vm = v + (m * H + h) * dv;
                double qk = 0.0;
                for (int i = 0; i < dk; ++i) qk += qn[i] * (k_scale * km[i]);
                for (int j = 0; j < dv; ++j) on[j] += D * qk * vm[j];
            }
            if (S0) {
                double D = 1.0; /* all gates a..n act on the entry state */
                for (int64_t kk = a; kk <= n; ++kk) D *= exp(oracle_log_gamma(g[kk * H + h], tau));
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += qn[i] * S0[i * dv + j];
                    on[j] += D * acc;
                }
            }
        }
        if (state_out) {
            double* SN = state_out + u * dk * dv;
            double D0 = 1.0;
            for (int64_t kk = a; kk < b; ++kk) D0 *= exp(oracle_log_gamma(g[kk * H + h], tau));
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) SN[i * dv + j] = S0 ? D0 * S0[i * dv + j] : 0.0;
            for (int64_t m = a; m < b; ++m) {
                double D = 1.0;
                for (int64_t kk = m + 1; kk < b; ++kk) D *= exp(oracle_log_gamma(g[kk * H + h], tau));
                const double* km = k + (m * H + h) * dk;
                const double* vm = v + (m * H + h) * dv;
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) SN[i * dv + j] += D * (k_scale * km[i]) * vm[j];
            }
        }
    }
    return 0;
}

/*
 * Chunkwise form, [P1, "Prefill 与 Decode 为什么使用两种计算形态"]: split each sequence into
 * chunks [a, b] of `chunk` tokens (the last one may be shorter).  With the in-chunk inclusive
 * cumulative log-decay c_t = sum_{k=a..t} log(gamma_k) and the entry state S_{a-1}:
 *   O_t   = sum_{m=a..t} exp(c_t - c_m) (Q_t . K_m) V_m      (inner term)
 *         + exp(c_t) Q_t S_{a-1}                            (cross-chunk term)
 *   S_b   = exp(c_b) S_{a-1} + sum_{m=a..b} exp(c_b - c_m) K_m^T V_m   (chunk-end state)
 * This is the decomposition the GPU path computes; here it is evaluated in fp64 with plain
 * loops, so that a test can show it equals the recurrent form for every chunk size.
 */
int oracle_gret_chunkwise(const double* q, const double* k, const double* v, const double* g,
                          double tau, double k_scale, int64_t T, int H, int dk, int dv,
                          const int64_t* cu_seqlens, int n_seqs, const double* state_in,
                          double* state_out, double* o, int chunk) {
    if (check_seqs(cu_seqlens, n_seqs, T) || chunk < 1) return -1;
    int64_t units = (int64_t)n_seqs * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
        int s = (int)(u / H), h = (int)(u % H);
        double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
        double* Snew = (double*)malloc(sizeof(double) * (size_t)dk * dv);
        double* c = (double*)malloc(sizeof(double) * (size_t)chunk);
        if (state_in)
            memcpy(S, state_in + u * dk * dv, sizeof(double) * (size_t)dk * dv);
        else
            memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (int64_t a = cu_seqlens[s]; a < cu_seqlens[s + 1]; a += chunk) {
            int64_t b = a + chunk - 1;
            if (b > cu_seqlens[s + 1] - 1) b = cu_seqlens[s + 1] - 1;
            double run = 0.0;
            for (int64_t t = a; t <= b; ++t) {
                run += oracle_log_gamma(g[t * H + h], tau);
                c[t - a] = run;
            }
            for (int64_t t = a; t <= b; ++t) {
                const double* qt = q + (t * H + h) * dk;
                double* ot = o + (t * H + h) * dv;
                double ec = exp(c[t - a]);
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += qt[i] * S[i * dv + j];
                    ot[j] = ec * acc;
                }
                for (int64_t m = a; m <= t; ++m) {
                    const double* km = k + (m * H + h) * dk;
                    const double* vm = v + (m * H + h) * dv;
                    double qk = 0.0;
                    for (int i = 0; i < dk; ++i) qk += qt[i] * (k_scale * km[i]);
                    double w = exp(c[t - a] - c[m - a]) * qk;
                    for (int j = 0; j < dv; ++j) ot[j] += w * vm[j];
                }
            }
            double eb = exp(c[b - a]);
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) Snew[i * dv + j] = eb * S[i * dv + j];
            for (int64_t m = a; m <= b; ++m) {
                const double* km = k + (m * H + h) * dk;
                const double* vm = v + (m * H + h) * dv;
                double w = exp(c[b - a] - c[m - a]);
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) Snew[i * dv + j] += w * (k_scale * km[i]) * vm[j];
            }
            memcpy(S, Snew, sizeof(double) * (size_t)dk * dv);
        }
        if (state_out) memcpy(state_out + u * dk * dv, S, sizeof(double) * (size_t)dk * dv);
        free(S);
        free(Snew);
        free(c);
    }
    return 0;
}

/*
 * One recurrent decode step for a batch, [P1, "单 token Decode 的实现骨架"]: for each
 * (b, h):  S <- gamma S + (k_scale k)^T v ;  o = q S.  Same arithmetic as one iteration of
 * oracle_gret_recurrent; kept as its own entry so that decode is checked on its own layout:
 *   q, k : [B][H][dk]; v, o : [B][H][dv]; g : [B][H]; state : [B][H][dk][dv] (in place).
 */
int oracle_gret_decode_step(const double* q, const double* k, const double* v, const double* g,
                            double tau, double k_scale, int B, int H, int dk, int dv,
                            double* state, double* o) {
    int64_t units = (int64_t)B * H;
#pragma omp parallel for schedule(static)
    for (int64_t u = 0; u < units; ++u) {
        double* S = state + u * dk * dv;
        const double* qt = q + u * dk;
        const double* kt = k + u * dk;
        const double* vt = v + u * dv;
        double gamma = exp(oracle_log_gamma(g[u], tau));
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j)
                S[i * dv + j] = gamma * S[i * dv + j] + (k_scale * kt[i]) * vt[j];
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += qt[i] * S[i * dv + j];
            o[u * dv + j] = acc;
        }
    }
    return 0;
}

/*
 * Output epilogue, [P1, "路线二"]: per-head GroupNorm of the retention output, multiplied by
 * swish(X W_G).  Readings (the formula is stripped on the page): one group per head, the
 * statistics of token t over the dv channels of head h, biased variance, affine weight and bias
 * per channel (identity when NULL), swish(z) = z * sigmoid(z).  The output projection W_O is
 * not part of this step.
 *   o  : [T][H*dv]   x : [T][D]   wg : [D][H*dv]   y : [n_rows][H*dv]
 * Only the `n_rows` rows listed in `rows` are computed, and y row r holds token rows[r] (rows
 * are independent; a sample keeps the fp64 GEMM affordable).  rows == NULL means every token
 * 0..T-1 in order (n_rows is then ignored and y has T rows).
 */
int oracle_groupnorm_gate(const double* o, const double* x, const double* wg,
                          const double* gn_weight, const double* gn_bias, double eps, int64_t T,
                          int H, int dv, int D, const int64_t* rows, int64_t n_rows, double* y) {
    int64_t F = (int64_t)H * dv;
    int64_t nr = rows ? n_rows : T;
    for (int64_t r = 0; r < nr; ++r) {
        int64_t t = rows ? rows[r] : r;
        if (t < 0 || t >= T) return -1;
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nr; ++r) {
        int64_t t = rows ? rows[r] : r;
        double* z = (double*)malloc(sizeof(double) * (size_t)F);
        for (int64_t c = 0; c < F; ++c) z[c] = 0.0;
        for (int e = 0; e < D; ++e) {
            double xe = x[t * D + e];
            const double* w = wg + (int64_t)e * F;
            for (int64_t c = 0; c < F; ++c) z[c] += xe * w[c];
        }
        for (int h = 0; h < H; ++h) {
            const double* oh = o + t * F + (int64_t)h * dv;
            double mu = 0.0, var = 0.0;
            for (int j = 0; j < dv; ++j) mu += oh[j];
            mu /= dv;
            for (int j = 0; j < dv; ++j) var += (oh[j] - mu) * (oh[j] - mu);
            var /= dv;
            double inv = 1.0 / sqrt(var + eps);
            for (int j = 0; j < dv; ++j) {
                int64_t c = (int64_t)h * dv + j;
                double n = (oh[j] - mu) * inv;
                if (gn_weight) n *= gn_weight[c];
                if (gn_bias) n += gn_bias[c];
                double zc = z[c];
                double swish = zc / (1.0 + exp(-zc));
                y[r * F + c] = n * swish;
            }
        }
        free(z);
    }
    return 0;
}

/*
 * Element-wise (per key channel) gate, the alternative that [P1, "路线二"] weighs against the
 * head-wise scalar gate: instead of one gamma per head and token, every key channel i of the
 * state has its own decay alpha_t[i] = sigmoid(g_t[i])^(1/tau), so
 *   S[i][:] <- alpha_t[i] * S[i][:] + (k_scale * K_t[i]) V_t      (decay first, then add)
 *   O_t <- Q_t S
 * Reading: "element-wise" is taken per state row (one gate per key channel, d_k gates per
 * head and token); a separate gate for each of the d_k * d_v state entries would need a gate
 * tensor the size of the state per token, which the page does not describe.
 * Layout as above except g: [T][H][dk].  Returns 0, or -1 on inconsistent sequence offsets.
 */
int oracle_gret_recurrent_ew(const double* q, const double* k, const double* v, const double* g,
                             double tau, double k_scale, int64_t T, int H, int dk, int dv,
                             const int64_t* cu_seqlens, int n_seqs, const double* state_in,
                             double* state_out, double* o) {
    if (check_seqs(cu_seqlens, n_seqs, T)) return -1;
    int64_t units = (int64_t)n_seqs * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
        int s = (int)(u / H), h = (int)(u % H);
        double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
        if (state_in)
            memcpy(S, state_in + u * dk * dv, sizeof(double) * (size_t)dk * dv);
        else
            memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (int64_t t = cu_seqlens[s]; t < cu_seqlens[s + 1]; ++t) {
            const double* qt = q + (t * H + h) * dk;
            const double* kt = k + (t * H + h) * dk;
            const double* vt = v + (t * H + h) * dv;
            const double* gt = g + (t * H + h) * dk;
            for (int i = 0; i < dk; ++i) {
                double alpha = exp(oracle_log_gamma(gt[i], tau));
                for (int j = 0; j < dv; ++j)
                    S[i * dv + j] = alpha * S[i * dv + j] + (k_scale * kt[i]) * vt[j];
            }
            double* ot = o + (t * H + h) * dv;
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += qt[i] * S[i * dv + j];
                ot[j] = acc;
            }
        }
        if (state_out) memcpy(state_out + u * dk * dv, S, sizeof(double) * (size_t)dk * dv);
        free(S);
    }
    return 0;
}

/*
 * Sliding-window attention, the other Self-Decoder mixer of [P1] (section "路线一：滑动窗口注意力"):
 * position i attends only to the most recent `window` positions of its own sequence, j in
 * [i - window + 1, i], with softmax normalisation over exactly those positions:
 *   o_i = sum_j softmax_j(scale * q_i . k_j) v_j
 * (the page's formula and mask were stripped; the reading is the causal window mask that is 0
 * inside the window and -inf outside, with the usual 1/sqrt(d) scale passed as `scale`).
 * Layout: q, k [T][H][d], v, o [T][H][dv].  Returns 0, or -1 on bad offsets or window < 1.
 */
int oracle_swa(const double* q, const double* k, const double* v, double scale, int window,
               int64_t T, int H, int d, int dv, const int64_t* cu_seqlens, int n_seqs,
               double* o) {
    if (check_seqs(cu_seqlens, n_seqs, T) || window < 1) return -1;
    int64_t units = (int64_t)n_seqs * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < units; ++u) {
        int s = (int)(u / H), h = (int)(u % H);
        int64_t a = cu_seqlens[s], e = cu_seqlens[s + 1];
        double* w = (double*)malloc(sizeof(double) * (size_t)window);
        for (int64_t i = a; i < e; ++i) {
            int64_t j0 = i - window + 1 < a ? a : i - window + 1;
            const double* qi = q + (i * H + h) * d;
            double mx = -INFINITY;
            for (int64_t j = j0; j <= i; ++j) {
                const double* kj = k + (j * H + h) * d;
                double sc = 0.0;
                for (int c = 0; c < d; ++c) sc += qi[c] * kj[c];
                w[j - j0] = scale * sc;
                if (w[j - j0] > mx) mx = w[j - j0];
            }
            double den = 0.0;
            for (int64_t j = j0; j <= i; ++j) {
                w[j - j0] = exp(w[j - j0] - mx);
                den += w[j - j0];
            }
            double* oi = o + (i * H + h) * dv;
            for (int c = 0; c < dv; ++c) oi[c] = 0.0;
            for (int64_t j = j0; j <= i; ++j) {
                const double* vj = v + (j * H + h) * dv;
                for (int c = 0; c < dv; ++c) oi[c] += (w[j - j0] / den) * vj[c];
            }
        }
        free(w);
    }
    return 0;
}
