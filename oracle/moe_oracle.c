/*
 * moe_oracle.c -- plain, slow, single-threaded CPU reference of the MoE-layer forward.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load
 * this file: only the test suite, the smoke check and the benchmark's CPU
 * baseline use it. It shares no code with the CUDA library.
 *
 * Every floating-point value is accumulated in double precision unless a step
 * is defined by the method in fp32 (the balancing thresholds and the ranking
 * key with a Loss-Free bias, which the kernels decide in fp32 too). Inputs
 * arrive as float arrays whose values are already representable in the
 * storage dtype (bf16 values are passed as exact floats).
 *
 * Sources (page title, section / equation):
 *  [SWR]  "Switch Transformers paper review" (tildalice.io/?p=118):
 *         Switch Routing Steps 1-3; Expert Capacity and token drop; the
 *         auxiliary load balancing loss (f_i, P_i, alpha = 1e-2); the
 *         selective-precision router pseudo-code; the FFN max(0,xW1+b1)W2+b2;
 *         the Shazeer top-k gate Softmax(TopK(x W_g)).
 *  [SWI]  "Switch Transformer read for implementation: top-1 routing and expert
 *         parallelism" (molayo1419.me): forward pass permutes token order
 *         twice; expert capacity; overflow tokens take the residual path.
 *  [QB]   "MoE travelogue 6: optimal assignment promotes balance"
 *         (kexue.fm/archives/11619): Method review eqs. (1)-(2) (Loss-Free);
 *         Linear programming eqs. (3)-(4); Max-min eqs. (5)-(7); Divide and
 *         conquer eqs. (8)-(11); Alternating iteration (the QB algorithm box);
 *         Mind the pitfall (select with the old beta, then update; the
 *         one-iteration-per-step form); Demo code (MaxVio/MinVio/AvgVio).
 *  [QW]   "Qwen global-batch load balance for MoE LLM training"
 *         (agentlenshq.com): micro-batch vs global-batch balance loss.
 *  [MOE]  "Mixture of Experts (MoE)" (royzero.tistory.com), section 6: top-k
 *         gate as softmax over the selected scores.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_NOT_CONVERGED 5
#define ORC_ERR_INTERNAL 6

#define ORC_SOFTMAX 0
#define ORC_SIGMOID 1

#define ORC_QB_STEP 0
#define ORC_QB_SOLVE 1
#define ORC_QB_MIDPOINT 0
#define ORC_QB_BOUNDARY 1
#define ORC_QB_BIP 2

/* Ranking order used everywhere: larger key first, equal keys -> lower index first. */
static int ranks_before(double ka, int ia, double kb, int ib) {
    return ka > kb || (ka == kb && ia < ib);
}

/* Indices of the k best keys, best first: k rounds of "take the best remaining". */
static void select_best(const double* key, int n, int k, int* out, unsigned char* taken) {
    memset(taken, 0, (size_t)n);
    for (int r = 0; r < k; ++r) {
        int best = -1;
        for (int j = 0; j < n; ++j) {
            if (taken[j]) continue;
            if (best < 0 || ranks_before(key[j], j, key[best], best)) best = j;
        }
        out[r] = best;
        taken[best] = 1;
    }
}

/* fp32 add, rounded to nearest: the ranking key rho_i + b_i of [QB] eq. (1). */
static float add_f32(float a, float b) {
    volatile float s = a + b;
    return s;
}

/*
 * Router: projection, score function, ranking and gate ([SWR] Switch Routing
 * Steps 1-3; selective precision: the projection and softmax in fp32 or
 * better -- here fp64; [SWR] Shazeer gate for k >= 2; [QB] eq. (1): the bias
 * b enters the ranking only, the gate stays rho_i).
 *
 *   h = x W_r  (x [m,d], W_r [d,n]), or h = logits_in when given.
 *   softmax: p = exp(h - max h) / sum;  sigmoid: rho = 1 / (1 + exp(-h)).
 *   key: with a bias b: fp32(fp32(score) + b); softmax without bias: h;
 *        sigmoid without bias: rho.
 *   top-k by key, ties to the lowest expert index, listed best first.
 *   gate: sigmoid -> rho_sel; softmax -> p_sel, or (renorm) p_sel / sum of
 *         the selected p, i.e. a softmax over the selected logits.
 *   margin[i] = key of the k-th pick minus key of the (k+1)-th best (inf if k == n).
 */
int orc_router(const float* x, const float* w_r, const float* logits_in, int64_t m, int d, int n, int k,
               int fn, int renorm, const float* rank_bias, double* probs_out, int32_t* topk_idx,
               double* topk_gate, double* margin_out) {
    if (m < 0 || n < 1 || k < 1 || k > n || (fn != ORC_SOFTMAX && fn != ORC_SIGMOID)) return ORC_ERR_ARG;
    double* h = (double*)malloc(sizeof(double) * (size_t)n);
    double* p = (double*)malloc(sizeof(double) * (size_t)n);
    double* key = (double*)malloc(sizeof(double) * (size_t)n);
    int* sel = (int*)malloc(sizeof(int) * (size_t)(n));
    unsigned char* taken = (unsigned char*)malloc((size_t)n);
    for (int64_t i = 0; i < m; ++i) {
        for (int j = 0; j < n; ++j) {
            if (logits_in) {
                h[j] = (double)logits_in[i * n + j];
            } else {
                double acc = 0.0;
                for (int t = 0; t < d; ++t) acc += (double)x[i * d + t] * (double)w_r[(int64_t)t * n + j];
                h[j] = acc;
            }
        }
        if (fn == ORC_SOFTMAX) {
            double mx = h[0];
            for (int j = 1; j < n; ++j) if (h[j] > mx) mx = h[j];
            double z = 0.0;
            for (int j = 0; j < n; ++j) { p[j] = exp(h[j] - mx); z += p[j]; }
            for (int j = 0; j < n; ++j) p[j] /= z;
        } else {
            for (int j = 0; j < n; ++j) p[j] = 1.0 / (1.0 + exp(-h[j]));
        }
        for (int j = 0; j < n; ++j) {
            if (rank_bias) key[j] = (double)add_f32((float)p[j], rank_bias[j]);
            else key[j] = (fn == ORC_SOFTMAX) ? h[j] : p[j];
        }
        int take = k < n ? k + 1 : k;
        select_best(key, n, take, sel, taken);
        if (margin_out) margin_out[i] = (k < n) ? key[sel[k - 1]] - key[sel[k]] : INFINITY;
        double selsum = 0.0;
        for (int r = 0; r < k; ++r) selsum += p[sel[r]];
        for (int r = 0; r < k; ++r) {
            topk_idx[i * k + r] = sel[r];
            double g = p[sel[r]];
            if (fn == ORC_SOFTMAX && renorm) g = p[sel[r]] / selsum;
            topk_gate[i * k + r] = g;
        }
        if (probs_out) for (int j = 0; j < n; ++j) probs_out[i * n + j] = p[j];
    }
    free(h); free(p); free(key); free(sel); free(taken);
    return ORC_OK;
}

/*
 * Capacity slots and the expert-major layout ([SWR] Expert Capacity and token
 * drop; [SWI] Expert Capacity, overflow to the residual path, and the
 * dispatch permutation that groups tokens by expert in their original order).
 *
 * Within each segment of seg_len tokens, assignments are visited in token
 * order; the r-th assignment to expert e (r counted from 0) gets slot r and is
 * kept if r < capacity, otherwise slot -1 (dropped, residual path only).
 * Kept rows are laid out expert-major: expert 0's rows first (segment 0's,
 * then segment 1's, ... each in token order), then expert 1's, ...
 */
int orc_capacity(const int32_t* topk_idx, int64_t m, int k, int n, int32_t capacity, int64_t seg_len,
                 int32_t* slot, int32_t* dest_row, int32_t* src_token, int32_t* expert_offsets,
                 int32_t* routed_count, int32_t* kept_count) {
    if (seg_len <= 0 || m % seg_len != 0 || capacity < 0 || k < 1 || k > n) return ORC_ERR_ARG;
    int64_t nseg = m / seg_len;
    int64_t* cnt = (int64_t*)calloc((size_t)n, sizeof(int64_t));
    for (int64_t s = 0; s < nseg; ++s) {
        memset(cnt, 0, sizeof(int64_t) * (size_t)n);
        for (int64_t i = s * seg_len; i < (s + 1) * seg_len; ++i) {
            for (int r = 0; r < k; ++r) {
                int e = topk_idx[i * k + r];
                if (e < 0 || e >= n) { free(cnt); return ORC_ERR_ARG; }
                int64_t rank = cnt[e]++;
                slot[i * k + r] = rank < capacity ? (int32_t)rank : -1;
            }
        }
        for (int e = 0; e < n; ++e) {
            routed_count[s * n + e] = (int32_t)cnt[e];
            kept_count[s * n + e] = (int32_t)(cnt[e] < capacity ? cnt[e] : capacity);
        }
    }
    expert_offsets[0] = 0;
    for (int e = 0; e < n; ++e) {
        int64_t tot = 0;
        for (int64_t s = 0; s < nseg; ++s) tot += kept_count[s * n + e];
        expert_offsets[e + 1] = expert_offsets[e] + (int32_t)tot;
    }
    for (int64_t r = 0; r < m * k; ++r) src_token[r] = -1;
    for (int64_t s = 0; s < nseg; ++s) {
        for (int64_t i = s * seg_len; i < (s + 1) * seg_len; ++i) {
            for (int r = 0; r < k; ++r) {
                int e = topk_idx[i * k + r];
                int32_t sl = slot[i * k + r];
                if (sl < 0) { dest_row[i * k + r] = -1; continue; }
                int64_t before = 0;
                for (int64_t s2 = 0; s2 < s; ++s2) before += kept_count[s2 * n + e];
                int64_t row = expert_offsets[e] + before + sl;
                dest_row[i * k + r] = (int32_t)row;
                src_token[row] = (int32_t)i;
            }
        }
    }
    free(cnt);
    return ORC_OK;
}

/* Dispatch: row r of the expert-major buffer is token src_token[r] ([SWI] forward pass, first permute). */
void orc_dispatch(const float* x, int64_t m, int d, const int32_t* src_token, int64_t rows, double* xbuf) {
    (void)m;
    for (int64_t r = 0; r < rows; ++r)
        for (int t = 0; t < d; ++t) xbuf[r * d + t] = (double)x[(int64_t)src_token[r] * d + t];
}

/*
 * Expert FFN ([SWR] Switch Layer: FFN(x) = max(0, x W1 + b1) W2 + b2, one weight
 * set per expert). Rows [expert_offsets[e], expert_offsets[e+1]) belong to
 * expert e. Weights are stored output-major: w1 [n, d_ff, d] holds W1_e^T,
 * w2 [n, d, d_ff] holds W2_e^T.
 */
void orc_expert_ffn(const double* xbuf, const int32_t* expert_offsets, int n, int d, int d_ff,
                    const float* w1, const float* b1, const float* w2, const float* b2, double* ybuf) {
    double* hid = (double*)malloc(sizeof(double) * (size_t)d_ff);
    for (int e = 0; e < n; ++e) {
        const float* W1 = w1 + (int64_t)e * d_ff * d;
        const float* W2 = w2 + (int64_t)e * d * d_ff;
        for (int64_t r = expert_offsets[e]; r < expert_offsets[e + 1]; ++r) {
            const double* xr = xbuf + r * d;
            for (int j = 0; j < d_ff; ++j) {
                double acc = (double)b1[(int64_t)e * d_ff + j];
                for (int t = 0; t < d; ++t) acc += xr[t] * (double)W1[(int64_t)j * d + t];
                hid[j] = acc > 0.0 ? acc : 0.0;
            }
            for (int c = 0; c < d; ++c) {
                double acc = (double)b2[(int64_t)e * d + c];
                for (int j = 0; j < d_ff; ++j) acc += hid[j] * (double)W2[(int64_t)c * d_ff + j];
                ybuf[r * d + c] = acc;
            }
        }
    }
    free(hid);
}

/* Round a double to the nearest bfloat16 value (ties to even), returned as double. */
static double round_bf16(double v) {
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u) return (double)f;
    uint32_t lsb = (u >> 16) & 1u;
    u = (u + 0x7FFFu + lsb) & 0xFFFF0000u;
    memcpy(&f, &u, 4);
    return (double)f;
}

/*
 * Combine ([SWI] restore token order, multiply by the gate, join the residual
 * path; [SWR] Step 3 y = p_i* E_i*(x); dropped assignments contribute nothing).
 *   y_i = [x_i if residual] + sum over kept r of g_ir * ybuf[dest_row_ir]
 * gate_bf16 != 0 rounds each gate to bf16 first (the selective-precision
 * recipe casts the gate back to bf16 for bf16 layers).
 */
void orc_combine(const double* ybuf, const int32_t* dest_row, const double* topk_gate, const float* residual,
                 int64_t m, int k, int d, int gate_bf16, double* y) {
    for (int64_t i = 0; i < m; ++i) {
        for (int c = 0; c < d; ++c) y[i * d + c] = residual ? (double)residual[i * d + c] : 0.0;
        for (int r = 0; r < k; ++r) {
            int32_t row = dest_row[i * k + r];
            if (row < 0) continue;
            double g = topk_gate[i * k + r];
            if (gate_bf16) g = round_bf16(g);
            for (int c = 0; c < d; ++c) y[i * d + c] += g * ybuf[(int64_t)row * d + c];
        }
    }
}

/*
 * Load statistics ([SWR] auxiliary loss L = alpha * N * sum_i f_i * P_i with
 * f_i the routed fraction and P_i the mean router probability; [QW] loss per
 * micro-batch averaged, versus f_i pooled over the global batch; [QB] Demo
 * code MaxVio/MinVio/AvgVio; [QB] eq. (2) Loss-Free update).
 *
 * Counts are taken from the routing decision (before capacity). For k > 1,
 * f_i = count_i / (k * m_seg) so that sum_i f_i = 1.
 *   f, P  : [(nseg + 1) * n], row nseg is the whole batch (pooled counts).
 *   aux   : [nseg + 3]; aux[s] per segment, aux[nseg] mean over segments
 *           (micro-batch loss), aux[nseg + 1] on pooled f and P (global),
 *           aux[nseg + 2] the hybrid loss of [QW] "balancing efficiency and
 *           effectiveness": the global-batch loss plus the micro-batch loss with
 *           the constant weight 0.01, aux[nseg + 1] + 0.01 * aux[nseg].
 *   vio   : [3] MaxVio, MinVio, AvgVio of the pooled counts: F_i = count_i /
 *           sum(count) * n - 1 -> max, min, mean |F_i|.
 *   bias  : b_i <- b_i - gamma * sign(F_i - 1/n) in fp32, with the sign decided
 *           exactly as sign(count_i * n - m * k).
 * probs may be NULL: P and aux are then not written.
 */
int orc_balance_stats(const double* probs, const int32_t* topk_idx, int64_t m, int n, int k, int64_t seg_len,
                      double alpha, double* f, double* P, double* aux, double* vio, const float* bias_in,
                      float gamma, float* bias_out) {
    if (seg_len <= 0 || m % seg_len != 0 || k < 1 || k > n) return ORC_ERR_ARG;
    int64_t nseg = m / seg_len;
    int64_t* tot = (int64_t*)calloc((size_t)n, sizeof(int64_t));
    int64_t* cnt = (int64_t*)calloc((size_t)n, sizeof(int64_t));
    double* psum_all = (double*)calloc((size_t)n, sizeof(double));
    double micro = 0.0;
    for (int64_t s = 0; s < nseg; ++s) {
        memset(cnt, 0, sizeof(int64_t) * (size_t)n);
        for (int64_t i = s * seg_len; i < (s + 1) * seg_len; ++i)
            for (int r = 0; r < k; ++r) cnt[topk_idx[i * k + r]]++;
        double a = 0.0;
        for (int e = 0; e < n; ++e) {
            tot[e] += cnt[e];
            f[s * n + e] = (double)cnt[e] / ((double)k * (double)seg_len);
            if (probs) {
                double ps = 0.0;
                for (int64_t i = s * seg_len; i < (s + 1) * seg_len; ++i) ps += probs[i * n + e];
                psum_all[e] += ps;
                P[s * n + e] = ps / (double)seg_len;
                a += f[s * n + e] * P[s * n + e];
            }
        }
        if (probs) { aux[s] = alpha * (double)n * a; micro += aux[s]; }
    }
    double g = 0.0;
    for (int e = 0; e < n; ++e) {
        f[nseg * n + e] = (double)tot[e] / ((double)k * (double)m);
        if (probs) {
            P[nseg * n + e] = psum_all[e] / (double)m;
            g += f[nseg * n + e] * P[nseg * n + e];
        }
    }
    if (probs) {
        aux[nseg] = micro / (double)nseg;
        aux[nseg + 1] = alpha * (double)n * g;
        aux[nseg + 2] = aux[nseg + 1] + 0.01 * aux[nseg];
    }
    if (vio) {
        double mx = -INFINITY, mn = INFINITY, av = 0.0, all = (double)m * (double)k;
        for (int e = 0; e < n; ++e) {
            double F = (double)tot[e] / all * (double)n - 1.0;
            if (F > mx) mx = F;
            if (F < mn) mn = F;
            av += fabs(F);
        }
        vio[0] = mx; vio[1] = mn; vio[2] = av / (double)n;
    }
    if (bias_in && bias_out) {
        for (int e = 0; e < n; ++e) {
            int64_t lhs = tot[e] * (int64_t)n, rhs = m * (int64_t)k;
            float b = bias_in[e];
            if (lhs > rhs) b = b - gamma;
            else if (lhs < rhs) b = b + gamma;
            bias_out[e] = b;
        }
    }
    free(tot); free(cnt); free(psum_all);
    return ORC_OK;
}

/*
 * Router gradient of the balance loss ([SWR] auxiliary load balancing loss: f_i comes from the
 * argmax and carries no gradient, so the gradient flows through P_i, the mean router score).
 * The loss is L = w_global * L_global + w_micro * L_micro with
 *   L_global = alpha N sum_i f_i P_i over the whole batch (pooled counts, m tokens),
 *   L_micro  = (1 / S) sum_s alpha N sum_i f^s_i P^s_i over the S segments of seg_len tokens
 * (w_global = 1, w_micro = 0.01 is the hybrid loss of [QW]). With f fixed,
 *   dL/dp_i(t) = w_global alpha N f_i / m + w_micro alpha N f^s_i / (S seg_len)   (t in segment s),
 * and through the score function
 *   softmax: dL/dh_j(t) = p_j(t) (dL/dp_j(t) - sum_i p_i(t) dL/dp_i(t)),
 *   sigmoid: dL/dh_j(t) = dL/dp_j(t) p_j(t) (1 - p_j(t)).
 * f is counted from topk_idx as in orc_balance_stats (count / (k m_seg)). dlogits [m, n].
 */
int orc_balance_loss_grad(const double* probs, const int32_t* topk_idx, int64_t m, int n, int k, int64_t seg_len,
                          int fn, double alpha, double w_micro, double w_global, double* dlogits) {
    if (seg_len <= 0 || m % seg_len != 0 || k < 1 || k > n || (fn != ORC_SOFTMAX && fn != ORC_SIGMOID))
        return ORC_ERR_ARG;
    const int64_t S = m / seg_len;
    double* fg = (double*)calloc((size_t)n, sizeof(double));
    double* fs = (double*)calloc((size_t)n, sizeof(double));
    double* g = (double*)malloc(sizeof(double) * (size_t)n);
    for (int64_t q = 0; q < m * k; ++q) fg[topk_idx[q]] += 1.0;
    for (int e = 0; e < n; ++e) fg[e] /= (double)k * (double)m;
    for (int64_t s = 0; s < S; ++s) {
        memset(fs, 0, sizeof(double) * (size_t)n);
        for (int64_t q = s * seg_len * k; q < (s + 1) * seg_len * k; ++q) fs[topk_idx[q]] += 1.0;
        for (int e = 0; e < n; ++e) {
            fs[e] /= (double)k * (double)seg_len;
            g[e] = w_global * alpha * (double)n * fg[e] / (double)m +
                   w_micro * alpha * (double)n * fs[e] / ((double)S * (double)seg_len);
        }
        for (int64_t t = s * seg_len; t < (s + 1) * seg_len; ++t) {
            const double* p = probs + t * n;
            double c = 0.0;
            for (int j = 0; j < n; ++j) c += p[j] * g[j];
            for (int j = 0; j < n; ++j)
                dlogits[t * n + j] = fn == ORC_SOFTMAX ? p[j] * (g[j] - c) : g[j] * p[j] * (1.0 - p[j]);
        }
    }
    free(fg); free(fs); free(g);
    return ORC_OK;
}

/* ---------------------------------------------------------------------------
 * Optimal assignment ([QB]).
 *
 * Problem (3)/(4): maximise sum x_ij s_ij subject to sum_j x_ij = k and
 * sum_i x_ij = C = m k / n. Alternating minimisation of the dual (8):
 *   alpha_i = threshold between the k-th and (k+1)-th largest of s_i - beta
 *   beta_j  = threshold between the C-th and (C+1)-th largest of s_j - alpha
 * Any value between the two order statistics minimises the sub-problem
 * (eqs. (10)-(11)); the page takes the (k+1)-th (BOUNDARY). The MIDPOINT rule
 * takes 0.5 * (a + b) of the two neighbours. Both are evaluated in fp32:
 * v = fp32(s - beta), u = fp32(s - alpha), mid = fp32(fp32(a + b) * 0.5).
 * --------------------------------------------------------------------------- */

typedef struct { float v; int i; } orc_kv;

static int cmp_desc(const void* pa, const void* pb) {
    const orc_kv* a = (const orc_kv*)pa;
    const orc_kv* b = (const orc_kv*)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->i < b->i) ? -1 : (a->i > b->i);
}

/* Threshold between the q-th and (q+1)-th largest of a list sorted descending (q counted from 1).
 * BIP ([QB], "Related work", the inequality-constrained problem (12)-(14)): the (q+1)-th value
 * clipped at zero, max(0, b), since its duals must stay non-negative. */
static float threshold_of(const orc_kv* sorted, int64_t q, int rule) {
    float a = sorted[q - 1].v, b = sorted[q].v;
    if (rule == ORC_QB_BOUNDARY) return b;
    if (rule == ORC_QB_BIP) return b > 0.0f ? b : 0.0f;
    volatile float sum = a + b;
    volatile float half = sum * 0.5f;
    return half;
}

/*
 * Row pass: for every token, sort v = fp32(s_i - beta) descending (ties: lower
 * expert first), record the top-k set into X (if given), count the picks per
 * expert, count tokens whose k-th and (k+1)-th values tie, and set alpha_i.
 */
static void qb_row_pass(const float* s, int64_t m, int n, int k, const float* beta, int rule, float* alpha,
                        unsigned char* X, int64_t* counts, int64_t* ties, orc_kv* buf) {
    if (counts) memset(counts, 0, sizeof(int64_t) * (size_t)n);
    if (ties) *ties = 0;
    for (int64_t i = 0; i < m; ++i) {
        for (int j = 0; j < n; ++j) {
            volatile float v = s[i * n + j] - beta[j];
            buf[j].v = v;
            buf[j].i = j;
        }
        qsort(buf, (size_t)n, sizeof(orc_kv), cmp_desc);
        if (X) memset(X + i * n, 0, (size_t)n);
        for (int r = 0; r < k; ++r) {
            if (X) X[i * n + buf[r].i] = 1;
            if (counts) counts[buf[r].i]++;
        }
        if (ties && buf[k - 1].v == buf[k].v) (*ties)++;
        if (alpha) alpha[i] = threshold_of(buf, k, rule);
    }
}

/* Column pass: beta_j = threshold between the C-th and (C+1)-th largest of fp32(s_ij - alpha_i) over i. */
static void qb_col_pass(const float* s, int64_t m, int n, int64_t C, const float* alpha, int rule, float* beta,
                        orc_kv* buf) {
    for (int j = 0; j < n; ++j) {
        for (int64_t i = 0; i < m; ++i) {
            volatile float u = s[i * n + j] - alpha[i];
            buf[i].v = u;
            buf[i].i = (int)i;
        }
        qsort(buf, (size_t)m, sizeof(orc_kv), cmp_desc);
        beta[j] = threshold_of(buf, C, rule);
    }
}

/*
 * Exact finish for the balanced assignment: successive shortest paths on the
 * n-node expert graph. X is optimal for its own column counts (every token
 * holds the top-k of s_i - beta for one beta, which satisfies the optimality
 * condition (7)); moving one unit of load from an over-full expert to an
 * under-full one along a shortest path keeps it optimal.
 *
 *   arc a -> b: some token i with x_ia = 1, x_ib = 0 swaps a for b; its cost is
 *   W[a][b] = min_i (s_ia - s_ib) in fp64, the argmin token is the lowest index.
 *   distances: every over-full expert starts at 0; rounds of
 *   dist'[b] = min(dist[b], min_a dist[a] + W[a][b]) (all b from the previous
 *   round's dist) until nothing changes; settle[b] = the round (1-based) of b's
 *   last decrease, 0 for the over-full experts; pred[b] = lowest a with
 *   dist[a] + W[a][b] == dist[b] and settle[a] < settle[b]. (The value that set
 *   dist[b] in its last round came from an a already final by then, so such an
 *   a exists; settle decreases along pred, so the path ends at an over-full
 *   expert even when zero-cost cycles make several arcs tight.)
 *   target: under-full expert with the least distance (lowest index on ties);
 *   every arc of its path moves its argmin token.
 * Stops when all counts equal C or after max_repair moves.
 */
static int qb_repair(const float* s, int64_t m, int n, int64_t C, unsigned char* X, int64_t* cnt, int max_repair,
                     int32_t* augments) {
    double* W = (double*)malloc(sizeof(double) * (size_t)n * n);
    int64_t* A = (int64_t*)malloc(sizeof(int64_t) * (size_t)n * n);
    double* dist = (double*)malloc(sizeof(double) * (size_t)n);
    double* nd = (double*)malloc(sizeof(double) * (size_t)n);
    int* pred = (int*)malloc(sizeof(int) * (size_t)n);
    int* settle = (int*)malloc(sizeof(int) * (size_t)n);
    int* path = (int*)malloc(sizeof(int) * (size_t)(n + 1));
    int* sel = (int*)malloc(sizeof(int) * (size_t)n);
    int* unsel = (int*)malloc(sizeof(int) * (size_t)n);
    int status = ORC_OK;
    *augments = 0;
    for (;;) {
        int over = 0;
        for (int e = 0; e < n; ++e) if (cnt[e] > C) over = 1;
        if (!over) break;
        if (*augments >= max_repair) { status = ORC_ERR_NOT_CONVERGED; break; }
        for (int64_t q = 0; q < (int64_t)n * n; ++q) { W[q] = INFINITY; A[q] = -1; }
        for (int64_t i = 0; i < m; ++i) {
            int ns = 0, nu = 0;
            for (int j = 0; j < n; ++j) { if (X[i * n + j]) sel[ns++] = j; else unsel[nu++] = j; }
            for (int p = 0; p < ns; ++p) {
                int a = sel[p];
                for (int q = 0; q < nu; ++q) {
                    int b = unsel[q];
                    double c = (double)s[i * n + a] - (double)s[i * n + b];
                    if (c < W[a * n + b]) { W[a * n + b] = c; A[a * n + b] = i; }
                }
            }
        }
        for (int e = 0; e < n; ++e) { dist[e] = cnt[e] > C ? 0.0 : INFINITY; settle[e] = 0; }
        int settled = 0;
        for (int round = 0; round <= n; ++round) {
            int changed = 0;
            for (int b = 0; b < n; ++b) {
                double best = dist[b];
                for (int a = 0; a < n; ++a) {
                    if (a == b || dist[a] == INFINITY || W[a * n + b] == INFINITY) continue;
                    double c = dist[a] + W[a * n + b];
                    if (c < best) best = c;
                }
                nd[b] = best;
                if (best != dist[b]) { changed = 1; settle[b] = round + 1; }
            }
            memcpy(dist, nd, sizeof(double) * (size_t)n);
            if (!changed) { settled = 1; break; }
        }
        if (!settled) { status = ORC_ERR_INTERNAL; break; }
        for (int b = 0; b < n; ++b) {
            pred[b] = -1;
            if (dist[b] == INFINITY) continue;
            for (int a = 0; a < n; ++a) {
                if (a == b || dist[a] == INFINITY || W[a * n + b] == INFINITY) continue;
                if (dist[a] + W[a * n + b] == dist[b] && settle[a] < settle[b]) { pred[b] = a; break; }
            }
        }
        int target = -1;
        for (int e = 0; e < n; ++e)
            if (cnt[e] < C && dist[e] < INFINITY && (target < 0 || dist[e] < dist[target])) target = e;
        if (target < 0) { status = ORC_ERR_INTERNAL; break; }
        int len = 0, node = target;
        path[len++] = node;
        while (pred[node] >= 0 && len <= n) { node = pred[node]; path[len++] = node; }
        if (len > n || cnt[node] <= C) { status = ORC_ERR_INTERNAL; break; }
        /* path[len-1] is the over-full root, path[0] the target. */
        for (int p = len - 1; p > 0; --p) {
            int a = path[p], b = path[p - 1];
            int64_t i = A[a * n + b];
            if (i < 0 || !X[i * n + a] || X[i * n + b]) { status = ORC_ERR_INTERNAL; break; }
            X[i * n + a] = 0;
            X[i * n + b] = 1;
        }
        if (status != ORC_OK) break;
        cnt[node]--;
        cnt[target]++;
        (*augments)++;
    }
    free(W); free(A); free(dist); free(nd); free(pred); free(settle); free(path); free(sel); free(unsel);
    return status;
}

/*
 * Balanced assignment ([QB] Alternating iteration box and its practical form in
 * Mind the pitfall).
 *
 * STEP  (one training step, warm start from the previous beta):
 *   x = topk(s - beta_old); alpha from s - beta_old; beta_new from s - alpha.
 *   The selection uses the old beta; beta is updated afterwards.
 * SOLVE (balanced assignment of one batch):
 *   repeat: row pass with the current beta (x = topk(s - beta), its counts,
 *   alpha); stop if every count equals C or max_iters beta updates are done;
 *   otherwise update beta by the column pass. If the final x is not balanced,
 *   finish with the exact repair. beta_inout returns the last QB beta.
 * Output: topk_idx [m,k], each token's experts in ascending index order.
 * info [4]: beta updates done, repair moves, remaining excess, tokens whose
 * k-th and (k+1)-th values of s - beta tied in the last row pass.
 */
int orc_balance_assign(const float* s, int64_t m, int n, int k, float* beta_inout, int mode, int rule,
                       int max_iters, int max_repair, int32_t* topk_idx, int32_t* info) {
    if (n < 2 || k < 1 || k >= n || m < 1 || ((m * k) % n) != 0) return ORC_ERR_ARG;
    if (mode != ORC_QB_STEP && mode != ORC_QB_SOLVE) return ORC_ERR_ARG;
    if (rule != ORC_QB_MIDPOINT && rule != ORC_QB_BOUNDARY && rule != ORC_QB_BIP) return ORC_ERR_ARG;
    int64_t C = m * k / n;
    float* alpha = (float*)malloc(sizeof(float) * (size_t)m);
    unsigned char* X = (unsigned char*)malloc((size_t)m * n);
    int64_t* cnt = (int64_t*)malloc(sizeof(int64_t) * (size_t)n);
    orc_kv* buf = (orc_kv*)malloc(sizeof(orc_kv) * (size_t)(m > n ? m : n));
    int64_t ties = 0;
    int32_t iters = 0, augments = 0;
    int status = ORC_OK;
    if (mode == ORC_QB_STEP) {
        qb_row_pass(s, m, n, k, beta_inout, rule, alpha, X, cnt, &ties, buf);
        qb_col_pass(s, m, n, C, alpha, rule, beta_inout, buf);
        iters = 1;
    } else {
        for (;;) {
            qb_row_pass(s, m, n, k, beta_inout, rule, alpha, X, cnt, &ties, buf);
            int balanced = 1;
            for (int e = 0; e < n; ++e) if (cnt[e] != C) balanced = 0;
            if (balanced || iters >= max_iters) break;
            qb_col_pass(s, m, n, C, alpha, rule, beta_inout, buf);
            iters++;
        }
        status = qb_repair(s, m, n, C, X, cnt, max_repair, &augments);
    }
    int64_t excess = 0;
    for (int e = 0; e < n; ++e) {
        int64_t c = 0;
        for (int64_t i = 0; i < m; ++i) c += X[i * n + e];
        if (c > C) excess += c - C;
    }
    for (int64_t i = 0; i < m; ++i) {
        int r = 0;
        for (int j = 0; j < n; ++j) if (X[i * n + j]) topk_idx[i * k + (r++)] = j;
        if (r != k) status = ORC_ERR_INTERNAL;
    }
    if (info) { info[0] = iters; info[1] = augments; info[2] = (int32_t)excess; info[3] = (int32_t)ties; }
    free(alpha); free(X); free(cnt); free(buf);
    return status;
}

/*
 * SignSGD on beta ([QB], "Gradient descent", eqs. (15)-(17)): with alpha from the row pass, the
 * loss l(beta) = sum_ij max(0, s_ij - alpha_i - beta_j) + (m k / n) sum_j beta_j has
 *   dl/dbeta_j = m k / n - sum_i chi(s_ij - alpha_i - beta_j > 0),
 * and the step is beta_j <- beta_j - gamma sign(dl/dbeta_j), used in place of the quantile
 * update. One step: the row pass selects the top-k of s - beta (old beta) and sets alpha by
 * `rule`; then count_j = #{i : fp32(s_ij - alpha_i) > beta_j} (the sign of the second fp32
 * subtraction is that of the exact difference, so this is the indicator as written; sign(0) = 0
 * leaves beta_j unchanged) and beta_j moves by gamma with one fp32 add or subtract.
 * topk_idx / info as orc_balance_assign's STEP.
 */
int orc_qb_sign_step(const float* s, int64_t m, int n, int k, float* beta_inout, float gamma, int rule,
                     int32_t* topk_idx, int32_t* info) {
    if (n < 2 || k < 1 || k >= n || m < 1 || ((m * k) % n) != 0) return ORC_ERR_ARG;
    if (rule != ORC_QB_MIDPOINT && rule != ORC_QB_BOUNDARY && rule != ORC_QB_BIP) return ORC_ERR_ARG;
    const int64_t C = m * k / n;
    float* alpha = (float*)malloc(sizeof(float) * (size_t)m);
    unsigned char* X = (unsigned char*)malloc((size_t)m * n);
    int64_t* cnt = (int64_t*)malloc(sizeof(int64_t) * (size_t)n);
    orc_kv* buf = (orc_kv*)malloc(sizeof(orc_kv) * (size_t)n);
    int64_t ties = 0;
    qb_row_pass(s, m, n, k, beta_inout, rule, alpha, X, cnt, &ties, buf);
    int64_t excess = 0;
    for (int e = 0; e < n; ++e) if (cnt[e] > C) excess += cnt[e] - C;
    for (int j = 0; j < n; ++j) {
        int64_t c = 0;
        for (int64_t i = 0; i < m; ++i) {
            volatile float u = s[i * n + j] - alpha[i];
            if (u > beta_inout[j]) c++;
        }
        if (c > C) beta_inout[j] = add_f32(beta_inout[j], gamma);        /* gradient < 0 */
        else if (c < C) beta_inout[j] = add_f32(beta_inout[j], -gamma);  /* gradient > 0 */
    }
    for (int64_t i = 0; i < m; ++i) {
        int r = 0;
        for (int j = 0; j < n; ++j) if (X[i * n + j]) topk_idx[i * k + (r++)] = j;
    }
    if (info) { info[0] = 1; info[1] = 0; info[2] = (int32_t)excess; info[3] = (int32_t)ties; }
    free(alpha); free(X); free(cnt); free(buf);
    return ORC_OK;
}

/*
 * The practical QB step on mini-batches ([QB] "Mind the pitfall", closing paragraph): an exact
 * beta over the whole batch needs the (m k / n + 1)-th largest of m values per expert, too
 * costly when m is in the millions, so the batch is split into mini-batches of seg_len tokens,
 * beta is computed on each by the formula, and the results are averaged.
 *   x = topk(s - beta_old) and alpha from s - beta_old for every token (the row pass of STEP:
 *   selection with the old beta, before the update);
 *   for each mini-batch b (tokens b L .. b L + L - 1, L = seg_len, C_b = L k / n): beta_b by the
 *   column pass of those tokens alone;
 *   beta_new_j = fp32( (sum over b = 0, 1, ... of (double) beta_b_j) / B ), B = m / L, the sum
 *   taken in mini-batch order.
 * seg_len = m is the STEP of orc_balance_assign. Requires L | m and (L k) % n == 0.
 * topk_idx / info as orc_balance_assign's STEP (info[0] = 1).
 */
int orc_balance_step_minibatch(const float* s, int64_t m, int n, int k, float* beta_inout, int rule, int64_t seg_len,
                               int32_t* topk_idx, int32_t* info) {
    if (n < 2 || k < 1 || k >= n || m < 1 || seg_len < 1 || m % seg_len != 0 || ((seg_len * k) % n) != 0)
        return ORC_ERR_ARG;
    if (rule != ORC_QB_MIDPOINT && rule != ORC_QB_BOUNDARY && rule != ORC_QB_BIP) return ORC_ERR_ARG;
    const int64_t nb = m / seg_len, Cb = seg_len * k / n, C = m * k / n;
    float* alpha = (float*)malloc(sizeof(float) * (size_t)m);
    unsigned char* X = (unsigned char*)malloc((size_t)m * n);
    int64_t* cnt = (int64_t*)malloc(sizeof(int64_t) * (size_t)n);
    orc_kv* buf = (orc_kv*)malloc(sizeof(orc_kv) * (size_t)(seg_len > n ? seg_len : n));
    float* bb = (float*)malloc(sizeof(float) * (size_t)n);
    double* acc = (double*)calloc((size_t)n, sizeof(double));
    int64_t ties = 0;
    qb_row_pass(s, m, n, k, beta_inout, rule, alpha, X, cnt, &ties, buf);
    for (int64_t b = 0; b < nb; ++b) {
        qb_col_pass(s + b * seg_len * n, seg_len, n, Cb, alpha + b * seg_len, rule, bb, buf);
        for (int j = 0; j < n; ++j) acc[j] += (double)bb[j];
    }
    for (int j = 0; j < n; ++j) beta_inout[j] = (float)(acc[j] / (double)nb);
    int64_t excess = 0;
    for (int e = 0; e < n; ++e) if (cnt[e] > C) excess += cnt[e] - C;
    for (int64_t i = 0; i < m; ++i) {
        int r = 0;
        for (int j = 0; j < n; ++j) if (X[i * n + j]) topk_idx[i * k + (r++)] = j;
    }
    if (info) { info[0] = 1; info[1] = 0; info[2] = (int32_t)excess; info[3] = (int32_t)ties; }
    free(alpha); free(X); free(cnt); free(buf); free(bb); free(acc);
    return ORC_OK;
}

/* One QB row pass alone: alpha_i, the top-k of s_i - beta (best first) and the per-expert counts. */
void orc_qb_row(const float* s, int64_t m, int n, int k, const float* beta, int rule, float* alpha,
                int32_t* topk_idx, int64_t* counts) {
    orc_kv* buf = (orc_kv*)malloc(sizeof(orc_kv) * (size_t)n);
    for (int64_t i = 0; i < m; ++i) {
        for (int j = 0; j < n; ++j) {
            volatile float v = s[i * n + j] - beta[j];
            buf[j].v = v;
            buf[j].i = j;
        }
        qsort(buf, (size_t)n, sizeof(orc_kv), cmp_desc);
        for (int r = 0; r < k; ++r) topk_idx[i * k + r] = buf[r].i;
        alpha[i] = threshold_of(buf, k, rule);
    }
    free(buf);
    if (counts) {
        memset(counts, 0, sizeof(int64_t) * (size_t)n);
        for (int64_t q = 0; q < m * k; ++q) counts[topk_idx[q]]++;
    }
}

/* One QB column pass alone: beta_j from s - alpha with C = m k / n. */
void orc_qb_col(const float* s, int64_t m, int n, int64_t C, const float* alpha, int rule, float* beta) {
    orc_kv* buf = (orc_kv*)malloc(sizeof(orc_kv) * (size_t)m);
    qb_col_pass(s, m, n, C, alpha, rule, beta, buf);
    free(buf);
}

/*
 * Optimality certificate for an assignment with given column counts: X is
 * optimal among assignments with the same row and column sums iff the expert
 * graph (arcs as in the repair) has no negative cycle. Bellman-Ford from a
 * virtual source joined to every expert at cost 0; still improving by more
 * than tol after n rounds means a negative cycle. Returns 1 if optimal.
 */
int orc_is_optimal(const float* s, int64_t m, int n, const int32_t* topk_idx, int k, double tol) {
    double* W = (double*)malloc(sizeof(double) * (size_t)n * n);
    double* dist = (double*)calloc((size_t)n, sizeof(double));
    unsigned char* in = (unsigned char*)malloc((size_t)n);
    for (int64_t q = 0; q < (int64_t)n * n; ++q) W[q] = INFINITY;
    for (int64_t i = 0; i < m; ++i) {
        memset(in, 0, (size_t)n);
        for (int r = 0; r < k; ++r) in[topk_idx[i * k + r]] = 1;
        for (int a = 0; a < n; ++a) {
            if (!in[a]) continue;
            for (int b = 0; b < n; ++b) {
                if (in[b]) continue;
                double c = (double)s[i * n + a] - (double)s[i * n + b];
                if (c < W[a * n + b]) W[a * n + b] = c;
            }
        }
    }
    int optimal = 0;
    for (int round = 0; round <= n; ++round) {
        int changed = 0;
        for (int a = 0; a < n; ++a)
            for (int b = 0; b < n; ++b) {
                if (W[a * n + b] == INFINITY) continue;
                if (dist[a] + W[a * n + b] < dist[b] - tol) { dist[b] = dist[a] + W[a * n + b]; changed = 1; }
            }
        if (!changed) { optimal = 1; break; }
    }
    free(W); free(dist); free(in);
    return optimal;
}
