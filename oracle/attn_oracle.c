/*
 * Oracle for the attention forward pass (and its gradients, below) -- TEST
 * INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
 * load this library.  It shares no code with the CUDA path.
 *
 * What it computes is the plain definition of attention that the pages give
 * as the three-step "standard attention" (mooersco.com page, section
 * "标准 Attention 的瓶颈在哪": S = Q K^T, P = softmax(S) by rows, O = P V; the
 * same three steps are listed in section 二 of the gitcode.csdn.net page),
 * with the score scale of 1/sqrt(head_dim) applied to the scores before the
 * softmax (hwcomputing.csdn.net page, "融合kernel" listing: the Scale step).
 * The pages state that the tiled online-softmax method reaches exactly this
 * result (hwcomputing.csdn.net page, "在线softmax" paragraph; gitcode.csdn.net
 * page, section 三), so the oracle is the definition written out, in double
 * precision, one query row at a time:
 *
 *   s_j   = scale * sum_d q[i,d] * k[j,d]        for every visible key j
 *   M     = max_j s_j
 *   w_j   = exp(s_j - M)
 *   Z     = sum_j w_j
 *   O[i]  = sum_j (w_j / Z) * v[j,:]
 *   LSE_i = M + ln Z                              (natural log, scale included)
 *
 * Readings taken where the pages are silent:
 *   - causal masking ("is_causal=True" in the PyTorch section of the
 *     mooersco.com page) keeps key j for query i iff j <= i (top-left
 *     alignment, as PyTorch's scaled_dot_product_attention does);
 *   - GQA/MQA (gitcode.csdn.net page, section 六) maps query head hq to key/value
 *     head hq / (Hq / Hkv): contiguous groups;
 *   - the row log-sum-exp is not on the pages; it is emitted in natural log
 *     with the scale included.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/*
 * One query row over the keys j0 .. j0 + n_vis - 1 of one kv head.
 * q: [D]; k, v: [Nk, D]; bias: NULL or the row's additive score bias [Nk]
 * (-inf removes a key); s: scratch [Nk].  A row with no key left (n_vis == 0,
 * or every biased score -inf) has no softmax: O = 0 and LSE = -inf.
 */
static void attend_row(const float *q, const float *k, const float *v, const float *bias,
                       int64_t j0, int64_t n_vis, int64_t D, double scale, double *s, double *o,
                       double *lse) {
    /* pass 1: scores */
    double M = -INFINITY;
    for (int64_t j = j0; j < j0 + n_vis; ++j) {
        double acc = 0.0;
        const float *kj = k + j * D;
        for (int64_t d = 0; d < D; ++d) acc += (double)q[d] * (double)kj[d];
        s[j] = scale * acc;
        if (bias) s[j] += (double)bias[j];
        if (s[j] > M) M = s[j];
    }
    for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
    if (M == -INFINITY) { /* no visible key */
        *lse = -INFINITY;
        return;
    }
    /* pass 2: softmax weights */
    double Z = 0.0;
    for (int64_t j = j0; j < j0 + n_vis; ++j) {
        s[j] = exp(s[j] - M);
        Z += s[j];
    }
    /* pass 3: weighted sum of values */
    for (int64_t j = j0; j < j0 + n_vis; ++j) {
        const double p = s[j] / Z;
        const float *vj = v + j * D;
        for (int64_t d = 0; d < D; ++d) o[d] += p * (double)vj[d];
    }
    *lse = M + log(Z);
}

/*
 * q:      [B, Hq, R, D] float32 query rows (values already rounded to the storage dtype)
 * q_pos:  [R] position of each supplied row in 0..Nq-1, or NULL (then R must equal Nq)
 * k, v:   [B, Hkv, Nk, D] float32
 * o:      [B, Hq, R, D] float64 output;  lse: [B, Hq, R] float64 output (may be NULL)
 *
 * Masks beyond causal (the pages put the mask step on the vector unit, and
 * PyTorch's scaled_dot_product_attention, which the mooersco.com page calls,
 * takes an attn_mask).  Readings taken:
 *   - a key window: key j is visible to query i iff i - window_left <= j and
 *     j <= i + window_right, a negative bound meaning no bound on that side;
 *     causal is the right bound 0 (top-left alignment, as above);
 *   - an additive bias (float attn_mask): bias[b, h, i, j] is added to the
 *     scaled score, -inf removing the key.  Element (b, hq, i, j) sits at
 *     b * bias_sb + hq * bias_sh + i * bias_sq + j (a zero stride broadcasts);
 *     bias may be NULL;
 *   - a row with no key left has no softmax: O = 0 and LSE = -inf.
 * Returns 0, or a negative number for invalid arguments.
 */
int oracle_attention_ex(const float *q, const int64_t *q_pos, int64_t R, const float *k,
                        const float *v, double *o, double *lse, int64_t B, int64_t Hq,
                        int64_t Hkv, int64_t Nq, int64_t Nk, int64_t D, double scale, int causal,
                        int64_t window_left, int64_t window_right, const float *bias,
                        int64_t bias_sb, int64_t bias_sh, int64_t bias_sq, int nthreads) {
    if (!q || !k || !v || !o) return -1;
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || D < 1 || R < 1) return -2;
    if (Hq % Hkv != 0) return -3;
    if (!q_pos && R != Nq) return -4;
    if (q_pos)
        for (int64_t r = 0; r < R; ++r)
            if (q_pos[r] < 0 || q_pos[r] >= Nq) return -5;
    if (bias && (bias_sb < 0 || bias_sh < 0 || bias_sq < 0)) return -7;
    const int64_t group = Hq / Hkv;
    const int64_t total = B * Hq * R;
    int err = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)Nk);
        if (!s) {
#pragma omp atomic write
            err = -6;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t t = 0; t < total; ++t) {
            if (!s) continue;
            const int64_t r = t % R;
            const int64_t bh = t / R;
            const int64_t b = bh / Hq, hq = bh % Hq;
            const int64_t kvh = hq / group;
            const int64_t i = q_pos ? q_pos[r] : r;
            /* visible keys: j0 .. j1 (inclusive), clipped to 0 .. Nk-1 */
            int64_t j0 = 0, j1 = Nk - 1;
            if (causal && i < j1) j1 = i;
            if (window_right >= 0 && i + window_right < j1) j1 = i + window_right;
            if (window_left >= 0 && i - window_left > j0) j0 = i - window_left;
            const int64_t n_vis = j1 >= j0 ? j1 - j0 + 1 : 0;
            const float *kb = k + (b * Hkv + kvh) * Nk * D;
            const float *vb = v + (b * Hkv + kvh) * Nk * D;
            const float *brow = bias ? bias + b * bias_sb + hq * bias_sh + i * bias_sq : NULL;
            double lse_row;
            attend_row(q + t * D, kb, vb, brow, j0, n_vis, D, scale, s, o + t * D, &lse_row);
            if (lse) lse[t] = lse_row;
        }
        free(s);
    }
    return err;
}

/* The unmasked / causal oracle: oracle_attention_ex with no window and no bias. */
int oracle_attention(const float *q, const int64_t *q_pos, int64_t R, const float *k,
                     const float *v, double *o, double *lse, int64_t B, int64_t Hq,
                     int64_t Hkv, int64_t Nq, int64_t Nk, int64_t D, double scale, int causal,
                     int nthreads) {
    return oracle_attention_ex(q, q_pos, R, k, v, o, lse, B, Hq, Hkv, Nq, Nk, D, scale, causal,
                               -1, -1, NULL, 0, 0, 0, nthreads);
}

/*
 * Gradients of the attention forward pass -- TEST INFRASTRUCTURE ONLY.
 *
 * The pages mention training only to say that back-propagation has to keep
 * the gradients (hwcomputing.csdn.net page, section "标准Attention：一次摊开整本
 * 词典").  Reading: the backward pass is the exact gradient of the operation
 * above, O = softmax(scale * Q K^T) V (causal: keys j <= i only), for a given
 * upstream gradient dO.  Written out by the chain rule, per query row i of one
 * head, in double precision, with P recomputed here from Q and K:
 *
 *   P_ij   = exp(scale * q_i . k_j - LSE_i)          (the forward softmax)
 *   dV_j  += P_ij dO_i
 *   dP_ij  = dO_i . v_j
 *   Delta_i = sum_j P_ij dP_ij                        (= dO_i . O_i)
 *   dS_ij  = P_ij (dP_ij - Delta_i)
 *   dQ_i   = scale * sum_j dS_ij k_j
 *   dK_j  += scale * dS_ij q_i
 *
 * GQA: dK and dV of a key/value head sum over the query heads of its group.
 * Key windows (oracle_attention_bwd_ex; same reading as the forward pass):
 * the sums run over the keys i - window_left .. i + window_right only; a row
 * with no such key has O = 0, so it contributes nothing (dQ_i = 0, Delta_i = 0).
 * An additive score bias (oracle_attention_bwd_ex; the forward pass's float
 * attn_mask reading): the forward softmax is of scale * q_i . k_j + bias_ij,
 * so P above includes the bias and nothing else changes (the bias is a given
 * input: no gradient is formed for it); a key whose bias is -inf has P = 0,
 * and a row whose every visible key has a bias of -inf is a row with no key.
 * bias may be NULL; element (b, hq, i, j) at b * bias_sb + hq * bias_sh +
 * i * bias_sq + j, a zero stride broadcasting that dimension.
 * All arrays are float32 inputs (rounded values) and float64 outputs:
 * q, dout [B, Hq, Nq, D]; k, v [B, Hkv, Nk, D]; dq [B, Hq, Nq, D];
 * dk, dv [B, Hkv, Nk, D]; delta [B, Hq, Nq] (may be NULL).
 * Returns 0, or a negative number for invalid arguments.
 */
int oracle_attention_bwd_ex(const float *q, const float *k, const float *v, const float *dout,
                            double *dq, double *dk, double *dv, double *delta, int64_t B,
                            int64_t Hq, int64_t Hkv, int64_t Nq, int64_t Nk, int64_t D,
                            double scale, int causal, int64_t window_left,
                            int64_t window_right, const float *bias, int64_t bias_sb,
                            int64_t bias_sh, int64_t bias_sq, int nthreads) {
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return -1;
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || D < 1) return -2;
    if (Hq % Hkv != 0) return -3;
    if (bias && (bias_sb < 0 || bias_sh < 0 || bias_sq < 0)) return -7;
    const int64_t group = Hq / Hkv;
    int err = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    /* one (b, kv head) per task: its dK and dV rows are written by that task only */
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)Nk);
        double *dp = (double *)malloc(sizeof(double) * (size_t)Nk);
        if (!p || !dp) {
#pragma omp atomic write
            err = -6;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t bk = 0; bk < B * Hkv; ++bk) {
            if (!p || !dp) continue;
            const int64_t b = bk / Hkv, kvh = bk % Hkv;
            const float *kb = k + bk * Nk * D;
            const float *vb = v + bk * Nk * D;
            double *dkb = dk + bk * Nk * D;
            double *dvb = dv + bk * Nk * D;
            for (int64_t x = 0; x < Nk * D; ++x) dkb[x] = dvb[x] = 0.0;
            for (int64_t hq = kvh * group; hq < (kvh + 1) * group; ++hq) {
                const int64_t bh = b * Hq + hq;
                for (int64_t i = 0; i < Nq; ++i) {
                    const float *qi = q + (bh * Nq + i) * D;
                    const float *gi = dout + (bh * Nq + i) * D;
                    double *dqi = dq + (bh * Nq + i) * D;
                    /* visible keys j0 .. j1 (inclusive) */
                    int64_t j0 = 0, j1 = Nk - 1;
                    if (causal && i < j1) j1 = i;
                    if (window_right >= 0 && i + window_right < j1) j1 = i + window_right;
                    if (window_left >= 0 && i - window_left > j0) j0 = i - window_left;
                    double *dqi0 = dq + (bh * Nq + i) * D;
                    const float *brow =
                        bias ? bias + b * bias_sb + hq * bias_sh + i * bias_sq : NULL;
                    /* forward softmax of the row */
                    double M = -INFINITY;
                    for (int64_t j = j0; j <= j1; ++j) {
                        double acc = 0.0;
                        for (int64_t d = 0; d < D; ++d) acc += (double)qi[d] * (double)kb[j * D + d];
                        p[j] = scale * acc;
                        if (brow) p[j] += (double)brow[j];
                        if (p[j] > M) M = p[j];
                    }
                    if (M == -INFINITY) { /* no visible key: O = 0, nothing to propagate */
                        for (int64_t d = 0; d < D; ++d) dqi0[d] = 0.0;
                        if (delta) delta[bh * Nq + i] = 0.0;
                        continue;
                    }
                    double Z = 0.0;
                    for (int64_t j = j0; j <= j1; ++j) {
                        p[j] = exp(p[j] - M);
                        Z += p[j];
                    }
                    for (int64_t j = j0; j <= j1; ++j) p[j] /= Z;
                    /* dP, Delta */
                    double dl = 0.0;
                    for (int64_t j = j0; j <= j1; ++j) {
                        double acc = 0.0;
                        for (int64_t d = 0; d < D; ++d) acc += (double)gi[d] * (double)vb[j * D + d];
                        dp[j] = acc;
                        dl += p[j] * acc;
                    }
                    if (delta) delta[bh * Nq + i] = dl;
                    /* dS, then the three gradients */
                    for (int64_t d = 0; d < D; ++d) dqi[d] = 0.0;
                    for (int64_t j = j0; j <= j1; ++j) {
                        const double ds = p[j] * (dp[j] - dl);
                        for (int64_t d = 0; d < D; ++d) {
                            dqi[d] += scale * ds * (double)kb[j * D + d];
                            dkb[j * D + d] += scale * ds * (double)qi[d];
                            dvb[j * D + d] += p[j] * (double)gi[d];
                        }
                    }
                }
            }
        }
        free(p);
        free(dp);
    }
    return err;
}

/* The unwindowed gradients (causal or not). */
int oracle_attention_bwd(const float *q, const float *k, const float *v, const float *dout,
                         double *dq, double *dk, double *dv, double *delta, int64_t B,
                         int64_t Hq, int64_t Hkv, int64_t Nq, int64_t Nk, int64_t D,
                         double scale, int causal, int nthreads) {
    return oracle_attention_bwd_ex(q, k, v, dout, dq, dk, dv, delta, B, Hq, Hkv, Nq, Nk, D, scale,
                                   causal, -1, -1, NULL, 0, 0, 0, nthreads);
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
