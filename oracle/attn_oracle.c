/*
 * Oracle for the attention forward pass -- TEST INFRASTRUCTURE ONLY.
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

/* One query row.  q: [D], k and v: [Nk, D] of one kv head.  s: scratch [Nk]. */
static void attend_row(const float *q, const float *k, const float *v, int64_t n_vis,
                       int64_t D, double scale, double *s, double *o, double *lse) {
    /* pass 1: scores */
    double M = -INFINITY;
    for (int64_t j = 0; j < n_vis; ++j) {
        double acc = 0.0;
        const float *kj = k + j * D;
        for (int64_t d = 0; d < D; ++d) acc += (double)q[d] * (double)kj[d];
        s[j] = scale * acc;
        if (s[j] > M) M = s[j];
    }
    /* pass 2: softmax weights */
    double Z = 0.0;
    for (int64_t j = 0; j < n_vis; ++j) {
        s[j] = exp(s[j] - M);
        Z += s[j];
    }
    /* pass 3: weighted sum of values */
    for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
    for (int64_t j = 0; j < n_vis; ++j) {
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
 * Returns 0, or a negative number for invalid arguments.
 */
int oracle_attention(const float *q, const int64_t *q_pos, int64_t R, const float *k,
                     const float *v, double *o, double *lse, int64_t B, int64_t Hq,
                     int64_t Hkv, int64_t Nq, int64_t Nk, int64_t D, double scale, int causal,
                     int nthreads) {
    if (!q || !k || !v || !o) return -1;
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || D < 1 || R < 1) return -2;
    if (Hq % Hkv != 0) return -3;
    if (!q_pos && R != Nq) return -4;
    if (q_pos)
        for (int64_t r = 0; r < R; ++r)
            if (q_pos[r] < 0 || q_pos[r] >= Nq) return -5;
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
            int64_t n_vis = Nk;
            if (causal) n_vis = (i + 1 < Nk) ? i + 1 : Nk;
            const float *kb = k + (b * Hkv + kvh) * Nk * D;
            const float *vb = v + (b * Hkv + kvh) * Nk * D;
            double lse_row;
            attend_row(q + t * D, kb, vb, n_vis, D, scale, s, o + t * D, &lse_row);
            if (lse) lse[t] = lse_row;
        }
        free(s);
    }
    return err;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
