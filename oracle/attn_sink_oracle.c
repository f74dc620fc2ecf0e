/*
 * attn_sink_oracle.c -- plain fp64 CPU oracle for sink-softmax GQA attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The CUDA
 * product path never calls it, and the two share no code, header, table or
 * helper.
 *
 * What is computed (sources):
 *   - "GPT-OSS on day 0" (Perplexity), section "Attention: GQA with Attention
 *     Sinks": every attention head carries a pre-trained sink parameter that
 *     enters the softmax.
 *   - same page, section "Sink Attention": the sink is an extra bias term that
 *     joins the Q.K products before the softmax; the softmax is computed with
 *     the maximum subtracted for stability.  The page's formula was lost in
 *     extraction; the definition used is
 *         p_j = exp(s_j - m) / (sum_k exp(s_k - m) + exp(sink_h - m)),
 *     i.e. the sink is one more logit whose value row is zero.
 *   - "GPT-OSS 20B Egitimi: Unsloth, A100 ve Hopper Uyumlulugu", section 1:
 *     grouped multi-query attention, alternating dense and locally banded
 *     causal layers; the band width is sliding_window = 128 ("GPT-OSS-120B
 *     4-bit ...", section 3 "inference optimisation").
 *
 * Readings taken where the pages are silent (all stated once more in the
 * project's design notes):
 *   - s_ij = scale * <q_i, k_j>; the sink is a raw logit, NOT multiplied by
 *     scale.  Natural exponent throughout.
 *   - Query row i of Lq sits at absolute position p_i = i + (Lk - Lq)
 *     (bottom-right causal alignment).  Key j is visible to row i iff
 *     j <= p_i and (window <= 0 or j > p_i - window): a window of w shows
 *     exactly w keys, the query's own key included.
 *   - GQA: query head h reads KV head g = h / (Hq / Hkv) (consecutive query
 *     heads share a KV head).
 *   - LSE_i = M + ln Z includes the sink term.
 *   - A row whose softmax has no finite logit at all (no visible key and
 *     sink = -inf) gives O = 0 and LSE = -inf.
 *
 * Layouts (row-major, all fp64 here):
 *   q, out, dout, dq : [B, Lq, Hq, D]      k, v, dk, dv : [B, Lk, Hkv, D]
 *   lse              : [B, Hq, Lq]         sinks, dsinks: [Hq]
 *   decode: q/out [B, Hq, D], caches [B, Lmax, Hkv, D], seqlens [B], lse [B, Hq]
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC (no -ffast-math: the -inf cases are
 * part of the definition).
 */
#include <math.h>
#include <omp.h>
#include <stdlib.h>
#include <string.h>

static int key_visible(long j, long p, int window)
{
    if (j > p) return 0;
    if (window > 0 && j <= p - window) return 0;
    return 1;
}

static double dot(const double *a, const double *b, int D)
{
    double s = 0.0;
    for (int d = 0; d < D; ++d) s += a[d] * b[d];
    return s;
}

/*
 * One query row of the forward pass, straight from the definition:
 *   z_j = scale * <q, k_j>       for every visible key j
 *   M   = max(sink, max_j z_j)
 *   Z   = exp(sink - M) + sum_j exp(z_j - M)
 *   O   = sum_j exp(z_j - M) v_j / Z
 *   LSE = M + ln Z
 * k_row(j) / v_row(j) are given as base + j*row_stride.
 */
static void fwd_row(const double *q, const double *k0, const double *v0, long row_stride,
                    long nkeys, long p, int window, double scale, double sink, int D,
                    double *o, double *lse)
{
    double M = sink;
    for (long j = 0; j < nkeys; ++j) {
        if (!key_visible(j, p, window)) continue;
        double z = scale * dot(q, k0 + j * row_stride, D);
        if (z > M) M = z;
    }
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (M == -INFINITY) {           /* no finite logit at all */
        *lse = -INFINITY;
        return;
    }
    double Z = exp(sink - M);       /* the sink's mass: no value row */
    for (long j = 0; j < nkeys; ++j) {
        if (!key_visible(j, p, window)) continue;
        double e = exp(scale * dot(q, k0 + j * row_stride, D) - M);
        Z += e;
        const double *vj = v0 + j * row_stride;
        for (int d = 0; d < D; ++d) o[d] += e * vj[d];
    }
    for (int d = 0; d < D; ++d) o[d] /= Z;
    *lse = M + log(Z);
}

/* Prefill forward over every (b, h, i). */
void oracle_fwd(const double *q, const double *k, const double *v, const double *sinks,
                double *out, double *lse, int B, int Lq, int Lk, int Hq, int Hkv, int D,
                int window, double scale)
{
    const int G = Hq / Hkv;
    const long nrows = (long)B * Hq * Lq;
#pragma omp parallel for schedule(dynamic, 16)
    for (long r = 0; r < nrows; ++r) {
        const int b = (int)(r / ((long)Hq * Lq));
        const int h = (int)((r / Lq) % Hq);
        const int i = (int)(r % Lq);
        const int g = h / G;
        const double *qi = q + (((long)b * Lq + i) * Hq + h) * D;
        const double *kb = k + ((long)b * Lk * Hkv + g) * D;
        const double *vb = v + ((long)b * Lk * Hkv + g) * D;
        double *oi = out + (((long)b * Lq + i) * Hq + h) * D;
        fwd_row(qi, kb, vb, (long)Hkv * D, Lk, (long)i + (Lk - Lq), window, scale, sinks[h],
                D, oi, &lse[((long)b * Hq + h) * Lq + i]);
    }
}

/* Forward for a list of sampled rows (b, h, i); out_rows [n, D], lse_rows [n]. */
void oracle_fwd_rows(const double *q, const double *k, const double *v, const double *sinks,
                     const int *rb, const int *rh, const int *ri, int n,
                     double *out_rows, double *lse_rows, int B, int Lq, int Lk, int Hq,
                     int Hkv, int D, int window, double scale)
{
    (void)B;
    const int G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < n; ++t) {
        const int b = rb[t], h = rh[t], i = ri[t], g = h / G;
        const double *qi = q + (((long)b * Lq + i) * Hq + h) * D;
        const double *kb = k + ((long)b * Lk * Hkv + g) * D;
        const double *vb = v + ((long)b * Lk * Hkv + g) * D;
        fwd_row(qi, kb, vb, (long)Hkv * D, Lk, (long)i + (Lk - Lq), window, scale, sinks[h],
                D, out_rows + (long)t * D, &lse_rows[t]);
    }
}

/*
 * Decode: one query per sequence, at position seqlens[b] - 1, over the first
 * seqlens[b] rows of the cache (its own key already appended).
 */
void oracle_decode(const double *q, const double *kc, const double *vc, const int *seqlens,
                   const double *sinks, double *out, double *lse, int B, int Lmax, int Hq,
                   int Hkv, int D, int window, double scale)
{
    const int G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (long r = 0; r < (long)B * Hq; ++r) {
        const int b = (int)(r / Hq), h = (int)(r % Hq), g = h / G;
        const long len = seqlens[b];
        const double *kb = kc + ((long)b * Lmax * Hkv + g) * D;
        const double *vb = vc + ((long)b * Lmax * Hkv + g) * D;
        fwd_row(q + r * D, kb, vb, (long)Hkv * D, len, len - 1, window, scale, sinks[h], D,
                out + r * D, &lse[r]);
    }
}

/*
 * Backward, derived from the definition (the pages give no gradient).  With
 * P_ij = exp(z_ij - LSE_i), P_sink_i = exp(sink_h - LSE_i), D_i = <dO_i, O_i>:
 *   dS_ij   = P_ij (<dO_i, v_j> - D_i)
 *   dq_i    = scale * sum_j dS_ij k_j
 *   dk_j    = scale * sum_{h in group, i} dS_ij q_i
 *   dv_j    = sum_{h in group, i} P_ij dO_i
 *   dsink_h = - sum_{b, i} P_sink_i D_i          (since dO_i/dsink = -P_sink_i O_i)
 * Pass 1 runs per query row (dq, D, P_sink); pass 2 runs per key (dk, dv),
 * recomputing P and dS for every row that sees the key.  O and LSE are
 * recomputed here in fp64; nothing is taken from any other implementation.
 */
void oracle_bwd(const double *q, const double *k, const double *v, const double *sinks,
                const double *dout, double *dq, double *dk, double *dv, double *dsinks,
                int B, int Lq, int Lk, int Hq, int Hkv, int D, int window, double scale)
{
    const int G = Hq / Hkv;
    const long nrows = (long)B * Hq * Lq;
    const long off = (long)Lk - Lq;
    double *LSE = (double *)malloc(sizeof(double) * nrows);
    double *Dr = (double *)malloc(sizeof(double) * nrows);
    double *Ps = (double *)malloc(sizeof(double) * nrows);

    /* pass 1: per query row */
#pragma omp parallel
    {
        double *o = (double *)malloc(sizeof(double) * D);
#pragma omp for schedule(dynamic, 16)
        for (long r = 0; r < nrows; ++r) {
            const int b = (int)(r / ((long)Hq * Lq));
            const int h = (int)((r / Lq) % Hq);
            const int i = (int)(r % Lq);
            const int g = h / G;
            const long p = i + off;
            const double *qi = q + (((long)b * Lq + i) * Hq + h) * D;
            const double *doi = dout + (((long)b * Lq + i) * Hq + h) * D;
            const double *kb = k + ((long)b * Lk * Hkv + g) * D;
            const double *vb = v + ((long)b * Lk * Hkv + g) * D;
            double *dqi = dq + (((long)b * Lq + i) * Hq + h) * D;
            double lse;
            fwd_row(qi, kb, vb, (long)Hkv * D, Lk, p, window, scale, sinks[h], D, o, &lse);
            const double Di = dot(doi, o, D);
            LSE[r] = lse;
            Dr[r] = Di;
            Ps[r] = (lse == -INFINITY) ? 0.0 : exp(sinks[h] - lse);
            for (int d = 0; d < D; ++d) dqi[d] = 0.0;
            if (lse == -INFINITY) continue;
            for (long j = 0; j < Lk; ++j) {
                if (!key_visible(j, p, window)) continue;
                const double *kj = kb + j * (long)Hkv * D;
                const double *vj = vb + j * (long)Hkv * D;
                const double P = exp(scale * dot(qi, kj, D) - lse);
                const double dS = P * (dot(doi, vj, D) - Di);
                for (int d = 0; d < D; ++d) dqi[d] += scale * dS * kj[d];
            }
        }
        free(o);
    }

    /* pass 2: per key */
#pragma omp parallel for schedule(dynamic, 16)
    for (long kr = 0; kr < (long)B * Hkv * Lk; ++kr) {
        const int b = (int)(kr / ((long)Hkv * Lk));
        const int g = (int)((kr / Lk) % Hkv);
        const long j = kr % Lk;
        const double *kj = k + (((long)b * Lk + j) * Hkv + g) * D;
        const double *vj = v + (((long)b * Lk + j) * Hkv + g) * D;
        double *dkj = dk + (((long)b * Lk + j) * Hkv + g) * D;
        double *dvj = dv + (((long)b * Lk + j) * Hkv + g) * D;
        for (int d = 0; d < D; ++d) { dkj[d] = 0.0; dvj[d] = 0.0; }
        for (int h = g * G; h < (g + 1) * G; ++h) {
            for (int i = 0; i < Lq; ++i) {
                const long p = i + off;
                if (!key_visible(j, p, window)) continue;
                const long r = ((long)b * Hq + h) * Lq + i;
                if (LSE[r] == -INFINITY) continue;
                const double *qi = q + (((long)b * Lq + i) * Hq + h) * D;
                const double *doi = dout + (((long)b * Lq + i) * Hq + h) * D;
                const double P = exp(scale * dot(qi, kj, D) - LSE[r]);
                const double dS = P * (dot(doi, vj, D) - Dr[r]);
                for (int d = 0; d < D; ++d) {
                    dvj[d] += P * doi[d];
                    dkj[d] += scale * dS * qi[d];
                }
            }
        }
    }

    /* dsink: fixed serial order over (b, i) per head */
    for (int h = 0; h < Hq; ++h) {
        double s = 0.0;
        for (int b = 0; b < B; ++b)
            for (int i = 0; i < Lq; ++i) {
                const long r = ((long)b * Hq + h) * Lq + i;
                s -= Ps[r] * Dr[r];
            }
        dsinks[h] = s;
    }
    free(LSE);
    free(Dr);
    free(Ps);
}

/*
 * Row statistics needed by dsink, for a whole problem: D_i and P_sink_i per
 * row ([B, Hq, Lq] each), from a full fp64 forward.  Lets a test check the
 * dsink reduction at sizes where the full backward is too slow.
 */
void oracle_row_stats(const double *q, const double *k, const double *v, const double *sinks,
                      const double *dout, double *Drow, double *Psink, int B, int Lq, int Lk,
                      int Hq, int Hkv, int D, int window, double scale)
{
    const int G = Hq / Hkv;
    const long nrows = (long)B * Hq * Lq;
#pragma omp parallel
    {
        double *o = (double *)malloc(sizeof(double) * D);
#pragma omp for schedule(dynamic, 16)
        for (long r = 0; r < nrows; ++r) {
            const int b = (int)(r / ((long)Hq * Lq));
            const int h = (int)((r / Lq) % Hq);
            const int i = (int)(r % Lq);
            const int g = h / G;
            const double *qi = q + (((long)b * Lq + i) * Hq + h) * D;
            const double *doi = dout + (((long)b * Lq + i) * Hq + h) * D;
            double lse;
            fwd_row(qi, k + ((long)b * Lk * Hkv + g) * D, v + ((long)b * Lk * Hkv + g) * D,
                    (long)Hkv * D, Lk, (long)i + (Lk - Lq), window, scale, sinks[h], D, o, &lse);
            Drow[r] = dot(doi, o, D);
            Psink[r] = (lse == -INFINITY) ? 0.0 : exp(sinks[h] - lse);
        }
        free(o);
    }
}

int oracle_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
    return n;
}
