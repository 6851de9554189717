/*
 * WavePrune causal attention: plain, slow fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the bench's
 * CPU-baseline leg may load this file's library. It shares no code, header,
 * table or helper with the CUDA library; neither side includes the other.
 *
 * Every step is written straight from the pages' definitions, in their order,
 * with no blocking, fusion or reordering. Sources, cited by tag below:
 *   [RN] "WavePrune：RoPE 通常只需一个旋转周期" — reading notes of
 *        arXiv:2610.06963 (cc.laoqi.cc). Primary authority.
 *   [KC] "WavePrune：RoPE只用一个旋转周期，长文本性能反而更好" (kongchang.com).
 *   [TW] "Guancheng Du @ducatiqwq" — the author's thread, posts (3/7) and (6/7).
 *
 * Readings taken where the pages are silent (listed again in the design notes):
 *   - half-split rotation layout pairs dims (c, c + d_h/2), like rotate_half;
 *   - a frequency scale multiplies f_c and is used for both angle and cutoff;
 *   - the logsumexp is natural-log and includes the softmax scale;
 *   - GQA maps query head h to KV head h / (Hq / Hkv).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define WPO_INTERLEAVED 0
#define WPO_HALF_SPLIT 1
#define WPO_MODE_GROUPED 0
#define WPO_MODE_CHANNEL 1
#define WPO_PI 3.14159265358979323846

/* ------------------------------------------------------------------------- */
/* Frequencies and cutoffs                                                   */
/* ------------------------------------------------------------------------- */

/* [RN §1.1, paper Eq. (2)-(5)]: channel c rotates by f_c = theta^(-2c/d_h)
 * radians per token, c = 0 .. d_h/2 - 1. [RN §1.1 last paragraph]: with
 * frequency scaling the cutoffs come from the scaled (actual) frequencies,
 * so the scale multiplies f_c. */
double wpo_freq(int c, int d_h, double theta, const double *freq_scale, double scale_all)
{
    double f = pow(theta, -2.0 * (double)c / (double)d_h);
    if (freq_scale)
        f *= freq_scale[c];
    return f * scale_all;
}

/* [RN §2.1, text after Eq. (6)]: threshold w_c = alpha*pi/f_c (alpha = 2 is one
 * period, w_c = 2*pi/f_c); distances are integers, so channel c is kept iff
 * distance <= floor(w_c). Saturates at INT32_MAX. */
int32_t wpo_channel_cutoff(double f, double alpha)
{
    double w = alpha * WPO_PI / f;
    double fl = floor(w);
    if (!(fl < 2147483647.0))
        return INT32_MAX;
    return (int32_t)fl;
}

/* The RoPE channel that owns head dim k.
 * Interleaved [KC, RoPE matrix]: channel i rotates the pair (x_{2i}, x_{2i+1}).
 * Half-split (reading): channel c rotates the pair (x_c, x_{c + d_h/2}). */
static int owner_channel(int k, int d_h, int layout)
{
    return layout == WPO_INTERLEAVED ? k / 2 : k % (d_h / 2);
}

/* The two dims of channel c (a, b), rotated as [[cos, -sin], [sin, cos]]. */
static void channel_dims(int c, int d_h, int layout, int *a, int *b)
{
    if (layout == WPO_INTERLEAVED) {
        *a = 2 * c;
        *b = 2 * c + 1;
    } else {
        *a = c;
        *b = c + d_h / 2;
    }
}

/* Per-channel cutoffs W_c [d_h/2] and per-group cutoffs W_g [d_h/16].
 * [RN §2.3, paper Eq. (8)]: 16 scalar head dims form group g, and
 * d'_g = max over the dims k of the group of d_k, where d_k is the cutoff of
 * the channel that dim k belongs to. */
int wpo_cutoffs(int d_h, double theta, const double *freq_scale, double scale_all, double alpha, int layout,
                int32_t *chan_cut, int32_t *group_cut)
{
    if (d_h <= 0 || d_h % 16 != 0)
        return 1;
    int C = d_h / 2, G = d_h / 16;
    for (int c = 0; c < C; ++c)
        chan_cut[c] = wpo_channel_cutoff(wpo_freq(c, d_h, theta, freq_scale, scale_all), alpha);
    for (int g = 0; g < G; ++g) {
        int32_t m = INT32_MIN;
        for (int k = 16 * g; k < 16 * g + 16; ++k) {
            int32_t w = chan_cut[owner_channel(k, d_h, layout)];
            if (w > m)
                m = w;
        }
        group_cut[g] = m;
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* RoPE                                                                      */
/* ------------------------------------------------------------------------- */

/* [KC, RoPE paragraph]: the pair of channel c at position m is multiplied by
 * [[cos(m f_c), -sin(m f_c)], [sin(m f_c), cos(m f_c)]]. [RN §1.1]: the query
 * channel at position i is rotated by i*f_c. Angle and rotation in fp64.
 * x, y: [B][N][H][d_h]; pos: [B][N] or NULL (then position = pos0 + t). */
void wpo_rope(const double *x, double *y, int64_t B, int64_t N, int H, int d_h, const int64_t *pos, int64_t pos0,
              double theta, const double *freq_scale, double scale_all, int layout)
{
    int C = d_h / 2;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t t = 0; t < N; ++t) {
            double p = pos ? (double)pos[b * N + t] : (double)(pos0 + t);
            for (int h = 0; h < H; ++h) {
                const double *xr = x + ((b * N + t) * H + h) * d_h;
                double *yr = y + ((b * N + t) * H + h) * d_h;
                for (int c = 0; c < C; ++c) {
                    int a, bb;
                    channel_dims(c, d_h, layout, &a, &bb);
                    double ang = p * wpo_freq(c, d_h, theta, freq_scale, scale_all);
                    double cs = cos(ang), sn = sin(ang);
                    double xa = xr[a], xb = xr[bb];
                    yr[a] = xa * cs - xb * sn;
                    yr[bb] = xa * sn + xb * cs;
                }
            }
        }
}

/* Round fp64 to the nearest bf16 (ties to even), returned as raw bits.
 * Directly from the double (no intermediate fp32 rounding). Finite values in
 * the normal bf16 range; zero keeps its sign. */
void wpo_round_bf16(const double *x, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) {
        double v = x[i];
        uint16_t sign = signbit(v) ? 0x8000u : 0u;
        double a = fabs(v);
        if (a == 0.0) {
            out[i] = sign;
            continue;
        }
        int e;
        double m = frexp(a, &e);            /* a = m * 2^e, m in [0.5, 1) */
        double k = nearbyint(ldexp(m, 8));  /* 8 significant bits, ties to even */
        float f = (float)ldexp(k, e - 8);   /* exact: k has at most 9 bits */
        uint32_t u;
        memcpy(&u, &f, 4);
        out[i] = (uint16_t)(sign | (u >> 16));
    }
}

/* ------------------------------------------------------------------------- */
/* WavePrune logits and attention                                            */
/* ------------------------------------------------------------------------- */

/* One causal logit (j <= i, dist = i - j).
 * Channel mode, [RN §2.1, paper Eq. (6)] and [TW (3/7)]:
 *   L = scale * sum_c phi^(c)(q)^T phi^(c)(k) * 1[dist <= W_c],
 * where the channel-c inner product is q_a k_a + q_b k_b over its two dims.
 * Grouped mode, [RN §2.3, paper Eq. (8)] and [TW (6/7)]: each 16-dim group runs
 * a plain dot product, and the group's single mask 1[dist <= W_g] is applied
 * to its result.
 * [RN §2.1, detail 1]: a dropped term is 0 (not -inf). [RN §2.1, detail 3]:
 * the scale is not renormalised by the number of kept channels. */
static double wp_logit(const double *q, const double *k, int64_t dist, int d_h, int mode, int layout,
                       const int32_t *cut, double scale)
{
    double acc = 0.0;
    if (mode == WPO_MODE_CHANNEL) {
        int C = d_h / 2;
        for (int c = 0; c < C; ++c) {
            if (dist > (int64_t)cut[c])
                continue;
            int a, b;
            channel_dims(c, d_h, layout, &a, &b);
            acc += q[a] * k[a] + q[b] * k[b];
        }
    } else {
        int G = d_h / 16;
        for (int g = 0; g < G; ++g) {
            if (dist > (int64_t)cut[g])
                continue;
            double s = 0.0;
            for (int t = 16 * g; t < 16 * g + 16; ++t)
                s += q[t] * k[t];
            acc += s;
        }
    }
    return scale * acc;
}

/* Full logit matrix of one head, L[i][j] for j <= i and -inf above the
 * diagonal ([RN §2.1]: future tokens keep the causal -inf). q, k: [N][d_h]. */
void wpo_logits(const double *q, const double *k, int64_t N, int d_h, int mode, int layout, const int32_t *cut,
                double scale, double *L)
{
    for (int64_t i = 0; i < N; ++i)
        for (int64_t j = 0; j < N; ++j)
            L[i * N + j] = j <= i ? wp_logit(q + i * d_h, k + j * d_h, i - j, d_h, mode, layout, cut, scale)
                                  : -INFINITY;
}

/* Softmax over the causal logits and the value average of one query row
 * ([RN §2.1, the formula after Eq. (6)]: A_ij = exp L_ij / sum_{k<=i} exp L_ik,
 * Y = A V). krow(j)/vrow(j) give key/value j. Writes o[d_h] and returns
 * LSE = ln sum_j exp L_ij (computed with the row max subtracted). */
static double attend_row(const double *q, const double *kbase, int64_t kstride, const double *vbase,
                         int64_t vstride, int64_t i, int d_h, int mode, int layout, const int32_t *cut,
                         double scale, double *L, double *o)
{
    double m = -INFINITY;
    for (int64_t j = 0; j <= i; ++j) {
        L[j] = wp_logit(q, kbase + j * kstride, i - j, d_h, mode, layout, cut, scale);
        if (L[j] > m)
            m = L[j];
    }
    double s = 0.0;
    for (int64_t j = 0; j <= i; ++j)
        s += exp(L[j] - m);
    double lse = m + log(s);
    for (int t = 0; t < d_h; ++t)
        o[t] = 0.0;
    for (int64_t j = 0; j <= i; ++j) {
        double a = exp(L[j] - lse);
        const double *vj = vbase + j * vstride;
        for (int t = 0; t < d_h; ++t)
            o[t] += a * vj[t];
    }
    return lse;
}

/* Causal prefill attention for a list of R query rows (b, h, i), positions
 * 0..N-1 so that distance = i - j. q_rows: [R][d_h] (the rows' query vectors);
 * k, v: [B][N][Hkv][d_h]. Outputs o [R][d_h], lse [R]. */
int wpo_attention_rows(const double *q_rows, const int64_t *row_b, const int64_t *row_h, const int64_t *row_i,
                       int64_t R, const double *k, const double *v, int64_t B, int64_t N, int Hq, int Hkv, int d_h,
                       int mode, int layout, const int32_t *cut, double scale, double *o, double *lse, int nthreads)
{
    if (Hkv <= 0 || Hq % Hkv != 0)
        return 1;
    int rep = Hq / Hkv;
    int64_t kstride = (int64_t)Hkv * d_h;
    int err = 0;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        double *L = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        if (!L) {
#pragma omp atomic write
            err = 2;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < R; ++r) {
            if (!L)
                continue;
            int64_t b = row_b[r], h = row_h[r], i = row_i[r];
            if (b < 0 || b >= B || h < 0 || h >= Hq || i < 0 || i >= N) {
#pragma omp atomic write
                err = 3;
                continue;
            }
            int64_t hk = h / rep;
            const double *kb = k + (b * N * Hkv + hk) * d_h;
            const double *vb = v + (b * N * Hkv + hk) * d_h;
            lse[r] = attend_row(q_rows + r * d_h, kb, kstride, vb, kstride, i, d_h, mode, layout, cut, scale, L,
                                o + r * d_h);
        }
        free(L);
    }
    return err;
}

/* Decode: one new query per sequence at position len_b - 1, keys 0..len_b-1
 * from the cache, grouped cutoffs ([RN §2.3 table, first row]: in decode a
 * skipped group's K is not needed). q: [B][Hq][d_h]; kc, vc: [B][Hkv][Lmax][d_h];
 * lens: [B]. Outputs o [B][Hq][d_h], lse [B][Hq]. This is row len-1 of the
 * prefill definition over the cached keys. */
int wpo_decode(const double *q, const double *kc, const double *vc, const int32_t *lens, int64_t B, int Hq, int Hkv,
               int d_h, int64_t Lmax, const int32_t *group_cut, double scale, double *o, double *lse, int nthreads)
{
    if (Hkv <= 0 || Hq % Hkv != 0)
        return 1;
    for (int64_t b = 0; b < B; ++b)
        if (lens[b] < 1 || lens[b] > Lmax)
            return 3;
    int rep = Hq / Hkv;
    int err = 0;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        double *L = (double *)malloc(sizeof(double) * (size_t)Lmax);
        if (!L) {
#pragma omp atomic write
            err = 2;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t bh = 0; bh < B * Hq; ++bh) {
            if (!L)
                continue;
            int64_t b = bh / Hq, h = bh % Hq, hk = h / rep;
            int64_t len = lens[b];
            const double *kb = kc + (b * Hkv + hk) * Lmax * d_h;
            const double *vb = vc + (b * Hkv + hk) * Lmax * d_h;
            lse[bh] = attend_row(q + bh * d_h, kb, d_h, vb, d_h, len - 1, d_h, WPO_MODE_GROUPED, 0, group_cut,
                                 scale, L, o + bh * d_h);
        }
        free(L);
    }
    return err;
}

/* ------------------------------------------------------------------------- */
/* Backward: gradients of the prefill definition                             */
/* ------------------------------------------------------------------------- */

/* [RN §2.3, the paragraph on the backward kernel; §4.6, Table 4] describes a
 * backward kernel (gradient operands masked before the MMA, dQ and dK formed
 * together under one mask) but prints no equations. The oracle therefore
 * differentiates the forward definition itself, by the chain rule, one step
 * per line of the forward pass:
 *   forward   L_ij = scale * sum_u 1[i - j <= W_u] <q_i[u], k_j[u]>  (j <= i)
 *             P_ij = exp(L_ij - LSE_i),   O_i = sum_j P_ij v_j
 *   backward  dV_j += P_ij dO_i
 *             dP_ij = <dO_i, v_j>
 *             dL_ij = P_ij (dP_ij - D_i),   D_i = sum_j P_ij dP_ij = <dO_i, O_i>
 *             dq_i[u] += scale * 1[i - j <= W_u] * dL_ij * k_j[u]
 *             dk_j[u] += scale * 1[i - j <= W_u] * dL_ij * q_i[u]
 * where u runs over channels (their two dims) in channel mode and over 16-dim
 * groups in grouped mode. A masked unit contributes nothing to either
 * gradient, exactly as it contributes 0 to the logit. */
static void logit_grad(const double *q, const double *k, int64_t dist, int d_h, int mode, int layout,
                       const int32_t *cut, double scale, double dl, double *dq, double *dk)
{
    double s = scale * dl;
    if (mode == WPO_MODE_CHANNEL) {
        int C = d_h / 2;
        for (int c = 0; c < C; ++c) {
            if (dist > (int64_t)cut[c])
                continue;
            int a, b;
            channel_dims(c, d_h, layout, &a, &b);
            dq[a] += s * k[a];
            dq[b] += s * k[b];
            dk[a] += s * q[a];
            dk[b] += s * q[b];
        }
    } else {
        int G = d_h / 16;
        for (int g = 0; g < G; ++g) {
            if (dist > (int64_t)cut[g])
                continue;
            for (int t = 16 * g; t < 16 * g + 16; ++t) {
                dq[t] += s * k[t];
                dk[t] += s * q[t];
            }
        }
    }
}

/* Gradients of sum(dO * O) for causal prefill over positions 0..N-1.
 * q, dout, dq: [B][N][Hq][d_h]; k, v, dk, dv: [B][N][Hkv][d_h]. The query
 * heads sharing a KV head (GQA, h -> h / (Hq / Hkv)) add into its dk, dv.
 * cut: channel cutoffs [d_h/2] (channel mode) or group cutoffs [d_h/16]. */
int wpo_attention_backward(const double *q, const double *k, const double *v, const double *dout, int64_t B,
                           int64_t N, int Hq, int Hkv, int d_h, int mode, int layout, const int32_t *cut,
                           double scale, double *dq, double *dk, double *dv, int nthreads)
{
    if (Hkv <= 0 || Hq % Hkv != 0 || N <= 0 || B <= 0)
        return 1;
    int rep = Hq / Hkv;
    int64_t qs = (int64_t)Hq * d_h, ks = (int64_t)Hkv * d_h;
    for (int64_t e = 0; e < B * N * qs; ++e)
        dq[e] = 0.0;
    for (int64_t e = 0; e < B * N * ks; ++e)
        dk[e] = dv[e] = 0.0;
    int err = 0;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#endif
#pragma omp parallel
    {
        double *L = (double *)malloc(sizeof(double) * (size_t)N);
        double *o = (double *)malloc(sizeof(double) * (size_t)d_h);
        if (!L || !o) {
#pragma omp atomic write
            err = 2;
        }
        /* one thread per (b, KV head): it owns that head's dk, dv */
#pragma omp for schedule(dynamic, 1)
        for (int64_t bk = 0; bk < B * Hkv; ++bk) {
            if (!L || !o)
                continue;
            int64_t b = bk / Hkv, hk = bk % Hkv;
            const double *kb = k + (b * N * Hkv + hk) * d_h;
            const double *vb = v + (b * N * Hkv + hk) * d_h;
            double *dkb = dk + (b * N * Hkv + hk) * d_h;
            double *dvb = dv + (b * N * Hkv + hk) * d_h;
            for (int64_t h = hk * rep; h < (hk + 1) * rep; ++h)
                for (int64_t i = 0; i < N; ++i) {
                    const double *qi = q + ((b * N + i) * Hq + h) * d_h;
                    const double *doi = dout + ((b * N + i) * Hq + h) * d_h;
                    double *dqi = dq + ((b * N + i) * Hq + h) * d_h;
                    double lse = attend_row(qi, kb, ks, vb, ks, i, d_h, mode, layout, cut, scale, L, o);
                    double D = 0.0;
                    for (int t = 0; t < d_h; ++t)
                        D += doi[t] * o[t];
                    for (int64_t j = 0; j <= i; ++j) {
                        double p = exp(L[j] - lse);
                        const double *vj = vb + j * ks;
                        double dp = 0.0;
                        for (int t = 0; t < d_h; ++t) {
                            dp += doi[t] * vj[t];
                            dvb[j * ks + t] += p * doi[t];
                        }
                        double dl = p * (dp - D);
                        logit_grad(qi, kb + j * ks, i - j, d_h, mode, layout, cut, scale, dl, dqi, dkb + j * ks);
                    }
                }
        }
        free(L);
        free(o);
    }
    return err;
}

/* ------------------------------------------------------------------------- */
/* Tile classes by brute force                                               */
/* ------------------------------------------------------------------------- */

/* [RN §2.3, the three-row table] and [TW (6/7)]: for a (query block, key block)
 * the distances i - j of its causal pairs span [l_D, r_D]; a group with cutoff
 * d' is skipped if d' < l_D, computed without a mask if d' >= r_D, and masked
 * otherwise. Here l_D and r_D are found by visiting every pair with j <= i.
 * cls (optional): [nqb][nkb][ncut], 0 skip / 1 full / 2 boundary / 3 = the
 * tile has no causal pair. counts: [ncut][3] (skip, full, boundary). */
int wpo_tile_classes(int64_t N, int BM, int BN, const int32_t *cut, int ncut, uint8_t *cls, int64_t *counts)
{
    if (N <= 0 || BM <= 0 || BN <= 0 || ncut <= 0)
        return 1;
    int64_t nqb = (N + BM - 1) / BM, nkb = (N + BN - 1) / BN;
    for (int g = 0; g < ncut; ++g)
        counts[3 * g] = counts[3 * g + 1] = counts[3 * g + 2] = 0;
    for (int64_t qb = 0; qb < nqb; ++qb)
        for (int64_t kb = 0; kb < nkb; ++kb) {
            int64_t lo = INT64_MAX, hi = -1;
            for (int64_t i = qb * BM; i < (qb + 1) * BM && i < N; ++i)
                for (int64_t j = kb * BN; j < (kb + 1) * BN && j < N; ++j) {
                    if (j > i)
                        continue;
                    int64_t dist = i - j;
                    if (dist < lo)
                        lo = dist;
                    if (dist > hi)
                        hi = dist;
                }
            for (int g = 0; g < ncut; ++g) {
                int c;
                if (hi < 0)
                    c = 3;
                else if ((int64_t)cut[g] < lo)
                    c = 0;
                else if ((int64_t)cut[g] >= hi)
                    c = 1;
                else
                    c = 2;
                if (cls)
                    cls[(qb * nkb + kb) * ncut + g] = (uint8_t)c;
                if (c < 3)
                    counts[3 * g + c] += 1;
            }
        }
    return 0;
}
