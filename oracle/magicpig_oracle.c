/*
 * MagicPIG LSH-sampled decode attention: plain fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library. It shares no
 * code, header, table or constant with the CUDA library; the two meet only
 * through the seeded input generator, which holds none of the method's
 * arithmetic.
 *
 * What it computes (method: "MagicPIG: LSH Sampling for Efficient LLM
 * Generation", Chen et al., 2024; the GrooveSquid summary page, medium
 * difficulty summary, states that the method estimates the attention output
 * by sampling rather than by TopK selection, and the sourcepulse project page,
 * "How It Works", states that the samples are chosen by locality-sensitive
 * hashing):
 *
 *   1. SimHash.  Every key k and query q (dimension d) is projected onto L*K
 *      random hyperplanes w_c (c = l*K + b).  Bit b of the table-l code is 1
 *      exactly when the projection k . w_c is strictly positive (a projection
 *      of exactly zero gives bit 0).  The code of table l is the K-bit integer
 *      sum_b bit_b * 2^b.
 *   2. Sampling rule.  Context token i (outside the exact set D) belongs to
 *      the sampled set S_h of query head h when its code equals the query's
 *      code in at least two of the L tables.
 *   3. Sampling probability.  With p_i = 1 - arccos(cos(q, k_i)) / pi (the
 *      SimHash per-bit collision probability) and x = p_i^K (per-table
 *      collision probability), u_i = P[Binomial(L, x) >= 2]
 *      = 1 - (1-x)^L - L x (1-x)^(L-1).  The oracle evaluates u as the plain
 *      sum over j = 2..L of C(L,j) x^j (1-x)^(L-j) (every term positive, no
 *      cancellation); the closed form is a test cross-check.
 *   4. Estimator.  With s_i = q . k_i / sqrt(d), w_i = exp(s_i) on the exact
 *      set D = [0, sink) U [N - window, N) and w_i = exp(s_i - log u_i) on S_h,
 *      the output is o = sum w_i v_i / sum w_i over D U S_h, and
 *      lse = log sum w_i.  S_h excludes D, so no token is counted twice.
 *
 * All arithmetic is fp64.  bf16 inputs arrive as raw 16-bit patterns and are
 * widened exactly.  No blocking, fusion or reordering beyond the definitions
 * above; a max shift is applied before exponentiation for range only.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define MPO_PI 3.14159265358979323846

/* Exact widening of a bf16 bit pattern (the upper half of an IEEE binary32). */
static double mpo_bf16(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int mpo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Step 1, SimHash codes of n rows x[r][0..d) against W[c][0..d), c < L*K.
 * codes[r*L + l] = sum_b [x_r . w_{l*K+b} > 0] << b.
 * margin (nullable) [n][L*K]: |x_r . w_c| / (||x_r|| ||w_c||), the relative
 * distance of the projection from the hyperplane; 0 when a norm is 0.
 */
void mpo_simhash(const uint16_t *x, int64_t n, int d, const uint16_t *W, int K, int L,
                 uint16_t *codes, double *margin)
{
    const int LK = L * K;
    double *wn = (double *)malloc(sizeof(double) * (LK > 0 ? LK : 1));
    for (int c = 0; c < LK; c++) {
        double s = 0.0;
        for (int j = 0; j < d; j++) {
            double w = mpo_bf16(W[(int64_t)c * d + j]);
            s += w * w;
        }
        wn[c] = sqrt(s);
    }
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; r++) {
        const uint16_t *xr = x + r * d;
        double xn = 0.0;
        for (int j = 0; j < d; j++) {
            double v = mpo_bf16(xr[j]);
            xn += v * v;
        }
        xn = sqrt(xn);
        for (int l = 0; l < L; l++) {
            unsigned code = 0;
            for (int b = 0; b < K; b++) {
                const int c = l * K + b;
                double dot = 0.0;
                for (int j = 0; j < d; j++)
                    dot += mpo_bf16(xr[j]) * mpo_bf16(W[(int64_t)c * d + j]);
                if (dot > 0.0)
                    code |= 1u << b;
                if (margin) {
                    double den = xn * wn[c];
                    margin[r * LK + c] = den > 0.0 ? fabs(dot) / den : 0.0;
                }
            }
            codes[r * L + l] = (uint16_t)code;
        }
    }
    free(wn);
}

/* Step 3, SimHash per-bit collision probability p = 1 - arccos(cos)/pi.
 * A zero-norm vector is orthogonal to everything: p = 1/2. */
double mpo_collision_prob(const double *q, const double *k, int d)
{
    double dot = 0.0, qq = 0.0, kk = 0.0;
    for (int j = 0; j < d; j++) {
        dot += q[j] * k[j];
        qq += q[j] * q[j];
        kk += k[j] * k[j];
    }
    if (qq == 0.0 || kk == 0.0)
        return 0.5;
    double c = dot / (sqrt(qq) * sqrt(kk));
    if (c > 1.0)
        c = 1.0;
    if (c < -1.0)
        c = -1.0;
    return 1.0 - acos(c) / MPO_PI;
}

/* Step 3, u = P[at least 2 of L independent tables collide], each table with
 * probability x = p^K: the sum over j = 2..L of C(L,j) x^j (1-x)^(L-j). */
double mpo_sampling_prob(double p, int K, int L)
{
    if (L < 2)
        return 0.0;
    const double x = pow(p, (double)K);
    if (x <= 0.0)
        return 0.0;
    if (x >= 1.0)
        return 1.0;
    double u = 0.0;
    double binom = 1.0; /* C(L, j), by the multiplicative recurrence */
    for (int j = 1; j <= L; j++) {
        binom = binom * (double)(L - j + 1) / (double)j;
        if (j >= 2)
            u += binom * pow(x, (double)j) * pow(1.0 - x, (double)(L - j));
    }
    return u > 1.0 ? 1.0 : u;
}

/* Step 2, membership of S_h for one (batch, kv head) unit given the codes.
 * kcodes [N][L], qcodes [G][L]; member [G][N] (1 = in S_h); n_sampled [G].
 * Tokens of D never enter S_h. */
void mpo_collide(const uint16_t *kcodes, const uint16_t *qcodes, int N, int L, int G,
                 int sink, int window, uint8_t *member, int32_t *n_sampled)
{
    for (int h = 0; h < G; h++) {
        int32_t cnt = 0;
        for (int i = 0; i < N; i++) {
            int in_d = (i < sink) || (i >= N - window);
            int matches = 0;
            for (int l = 0; l < L; l++)
                if (kcodes[(int64_t)i * L + l] == qcodes[h * L + l])
                    matches++;
            int in_s = !in_d && matches >= 2;
            member[(int64_t)h * N + i] = (uint8_t)in_s;
            cnt += in_s;
        }
        n_sampled[h] = cnt;
    }
}

/* Step 4, the estimator for one query head over N context rows.
 * member [N] marks S_h; D is derived from sink/window.  out [d], lse [1].
 * With D and S_h both empty the output is 0 and lse is -inf. */
void mpo_attend(const uint16_t *q, const uint16_t *Kr, const uint16_t *Vr, int N, int d,
                const uint8_t *member, int sink, int window, int K, int L,
                double *out, double *lse)
{
    double *qd = (double *)malloc(sizeof(double) * d);
    double *kd = (double *)malloc(sizeof(double) * d);
    double *t = (double *)malloc(sizeof(double) * (N > 0 ? N : 1));
    const double scale = 1.0 / sqrt((double)d);
    for (int j = 0; j < d; j++)
        qd[j] = mpo_bf16(q[j]);
    double m = -INFINITY;
    for (int i = 0; i < N; i++) {
        int in_d = (i < sink) || (i >= N - window);
        int in_s = !in_d && member[i];
        t[i] = -INFINITY;
        if (!in_d && !in_s)
            continue;
        double dot = 0.0;
        for (int j = 0; j < d; j++) {
            kd[j] = mpo_bf16(Kr[(int64_t)i * d + j]);
            dot += qd[j] * kd[j];
        }
        double s = dot * scale;
        if (in_s) {
            double p = mpo_collision_prob(qd, kd, d);
            double u = mpo_sampling_prob(p, K, L);
            s -= log(u);
        }
        t[i] = s;
        if (s > m)
            m = s;
    }
    for (int j = 0; j < d; j++)
        out[j] = 0.0;
    double z = 0.0;
    if (m > -INFINITY) {
        for (int i = 0; i < N; i++) {
            if (t[i] == -INFINITY)
                continue;
            double w = exp(t[i] - m);
            z += w;
            for (int j = 0; j < d; j++)
                out[j] += w * mpo_bf16(Vr[(int64_t)i * d + j]);
        }
        for (int j = 0; j < d; j++)
            out[j] /= z;
        *lse = m + log(z);
    } else {
        *lse = -INFINITY;
    }
    free(qd);
    free(kd);
    free(t);
}

/*
 * One decode step over a batch, given codes: for every (b, kv head) unit and
 * every query head h of its group, S_h by step 2 and the estimate by step 4.
 *   q       [B][Hq][d]          K, V [B][Hkv][Ncap][d]     (bf16 bits)
 *   kcodes  [B][Hkv][Ncap][L]   qcodes [B][Hq][L]
 *   seq_lens[B]                 member (nullable) [B][Hq][Ncap]
 *   out     [B][Hq][d]          lse [B][Hq]      n_sampled [B][Hq]
 * Query head h reads kv head h / (Hq / Hkv).  Units run in parallel.
 */
void mpo_decode(const uint16_t *q, const uint16_t *K, const uint16_t *V,
                const uint16_t *kcodes, const uint16_t *qcodes, const int32_t *seq_lens,
                int B, int Hq, int Hkv, int d, int Ncap, int Kbits, int L, int sink, int window,
                uint8_t *member, double *out, double *lse, int32_t *n_sampled)
{
    const int G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int b = 0; b < B; b++) {
        for (int kh = 0; kh < Hkv; kh++) {
            const int N = seq_lens[b];
            const int64_t unit = (int64_t)b * Hkv + kh;
            uint8_t *mem = (uint8_t *)malloc((size_t)G * (N > 0 ? N : 1));
            int32_t *cnt = (int32_t *)malloc(sizeof(int32_t) * G);
            mpo_collide(kcodes + unit * Ncap * L, qcodes + ((int64_t)b * Hq + kh * G) * L,
                        N, L, G, sink, window, mem, cnt);
            for (int g = 0; g < G; g++) {
                const int h = kh * G + g;
                const int64_t bh = (int64_t)b * Hq + h;
                mpo_attend(q + bh * d, K + unit * Ncap * d, V + unit * Ncap * d, N, d,
                           mem + (int64_t)g * N, sink, window, Kbits, L, out + bh * d, lse + bh);
                n_sampled[bh] = cnt[g];
                if (member) {
                    memset(member + bh * Ncap, 0, (size_t)Ncap);
                    memcpy(member + bh * Ncap, mem + (int64_t)g * N, (size_t)N);
                }
            }
            free(mem);
            free(cnt);
        }
    }
}
