/*
 * retnet_oracle.c -- plain, slow, fp64 CPU oracle for RetNet multi-scale retention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this library.  The CUDA product path never calls
 * it, links it or shares a line of code with it.
 *
 * Sources (cited by page title and section):
 *   [RN]  "阅读笔记：RetNet" (mzeromiko blog, reading notes on arXiv 2307.08621)
 *         §2.2 Recurrent Mode, §2.3 Parallel Mode, §2.4 Chunkwise Recurrent Mode,
 *         §三.2 Multi-Scale Retention (MSR), §三.3 Normalization.
 *
 * Readings taken where the page is silent (each restated where it is used):
 *   - xPos on real tensors: interleaved pairs (2j, 2j+1) are one complex
 *     coordinate; q and k of token p are both turned by the angle p*theta[j].
 *     Then the real dot product q'.k' equals Re[(q e^{in.theta})(k e^{im.theta})^dagger],
 *     which depends on n-m only ([RN] §2.1 last equation, §2.3 Theta_n).
 *   - Positions are 0-based absolute: token t of a call sits at p = pos0 + t.
 *   - The normalisations of [RN] §三.3 are per-row scalars:
 *       score_nm = (q_n.k_m) * s * gamma^(n-m) / c_n,  s = 1/sqrt(d_k) (flag),
 *       c_n = sqrt(sum_{j=0..p} gamma^j) with p the absolute position (flag),
 *       o_n = sum_m score_nm v_m / max(|sum_m score_nm|, 1)   (flag).
 *   - Chunk-local masks of [RN] §2.4 use 0-based row index r inside the chunk:
 *       zeta_r = gamma^(b'-1-r), xi_r = gamma^(r+1), with b' the chunk's actual
 *       length (shorter for a ragged tail chunk).
 *   - Recurrent order: the state is updated with token n before it is read.
 *
 * Layout ("BLHD", row-major): q,k: [batch][L][heads][d_k]; v,o: [batch][L][heads][d_v];
 * state: [batch][heads][d_k][d_v]; z (key-sum state): [batch][heads][d_k].
 * Every array is double.  Nothing here is blocked, fused or reordered beyond the
 * equations it follows; (batch, head) pairs are independent problems and are
 * spread over OpenMP threads.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_F_XPOS 1u
#define ORACLE_F_SCALE_SQRT_D 2u
#define ORACLE_F_NORM_D 4u
#define ORACLE_F_NORM_R 8u

typedef struct {
    int64_t batch, seqlen, heads, d_k, d_v;
} oracle_dims_t;

static inline const double *row_qk(const double *x, const oracle_dims_t *d, int64_t b, int64_t t, int64_t hh) {
    return x + ((b * d->seqlen + t) * d->heads + hh) * d->d_k;
}
static inline const double *row_v(const double *x, const oracle_dims_t *d, int64_t b, int64_t t, int64_t hh) {
    return x + ((b * d->seqlen + t) * d->heads + hh) * d->d_v;
}

/* xPos rotation of one row at absolute position p ([RN] §2.3: Q = (XW_Q) (.) Theta,
 * Theta_n = e^{in.theta}; K uses the conjugate, which on the real pair representation
 * with a real dot product is the same turn applied to k, see the header). */
static void xpos_rotate(const double *x, double *y, int64_t d, const double *theta, int64_t p, int on) {
    if (!on) {
        memcpy(y, x, sizeof(double) * (size_t)d);
        return;
    }
    for (int64_t j = 0; j < d / 2; ++j) {
        double a = (double)p * theta[j];
        double c = cos(a), s = sin(a);
        double x0 = x[2 * j], x1 = x[2 * j + 1];
        y[2 * j] = x0 * c - x1 * s;
        y[2 * j + 1] = x0 * s + x1 * c;
    }
}

static double dot(const double *a, const double *b, int64_t n) {
    double acc = 0.0;
    for (int64_t i = 0; i < n; ++i) acc += a[i] * b[i];
    return acc;
}

/* Per-row factor s / c_n of [RN] §三.3 (QK^T/sqrt(d) and the D~ row sum). */
static double row_factor(double gamma, int64_t d_k, int64_t p, unsigned flags) {
    double f = 1.0;
    if (flags & ORACLE_F_SCALE_SQRT_D) f /= sqrt((double)d_k);
    if (flags & ORACLE_F_NORM_D) {
        double rs = 0.0; /* sum_{j=0..p} D_{n,n-j} = sum gamma^j, written out */
        for (int64_t j = 0; j <= p; ++j) rs += pow(gamma, (double)j);
        f /= sqrt(rs);
    }
    return f;
}

static int set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
    return omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

/* Number of OpenMP threads the oracle will use for a call with nthreads (0 = default). */
int oracle_num_threads(int nthreads) { return set_threads(nthreads); }

/*
 * Parallel form, [RN] §2.3:  O = (Q K^T (.) D) V,  D_nm = gamma^(n-m) for n >= m else 0,
 * with the three normalisations of [RN] §三.3 applied as the flags ask.  This is the
 * plain quadratic definition: every score is formed, masked, scaled and summed.
 * No state enters: the call is a fresh sequence starting at absolute position pos0.
 */
int oracle_parallel(const double *q, const double *k, const double *v, double *o, oracle_dims_t d,
                    const double *gamma, const double *theta, int64_t pos0, unsigned flags, int nthreads) {
    set_threads(nthreads);
    const int xpos = (flags & ORACLE_F_XPOS) != 0;
    int64_t pairs = d.batch * d.heads;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < pairs; ++bh) {
        int64_t b = bh / d.heads, hh = bh % d.heads;
        double g = gamma[hh];
        double *qr = (double *)malloc(sizeof(double) * (size_t)(d.seqlen * d.d_k));
        double *kr = (double *)malloc(sizeof(double) * (size_t)(d.seqlen * d.d_k));
        double *acc = (double *)malloc(sizeof(double) * (size_t)d.d_v);
        for (int64_t t = 0; t < d.seqlen; ++t) {
            xpos_rotate(row_qk(q, &d, b, t, hh), qr + t * d.d_k, d.d_k, theta, pos0 + t, xpos);
            xpos_rotate(row_qk(k, &d, b, t, hh), kr + t * d.d_k, d.d_k, theta, pos0 + t, xpos);
        }
        for (int64_t n = 0; n < d.seqlen; ++n) {
            double f = row_factor(g, d.d_k, pos0 + n, flags);
            double sigma = 0.0;
            memset(acc, 0, sizeof(double) * (size_t)d.d_v);
            for (int64_t m = 0; m <= n; ++m) { /* D_nm = 0 for m > n */
                double score = dot(qr + n * d.d_k, kr + m * d.d_k, d.d_k) * pow(g, (double)(n - m)) * f;
                sigma += score;
                const double *vm = row_v(v, &d, b, m, hh);
                for (int64_t j = 0; j < d.d_v; ++j) acc[j] += score * vm[j];
            }
            double den = (flags & ORACLE_F_NORM_R) ? fmax(fabs(sigma), 1.0) : 1.0;
            double *on = (double *)row_v(o, &d, b, n, hh);
            for (int64_t j = 0; j < d.d_v; ++j) on[j] = acc[j] / den;
        }
        free(qr);
        free(kr);
        free(acc);
    }
    return 0;
}

/*
 * Recurrent form, [RN] §2.2:  S_n = gamma S_{n-1} + K_n^T V_n,  o_n = Q_n S_n.
 * The key-sum state z_n = gamma z_{n-1} + K_n carries the row sum sum_m score_nm
 * = (s/c_n) q_n . z_n that the R~ normalisation of [RN] §三.3 divides by.
 * state_in / z_in (may be NULL = zeros) hold S and z before the first token;
 * state_out / z_out (may be NULL) receive them after the last token.
 */
int oracle_recurrent(const double *q, const double *k, const double *v, double *o, oracle_dims_t d,
                     const double *gamma, const double *theta, int64_t pos0, unsigned flags,
                     const double *state_in, double *state_out, const double *z_in, double *z_out,
                     int nthreads) {
    set_threads(nthreads);
    const int xpos = (flags & ORACLE_F_XPOS) != 0;
    int64_t pairs = d.batch * d.heads;
    int64_t ssz = d.d_k * d.d_v;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < pairs; ++bh) {
        int64_t hh = bh % d.heads, b = bh / d.heads;
        double g = gamma[hh];
        double *S = (double *)malloc(sizeof(double) * (size_t)ssz);
        double *z = (double *)malloc(sizeof(double) * (size_t)d.d_k);
        double *qn = (double *)malloc(sizeof(double) * (size_t)d.d_k);
        double *kn = (double *)malloc(sizeof(double) * (size_t)d.d_k);
        if (state_in) memcpy(S, state_in + bh * ssz, sizeof(double) * (size_t)ssz);
        else memset(S, 0, sizeof(double) * (size_t)ssz);
        if (z_in) memcpy(z, z_in + bh * d.d_k, sizeof(double) * (size_t)d.d_k);
        else memset(z, 0, sizeof(double) * (size_t)d.d_k);
        /* D~ row sum a_p = sum_{j=0..p} gamma^j, carried as a_p = gamma a_{p-1} + 1 (the
         * recurrent view of the same sum), started from a_{-1} = 0 at absolute position 0. */
        double a = 0.0;
        for (int64_t p = 0; p < pos0; ++p) a = g * a + 1.0;
        for (int64_t n = 0; n < d.seqlen; ++n) {
            int64_t p = pos0 + n;
            xpos_rotate(row_qk(q, &d, b, n, hh), qn, d.d_k, theta, p, xpos);
            xpos_rotate(row_qk(k, &d, b, n, hh), kn, d.d_k, theta, p, xpos);
            const double *vn = row_v(v, &d, b, n, hh);
            for (int64_t i = 0; i < d.d_k; ++i) {
                for (int64_t j = 0; j < d.d_v; ++j) S[i * d.d_v + j] = g * S[i * d.d_v + j] + kn[i] * vn[j];
                z[i] = g * z[i] + kn[i];
            }
            a = g * a + 1.0;
            double f = 1.0;
            if (flags & ORACLE_F_SCALE_SQRT_D) f /= sqrt((double)d.d_k);
            if (flags & ORACLE_F_NORM_D) f /= sqrt(a);
            double den = 1.0;
            if (flags & ORACLE_F_NORM_R) den = fmax(fabs(f * dot(qn, z, d.d_k)), 1.0);
            double *on = (double *)row_v(o, &d, b, n, hh);
            for (int64_t j = 0; j < d.d_v; ++j) {
                double acc = 0.0;
                for (int64_t i = 0; i < d.d_k; ++i) acc += qn[i] * S[i * d.d_v + j];
                on[j] = acc * f / den;
            }
        }
        if (state_out) memcpy(state_out + bh * ssz, S, sizeof(double) * (size_t)ssz);
        if (z_out) memcpy(z_out + bh * d.d_k, z, sizeof(double) * (size_t)d.d_k);
        free(S);
        free(z);
        free(qn);
        free(kn);
    }
    return 0;
}

/*
 * Chunkwise recurrent form, [RN] §2.4, taken step by step for chunks of length B:
 *   R_i = K_[i]^T (V_[i] (.) zeta) + gamma^B R_{i-1},           zeta_r = gamma^(B-1-r)
 *   O_[i] = (Q_[i] K_[i]^T (.) D) V_[i] + (Q_[i] R_{i-1}) (.) xi,  xi_r = gamma^(r+1)
 * with D the chunk-local decay mask of [RN] §2.3 and r the 0-based row in the chunk.
 * A ragged tail chunk of length b' < B uses b' in zeta and in the decay gamma^b'.
 * The normalisations enter as the same per-row scalars as in the parallel form; the
 * R~ row sum is split the same way, with the key-sum state z_i in place of R_i.
 */
int oracle_chunkwise(const double *q, const double *k, const double *v, double *o, oracle_dims_t d,
                     const double *gamma, const double *theta, int64_t pos0, unsigned flags, int64_t chunk,
                     const double *state_in, double *state_out, const double *z_in, double *z_out,
                     int nthreads) {
    if (chunk <= 0) return 1;
    set_threads(nthreads);
    const int xpos = (flags & ORACLE_F_XPOS) != 0;
    int64_t pairs = d.batch * d.heads;
    int64_t ssz = d.d_k * d.d_v;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < pairs; ++bh) {
        int64_t hh = bh % d.heads, b = bh / d.heads;
        double g = gamma[hh];
        double *R = (double *)malloc(sizeof(double) * (size_t)ssz);
        double *Rn = (double *)malloc(sizeof(double) * (size_t)ssz);
        double *z = (double *)malloc(sizeof(double) * (size_t)d.d_k);
        double *zn = (double *)malloc(sizeof(double) * (size_t)d.d_k);
        double *qc = (double *)malloc(sizeof(double) * (size_t)(chunk * d.d_k));
        double *kc = (double *)malloc(sizeof(double) * (size_t)(chunk * d.d_k));
        double *acc = (double *)malloc(sizeof(double) * (size_t)d.d_v);
        if (state_in) memcpy(R, state_in + bh * ssz, sizeof(double) * (size_t)ssz);
        else memset(R, 0, sizeof(double) * (size_t)ssz);
        if (z_in) memcpy(z, z_in + bh * d.d_k, sizeof(double) * (size_t)d.d_k);
        else memset(z, 0, sizeof(double) * (size_t)d.d_k);
        for (int64_t t0 = 0; t0 < d.seqlen; t0 += chunk) {
            int64_t bl = d.seqlen - t0 < chunk ? d.seqlen - t0 : chunk; /* b' */
            for (int64_t r = 0; r < bl; ++r) {
                xpos_rotate(row_qk(q, &d, b, t0 + r, hh), qc + r * d.d_k, d.d_k, theta, pos0 + t0 + r, xpos);
                xpos_rotate(row_qk(k, &d, b, t0 + r, hh), kc + r * d.d_k, d.d_k, theta, pos0 + t0 + r, xpos);
            }
            /* O_[i]: inner-chunk plus cross-chunk terms, both from R_{i-1}. */
            for (int64_t r = 0; r < bl; ++r) {
                double f = row_factor(g, d.d_k, pos0 + t0 + r, flags);
                double xi = pow(g, (double)(r + 1));
                double sigma = 0.0;
                for (int64_t j = 0; j < d.d_v; ++j) acc[j] = 0.0;
                for (int64_t c = 0; c <= r; ++c) { /* (Q K^T (.) D) V inside the chunk */
                    double sc = dot(qc + r * d.d_k, kc + c * d.d_k, d.d_k) * pow(g, (double)(r - c));
                    sigma += sc;
                    const double *vc = row_v(v, &d, b, t0 + c, hh);
                    for (int64_t j = 0; j < d.d_v; ++j) acc[j] += sc * vc[j];
                }
                for (int64_t j = 0; j < d.d_v; ++j) { /* (Q R_{i-1}) (.) xi */
                    double cr = 0.0;
                    for (int64_t i = 0; i < d.d_k; ++i) cr += qc[r * d.d_k + i] * R[i * d.d_v + j];
                    acc[j] += xi * cr;
                }
                sigma += xi * dot(qc + r * d.d_k, z, d.d_k);
                double den = (flags & ORACLE_F_NORM_R) ? fmax(fabs(f * sigma), 1.0) : 1.0;
                double *orow = (double *)row_v(o, &d, b, t0 + r, hh);
                for (int64_t j = 0; j < d.d_v; ++j) orow[j] = acc[j] * f / den;
            }
            /* R_i = K_[i]^T (V_[i] (.) zeta) + gamma^b' R_{i-1}; z_i alike with V = 1. */
            double gb = pow(g, (double)bl);
            for (int64_t i = 0; i < d.d_k; ++i) {
                for (int64_t j = 0; j < d.d_v; ++j) Rn[i * d.d_v + j] = gb * R[i * d.d_v + j];
                zn[i] = gb * z[i];
            }
            for (int64_t r = 0; r < bl; ++r) {
                double zeta = pow(g, (double)(bl - 1 - r));
                const double *vr = row_v(v, &d, b, t0 + r, hh);
                for (int64_t i = 0; i < d.d_k; ++i) {
                    double kz = kc[r * d.d_k + i] * zeta;
                    for (int64_t j = 0; j < d.d_v; ++j) Rn[i * d.d_v + j] += kz * vr[j];
                    zn[i] += kz;
                }
            }
            memcpy(R, Rn, sizeof(double) * (size_t)ssz);
            memcpy(z, zn, sizeof(double) * (size_t)d.d_k);
        }
        if (state_out) memcpy(state_out + bh * ssz, R, sizeof(double) * (size_t)ssz);
        if (z_out) memcpy(z_out + bh * d.d_k, z, sizeof(double) * (size_t)d.d_k);
        free(R);
        free(Rn);
        free(z);
        free(zn);
        free(qc);
        free(kc);
        free(acc);
    }
    return 0;
}

/*
 * MSR epilogue, [RN] §三.2:  Y = GroupNorm_h(Concat(head_1..head_h)),  out = swish(G) (.) Y.
 * Groups are the heads: for each (token, head) row of d_v values, the biased mean and
 * variance are taken over the row, y = (x - mean) / sqrt(var + eps), unit affine.
 * swish(g) = g * sigmoid(g) = g / (1 + exp(-g)).  The W_O projection is not part of it.
 * y, g, out: [tokens][heads][d_v].
 */
int oracle_msr_epilogue(const double *y, const double *g, double *out, int64_t tokens, int64_t heads,
                        int64_t d_v, double eps, int nthreads) {
    set_threads(nthreads);
    int64_t rows = tokens * heads;
#pragma omp parallel for schedule(static)
    for (int64_t rr = 0; rr < rows; ++rr) {
        const double *x = y + rr * d_v;
        const double *gr = g + rr * d_v;
        double *orow = out + rr * d_v;
        double mean = 0.0;
        for (int64_t j = 0; j < d_v; ++j) mean += x[j];
        mean /= (double)d_v;
        double var = 0.0;
        for (int64_t j = 0; j < d_v; ++j) var += (x[j] - mean) * (x[j] - mean);
        var /= (double)d_v;
        double inv = 1.0 / sqrt(var + eps);
        for (int64_t j = 0; j < d_v; ++j) {
            double sw = gr[j] / (1.0 + exp(-gr[j]));
            orow[j] = sw * ((x[j] - mean) * inv);
        }
    }
    return 0;
}

/*
 * Gradient of the retention forward, for training ([RN] §2.4 notes that training uses the
 * chunkwise form; its outputs are those of the parallel form, so the gradient is that of the
 * definition).  With q~_n, k~_n the rotated rows (xPos), f_n the row factor of §三.3 (no R~)
 * and an optional state S0 before the first token (the chunkwise / recurrent state_in):
 *     O_n = f_n [ sum_{m<=n} gamma^(n-m) (q~_n . k~_m) v_m  +  gamma^(n+1) q~_n S0 ].
 * Given dO (the gradient of a loss with respect to O), by the product rule:
 *     dq~_n = f_n [ sum_{m<=n} gamma^(n-m) (dO_n . v_m) k~_m  +  gamma^(n+1) S0 dO_n ]
 *     dk~_m = sum_{n>=m} f_n gamma^(n-m) (dO_n . v_m) q~_n
 *     dv_m  = sum_{n>=m} f_n gamma^(n-m) (q~_n . k~_m) dO_n
 *     dS0   = sum_n f_n gamma^(n+1) q~_n^T dO_n
 * and dq_n = R(p theta)^T dq~_n, dk_m = R(p theta)^T dk~_m (the rotation is orthogonal).
 * R~ (a division by a function of q and k) is not covered: flags with it return -1.
 * state_in and dstate (both [batch][heads][d_k][d_v]) may be NULL.
 */
static void xpos_rotate_back(const double *y, double *x, int64_t d, const double *theta, int64_t p, int on) {
    if (!on) {
        memcpy(x, y, sizeof(double) * (size_t)d);
        return;
    }
    for (int64_t j = 0; j < d / 2; ++j) {
        double a = (double)p * theta[j];
        double c = cos(a), s = sin(a);
        double y0 = y[2 * j], y1 = y[2 * j + 1];
        x[2 * j] = y0 * c + y1 * s;
        x[2 * j + 1] = -y0 * s + y1 * c;
    }
}

int oracle_backward(const double *q, const double *k, const double *v, const double *dout, double *dq, double *dk,
                    double *dv, oracle_dims_t d, const double *gamma, const double *theta, int64_t pos0,
                    unsigned flags, const double *state_in, double *dstate, int nthreads) {
    if (flags & ORACLE_F_NORM_R) return -1;
    set_threads(nthreads);
    const int xpos = (flags & ORACLE_F_XPOS) != 0;
    const int64_t pairs = d.batch * d.heads, L = d.seqlen, dk_ = d.d_k, dv_ = d.d_v;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < pairs; ++bh) {
        int64_t b = bh / d.heads, hh = bh % d.heads;
        double g = gamma[hh];
        double *qr = (double *)malloc(sizeof(double) * (size_t)(L * dk_));
        double *kr = (double *)malloc(sizeof(double) * (size_t)(L * dk_));
        double *f = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        double *tq = (double *)malloc(sizeof(double) * (size_t)dk_);
        double *tk = (double *)malloc(sizeof(double) * (size_t)dk_);
        const double *S0 = state_in ? state_in + bh * dk_ * dv_ : NULL;
        for (int64_t t = 0; t < L; ++t) {
            xpos_rotate(row_qk(q, &d, b, t, hh), qr + t * dk_, dk_, theta, pos0 + t, xpos);
            xpos_rotate(row_qk(k, &d, b, t, hh), kr + t * dk_, dk_, theta, pos0 + t, xpos);
            f[t] = row_factor(g, dk_, pos0 + t, flags);
        }
        for (int64_t n = 0; n < L; ++n) { /* dq */
            const double *don = row_v(dout, &d, b, n, hh);
            memset(tq, 0, sizeof(double) * (size_t)dk_);
            for (int64_t m = 0; m <= n; ++m) {
                double w = pow(g, (double)(n - m)) * dot(don, row_v(v, &d, b, m, hh), dv_);
                for (int64_t i = 0; i < dk_; ++i) tq[i] += w * kr[m * dk_ + i];
            }
            if (S0) {
                double gn = pow(g, (double)(n + 1));
                for (int64_t i = 0; i < dk_; ++i) tq[i] += gn * dot(S0 + i * dv_, don, dv_);
            }
            for (int64_t i = 0; i < dk_; ++i) tq[i] *= f[n];
            xpos_rotate_back(tq, (double *)row_qk(dq, &d, b, n, hh), dk_, theta, pos0 + n, xpos);
        }
        for (int64_t m = 0; m < L; ++m) { /* dk, dv */
            const double *vm = row_v(v, &d, b, m, hh);
            double *dvm = (double *)row_v(dv, &d, b, m, hh);
            memset(tk, 0, sizeof(double) * (size_t)dk_);
            memset(dvm, 0, sizeof(double) * (size_t)dv_);
            for (int64_t n = m; n < L; ++n) {
                const double *don = row_v(dout, &d, b, n, hh);
                double a = f[n] * pow(g, (double)(n - m));
                double wk = a * dot(don, vm, dv_);
                double wv = a * dot(qr + n * dk_, kr + m * dk_, dk_);
                for (int64_t i = 0; i < dk_; ++i) tk[i] += wk * qr[n * dk_ + i];
                for (int64_t j = 0; j < dv_; ++j) dvm[j] += wv * don[j];
            }
            xpos_rotate_back(tk, (double *)row_qk(dk, &d, b, m, hh), dk_, theta, pos0 + m, xpos);
        }
        if (dstate) { /* dS0 */
            double *dS = dstate + bh * dk_ * dv_;
            memset(dS, 0, sizeof(double) * (size_t)(dk_ * dv_));
            for (int64_t n = 0; n < L; ++n) {
                const double *don = row_v(dout, &d, b, n, hh);
                double a = f[n] * pow(g, (double)(n + 1));
                for (int64_t i = 0; i < dk_; ++i)
                    for (int64_t j = 0; j < dv_; ++j) dS[i * dv_ + j] += a * qr[n * dk_ + i] * don[j];
            }
        }
        free(qr);
        free(kr);
        free(f);
        free(tq);
        free(tk);
    }
    return 0;
}
