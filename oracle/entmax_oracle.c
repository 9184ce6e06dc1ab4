/*
 * entmax_oracle.c -- plain, slow fp64 CPU oracle for fused alpha-entmax attention.
 *
 * TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline leg may build, load or call this file. The CUDA library and its Python
 * binding never touch it, and the two share no code.
 *
 * What it computes, and where each step comes from:
 *   - "AdaSplash-2: Faster Differentiable Sparse Attention", §2.2: scores
 *     S = Q K^T / sqrt(d) (here S = scale * Q K^T, scale given), O = pi(S) V.
 *   - same page, §2.3 Eq. 3: alpha-entmax(s) = [(alpha-1) s - tau 1]_+^{1/(alpha-1)}.
 *   - same page, §2.4 Eq. 4: f(tau) = -1 + sum_j [(alpha-1) s_j - tau]_+^{1/(alpha-1)},
 *     tau* is the root of f; bracket m-1 <= tau* <= m - n^{1-alpha}, m = (alpha-1) max s.
 *   - same page, §2.4 "Sorting-based solvers" (and §5): for alpha in {1.5, 2} the
 *     support is the top-k entries of the sorted scores, so tau has a closed form per k.
 *   - same page, §3.3 "Backward pass": gradients are nonzero only on the support.
 *     The Jacobian itself is not printed; it is derived from Eq. 3 by implicit
 *     differentiation of sum_j p_j = 1 (see orc_attn_rows / orc_attn_cols).
 *   - same page, Appendix C.4: bit-packed block mask, 32 column blocks per uint32.
 *   - "Hooshaai/gpt2-adasplash-attention" model card, "Causal Splash Masking with
 *     Sink Preservation": active set {0} U {j <= i : i - j <= W}.
 *   - "AdaSplash-2", §3.1 and Appendix C.3: the histogram initialisation of tau
 *     (orc_tau_hist), with Proposition 3.1's bound tau* - 1/B < tau_h <= tau*.
 *   - "AdaSplash-2", §4.3: NAPE gives half of the heads no positional encoding and half
 *     ALiBi (Press et al.), a per-head linear penalty on the scores by query-key distance:
 *     s_ij = scale q_i . k_j - m_h |i - j| (m_h = 0 for a head without it).
 *
 * Everything is fp64 with no intermediate rounding; inputs are widened exactly
 * from whatever the caller drew (bf16 or fp32). Rows are parallelised with
 * OpenMP; nothing is blocked, fused or reordered beyond that.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_METHOD_SORT 0
#define ORC_METHOD_BISECT 1
#define ORC_METHOD_AUTO 2   /* sort for alpha in {1.5, 2}, bisection otherwise */

int orc_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Active key set of query row i (model card "Causal Splash Masking"; key padding
 * keeps keys j < kv_len). window >= 0 implies causal. */
static int is_active(long i, long j, int causal, int window, int kv_len) {
    if (j >= kv_len) return 0;
    if (window >= 0) return j <= i && (j == 0 || i - j <= window);
    if (causal) return j <= i;
    return 1;
}

static int cmp_desc(const void *a, const void *b) {
    double x = *(const double *)a, y = *(const double *)b;
    return (x < y) - (x > y);
}

/* Eq. 4 evaluated directly: f(tau) = -1 + sum_j [z_j - tau]_+^{1/(alpha-1)}. */
double orc_f(const double *z, int n, double alpha, double tau) {
    double e = 1.0 / (alpha - 1.0), acc = -1.0;
    for (int j = 0; j < n; ++j) {
        double u = z[j] - tau;
        if (u > 0) acc += pow(u, e);
    }
    return acc;
}

/* Sort-based exact threshold for alpha in {1.5, 2} (AdaSplash-2 §2.4, "Sorting-based
 * solvers"). zs holds z = (alpha-1) s for the n active entries; it is sorted in place,
 * descending. For a support made of the top k entries, sum_{i<=k} (z_(i) - tau)^{1/(alpha-1)} = 1
 * has a closed form:
 *   alpha = 2  : tau_k = (S1 - 1) / k                        (linear)
 *   alpha = 1.5: k tau^2 - 2 S1 tau + (S2 - 1) = 0, smaller root
 *                tau_k = (S1 - sqrt(S1^2 - k (S2 - 1))) / k
 * with S1, S2 the sums of the top-k z and z^2. The support size is the largest k whose
 * tau_k lies below z_(k); that tau_k is tau*. Returns NAN for any other alpha. */
double orc_tau_sort(double *zs, int n, double alpha) {
    if (n <= 0) return NAN;
    qsort(zs, (size_t)n, sizeof(double), cmp_desc);
    double S1 = 0, S2 = 0, best = NAN;
    for (int k = 1; k <= n; ++k) {
        double zk = zs[k - 1];
        S1 += zk;
        S2 += zk * zk;
        double t;
        if (alpha == 2.0) {
            t = (S1 - 1.0) / k;
        } else if (alpha == 1.5) {
            double disc = S1 * S1 - (double)k * (S2 - 1.0);
            if (disc < 0) continue; /* this top-k piece never reaches 1 */
            t = (S1 - sqrt(disc)) / k;
        } else {
            return NAN;
        }
        if (t < zk) best = t;
    }
    return best;
}

/* Plain bisection on Eq. 4 over the §2.4 bracket [m - 1, m - n^{1-alpha}]; any alpha > 1. */
double orc_tau_bisect(const double *z, int n, double alpha, int iters) {
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) m = z[j] > m ? z[j] : m;
    double lo = m - 1.0, hi = m - pow((double)n, 1.0 - alpha);
    for (int it = 0; it < iters; ++it) {
        double mid = 0.5 * (lo + hi);
        if (orc_f(z, n, alpha, mid) > 0) lo = mid; else hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* Histogram initialisation of tau ("AdaSplash-2", §3.1 and Appendix C.3), for any alpha > 1.
 * z = (alpha-1) s for the n active entries (Eq. 3 units). The scores are shifted so that
 * the largest is 1 (z~ = z - (m - 1), m = max z), and each z~ in [0, 1] goes to bin
 * b = min(floor(B z~), B - 1), whose left edge k/B stands in for it: the histogram
 * objective is f_h(t) = -1 + sum_k H_k [k/B - t]_+^{1/(alpha-1)}. Entries with z~ < 0 are
 * left out: their edges lie at or below -1/B, and the root tau_h of f_h lies above -1/B
 * (Proposition 3.1: tau* - 1/B < tau_h <= tau*, with tau* >= 0 in shifted units).
 * tau_h is found on the bins: for alpha in {1.5, 2} the exact solve of §2.4 with each bin
 * counted H_k times (the support is a run of top bins), otherwise bisection of f_h over
 * [-1/B, 1] (200 halvings). Returns tau_h in Eq. 3 units, or NAN if B < 1 or n < 1. */
double orc_tau_hist(const double *z, int n, double alpha, int B) {
    if (n < 1 || B < 1) return NAN;
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) m = z[j] > m ? z[j] : m;
    double *H = (double *)calloc((size_t)B, sizeof(double));
    for (int j = 0; j < n; ++j) {
        const double zt = z[j] - (m - 1.0);
        if (zt < 0) continue;
        int b = (int)floor(B * zt);
        if (b > B - 1) b = B - 1;
        H[b] += 1.0;
    }
    double t = NAN;
    if (alpha == 2.0 || alpha == 1.5) {
        double S0 = 0, S1 = 0, S2 = 0;
        for (int k = B - 1; k >= 0; --k) {   /* top bins first */
            if (H[k] == 0) continue;
            const double e = (double)k / B;
            S0 += H[k];
            S1 += H[k] * e;
            S2 += H[k] * e * e;
            double tk;
            if (alpha == 2.0) {
                tk = (S1 - 1.0) / S0;
            } else {
                const double disc = S1 * S1 - S0 * (S2 - 1.0);
                if (disc < 0) continue;
                tk = (S1 - sqrt(disc)) / S0;
            }
            if (tk < e) t = tk;   /* every bin of this run lies above tk */
        }
    } else {
        const double ex = 1.0 / (alpha - 1.0);
        double lo = -1.0 / B, hi = 1.0;
        for (int it = 0; it < 200; ++it) {
            const double mid = 0.5 * (lo + hi);
            double f = -1.0;
            for (int k = 0; k < B; ++k) {
                const double u = (double)k / B - mid;
                if (u > 0 && H[k] > 0) f += H[k] * pow(u, ex);
            }
            if (f > 0) lo = mid; else hi = mid;
        }
        t = 0.5 * (lo + hi);
    }
    free(H);
    return t + (m - 1.0);
}

/* One row of alpha-entmax on raw scores s (entries equal to -inf are inactive).
 * Writes p (Eq. 3) and returns tau (Eq. 3 units). work holds n doubles. For alpha outside
 * {1.5, 2} the sorting solver has no closed form per support, and ORC_METHOD_AUTO takes
 * the bisection of Eq. 4 over the §2.4 bracket (200 halvings of a bracket of width < 1:
 * down to fp64 resolution). */
double orc_entmax_row(const double *s, int n, double alpha, int method, double *p, double *work) {
    int na = 0;
    for (int j = 0; j < n; ++j)
        if (s[j] != -INFINITY) work[na++] = (alpha - 1.0) * s[j];
    if (method == ORC_METHOD_AUTO) method = (alpha == 1.5 || alpha == 2.0) ? ORC_METHOD_SORT : ORC_METHOD_BISECT;
    double tau = (method == ORC_METHOD_SORT) ? orc_tau_sort(work, na, alpha)
                                             : orc_tau_bisect(work, na, alpha, 200);
    double e = 1.0 / (alpha - 1.0);
    for (int j = 0; j < n; ++j) {
        double u = (s[j] == -INFINITY) ? -1.0 : (alpha - 1.0) * s[j] - tau;
        p[j] = u > 0 ? pow(u, e) : 0.0;
    }
    return tau;
}

/* entmax over explicit score rows: S[r*ld + j], j < n. */
void orc_entmax_rows(const double *S, long rows, int n, long ld, double alpha, int method,
                     double *P, double *tau) {
#pragma omp parallel
    {
        double *work = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
#pragma omp for schedule(dynamic, 4)
        for (long r = 0; r < rows; ++r)
            tau[r] = orc_entmax_row(S + r * ld, n, alpha, method, P + r * ld, work);
        free(work);
    }
}

static double dotd(const double *a, const double *b, int d) {
    double acc = 0;
    for (int k = 0; k < d; ++k) acc += a[k] * b[k];
    return acc;
}

/* ---------------------------------------------------------------------------------
 * Attention. Tensors are contiguous [B, H, L, d] fp64; kv_len is int[B] (or NULL = L).
 * z_ij = (alpha-1) * scale * q_i . k_j for active j.
 * Per row:
 *   p_ij  = [z_ij - tau_i]_+^{1/(alpha-1)}                (Eq. 3)
 *   g_ij  = [z_ij - tau_i]_+^{(2-alpha)/(alpha-1)} = p_ij^{2-alpha} on the support, 0 off it
 *   O_i   = sum_j p_ij V_j
 *   Backward (derived from Eq. 3: dp_j/ds_k = g_j delta_jk - g_j g_k / sum g):
 *   dA_ij = dO_i . V_j,  delta_i = sum_j g_ij dA_ij / sum_j g_ij,
 *   dS_ij = g_ij (dA_ij - delta_i)      (gradient w.r.t. s_ij = scale q_i . k_j)
 *   dQ_i  = scale sum_j dS_ij K_j,  dK_j = scale sum_i dS_ij Q_i,  dV_j = sum_i p_ij dO_i
 * --------------------------------------------------------------------------------- */
typedef struct {
    int B, H, L, d;
    double alpha, scale;
    int causal, window;
    const int *kv_len;
    const double *alibi;   /* per-head slopes m_h [H], or NULL */
} orc_shape;

/* The score of an active pair: scale q_i . k_j, minus the ALiBi penalty m_h |i - j|. */
static double score(const orc_shape *sh, int h, long i, long j, const double *q, const double *k) {
    double s = sh->scale * dotd(q, k, sh->d);
    if (sh->alibi) s -= sh->alibi[h] * (double)(i > j ? i - j : j - i);
    return s;
}

static int kvl(const orc_shape *sh, int b) { return sh->kv_len ? sh->kv_len[b] : sh->L; }

/* Row pass for one (b, h, i): tau_i and everything that depends only on row i.
 * Any output pointer may be NULL. srow/p/g/work are scratch of L doubles. */
static void attn_row(const orc_shape *sh, int b, int h, int i, const double *Q, const double *K,
                     const double *V, const double *dO, double *O_i, double *tau_i, double *sumg_i,
                     double *Ot_i, double *delta_i, double *dQ_i, double *srow, double *p,
                     double *g, double *work) {
    const int L = sh->L, d = sh->d, kv = kvl(sh, b);
    const double alpha = sh->alpha;
    const size_t head = ((size_t)b * sh->H + h) * (size_t)L * d;
    const double *q = Q + head + (size_t)i * d;
    for (int j = 0; j < L; ++j)
        srow[j] = is_active(i, j, sh->causal, sh->window, kv) ? score(sh, h, i, j, q, K + head + (size_t)j * d)
                                                               : -INFINITY;
    double tau = orc_entmax_row(srow, L, alpha, ORC_METHOD_AUTO, p, work);
    double sg = 0, ge = (2.0 - alpha) / (alpha - 1.0);
    for (int j = 0; j < L; ++j) {
        double u = (srow[j] == -INFINITY) ? -1.0 : (alpha - 1.0) * srow[j] - tau;
        g[j] = u > 0 ? pow(u, ge) : 0.0;
        sg += g[j];
    }
    if (tau_i) *tau_i = tau;
    if (sumg_i) *sumg_i = sg;
    if (O_i) {
        for (int k = 0; k < d; ++k) O_i[k] = 0;
        for (int j = 0; j < L; ++j)
            if (p[j] != 0)
                for (int k = 0; k < d; ++k) O_i[k] += p[j] * V[head + (size_t)j * d + k];
    }
    if (Ot_i) {
        for (int k = 0; k < d; ++k) Ot_i[k] = 0;
        for (int j = 0; j < L; ++j)
            if (g[j] != 0)
                for (int k = 0; k < d; ++k) Ot_i[k] += g[j] * V[head + (size_t)j * d + k];
    }
    if (dO && (delta_i || dQ_i)) {
        const double *dOi = dO + head + (size_t)i * d;
        double num = 0;
        for (int j = 0; j < L; ++j)
            if (g[j] != 0) num += g[j] * dotd(dOi, V + head + (size_t)j * d, d);
        double dl = num / sg;
        if (delta_i) *delta_i = dl;
        if (dQ_i) {
            for (int k = 0; k < d; ++k) dQ_i[k] = 0;
            for (int j = 0; j < L; ++j) {
                if (g[j] == 0) continue;
                double dS = g[j] * (dotd(dOi, V + head + (size_t)j * d, d) - dl);
                for (int k = 0; k < d; ++k) dQ_i[k] += sh->scale * dS * K[head + (size_t)j * d + k];
            }
        }
    }
}

static orc_shape mkshape(int B, int H, int L, int d, double alpha, double scale, int causal,
                         int window, const int *kv_len, const double *alibi) {
    orc_shape sh = {B, H, L, d, alpha, scale, causal, window, kv_len, alibi};
    return sh;
}

/* Forward (and, when dO != NULL, the row-local part of the backward) for a list of rows.
 * rows[r] = (b*H + h)*L + i. Outputs are indexed by r: O[r*d], tau[r], sumg[r], Ot[r*d],
 * delta[r], dQ[r*d]; any may be NULL. */
int orc_attn_rows(int B, int H, int L, int d, double alpha, double scale, int causal, int window,
                  const int *kv_len, const double *alibi, const double *Q, const double *K, const double *V,
                  const double *dO, const long *rows, long nrows, double *O, double *tau,
                  double *sumg, double *Ot, double *delta, double *dQ) {
    orc_shape sh = mkshape(B, H, L, d, alpha, scale, causal, window, kv_len, alibi);
    if (!(alpha > 1.0)) return 1;
#pragma omp parallel
    {
        double *buf = (double *)malloc(sizeof(double) * 4 * (size_t)L);
#pragma omp for schedule(dynamic, 8)
        for (long r = 0; r < nrows; ++r) {
            long flat = rows[r];
            int i = (int)(flat % L);
            long bh = flat / L;
            int h = (int)(bh % H), b = (int)(bh / H);
            attn_row(&sh, b, h, i, Q, K, V, dO, O ? O + r * d : NULL, tau ? tau + r : NULL,
                     sumg ? sumg + r : NULL, Ot ? Ot + r * d : NULL, delta ? delta + r : NULL,
                     dQ ? dQ + r * d : NULL, buf, buf + L, buf + 2 * L, buf + 3 * L);
        }
        free(buf);
    }
    return 0;
}

/* Column pass of the backward for a list of key positions cols[c] = (b*H + h)*L + j.
 * Needs tau and delta of every row of the head (indexed [(b*H+h)*L + i]).
 * Writes dK[c*d], dV[c*d]. */
int orc_attn_cols(int B, int H, int L, int d, double alpha, double scale, int causal, int window,
                  const int *kv_len, const double *alibi, const double *Q, const double *K, const double *V,
                  const double *dO, const double *tau, const double *delta, const long *cols,
                  long ncols, double *dK, double *dV) {
    orc_shape sh = mkshape(B, H, L, d, alpha, scale, causal, window, kv_len, alibi);
    if (!(alpha > 1.0)) return 1;
    const double e = 1.0 / (alpha - 1.0), ge = (2.0 - alpha) / (alpha - 1.0);
#pragma omp parallel for schedule(dynamic, 8)
    for (long c = 0; c < ncols; ++c) {
        long flat = cols[c];
        int j = (int)(flat % L);
        long bh = flat / L;
        int b = (int)(bh / H), h = (int)(bh % H);
        const size_t head = (size_t)bh * (size_t)L * d;
        const int kv = kvl(&sh, b);
        double *dKj = dK + c * d, *dVj = dV + c * d;
        for (int k = 0; k < d; ++k) dKj[k] = dVj[k] = 0;
        const double *kj = K + head + (size_t)j * d, *vj = V + head + (size_t)j * d;
        for (int i = 0; i < L; ++i) {
            if (!is_active(i, j, sh.causal, sh.window, kv)) continue;
            const double *qi = Q + head + (size_t)i * d;
            double u = (alpha - 1.0) * score(&sh, h, i, j, qi, kj) - tau[bh * L + i];
            if (!(u > 0)) continue;
            double p = pow(u, e), g = pow(u, ge);
            const double *dOi = dO + head + (size_t)i * d;
            double dS = g * (dotd(dOi, vj, d) - delta[bh * L + i]);
            for (int k = 0; k < d; ++k) {
                dVj[k] += p * dOi[k];
                dKj[k] += scale * dS * qi[k];
            }
        }
    }
    return 0;
}

/* Block mask (AdaSplash-2 §3.3 Phase 3, Appendix C.4) at tile size Br x Bc, from fp64
 * z and the given tau: bit (it, jt) is set iff some row of query tile it has some
 * z_ij > tau_i with j in key tile jt. Packed 32 key tiles per uint32:
 * M[((b*H+h)*Tr + it)*Wc + jt/32] bit jt%32, Wc = ceil(Tc/32).
 * M_lo / M_hi: the same with tau_i + margin / tau_i - margin, so that tiles whose only
 * deciding entries lie within `margin` of tau can be told apart (M_lo != M_hi).
 * tau is indexed [(b*H+h)*L + i]. Any of M, M_lo, M_hi may be NULL. */
int orc_block_mask(int B, int H, int L, int d, double alpha, double scale, int causal, int window,
                   const int *kv_len, const double *alibi, const double *Q, const double *K,
                   const double *tau, int Br, int Bc, double margin, uint32_t *M, uint32_t *M_lo,
                   uint32_t *M_hi) {
    orc_shape sh = mkshape(B, H, L, d, alpha, scale, causal, window, kv_len, alibi);
    const int Tr = (L + Br - 1) / Br, Tc = (L + Bc - 1) / Bc, Wc = (Tc + 31) / 32;
    const size_t words = (size_t)B * H * Tr * Wc;
    if (M) memset(M, 0, words * sizeof(uint32_t));
    if (M_lo) memset(M_lo, 0, words * sizeof(uint32_t));
    if (M_hi) memset(M_hi, 0, words * sizeof(uint32_t));
#pragma omp parallel for schedule(dynamic, 1)
    for (long bht = 0; bht < (long)B * H * Tr; ++bht) {
        int it = (int)(bht % Tr);
        long bh = bht / Tr;
        int b = (int)(bh / H), h = (int)(bh % H);
        const size_t head = (size_t)bh * (size_t)L * d;
        const int kv = kvl(&sh, b);
        uint32_t *row = M ? M + (size_t)bht * Wc : NULL;
        uint32_t *rlo = M_lo ? M_lo + (size_t)bht * Wc : NULL;
        uint32_t *rhi = M_hi ? M_hi + (size_t)bht * Wc : NULL;
        for (int i = it * Br; i < L && i < (it + 1) * Br; ++i) {
            const double t = tau[bh * L + i];
            for (int j = 0; j < L; ++j) {
                if (!is_active(i, j, sh.causal, sh.window, kv)) continue;
                double z = (alpha - 1.0) * score(&sh, h, i, j, Q + head + (size_t)i * d, K + head + (size_t)j * d);
                uint32_t bit = 1u << ((j / Bc) % 32);
                size_t w = (size_t)(j / Bc) / 32;
                if (row && z > t) row[w] |= bit;
                if (rlo && z > t + margin) rlo[w] |= bit;
                if (rhi && z > t - margin) rhi[w] |= bit;
            }
        }
    }
    return 0;
}
