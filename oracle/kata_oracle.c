/*
 * kata_oracle.c -- plain, slow fp64 CPU oracle for causal kernelized linear
 * attention with the rank-one PSD feature, and for the LoLA self-recall-error
 * (SRE) sparse cache.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library. The CUDA product path never
 * links, loads or calls it, and it shares no code with that path.
 *
 * Every function works on one head at a time, in fp64, in the order the
 * formulas are written, with no blocking or reordering. The *_heads wrappers
 * only loop (OpenMP) over independent heads.
 *
 * Sources, by page title and section:
 *  [KATA]  "Kernelized Linear Attention: Breaking the Capacity Wall with
 *          Symmetric Cones" (technical summary).
 *          s1  problem definition: linear attention gives constant-time
 *              recurrent inference with a fixed-size state.
 *          s2.1 "Output gating": the normalised denominator acts as a
 *              parameter-free convex gate.
 *          s2.2 "PSD cone (rank one)": psi(u) = u u^T, so that
 *              <psi(u_i), psi(u_j)> = <u_i, u_j>^2.
 *          s2.3 chunked parallelism: the chunked state form is exact.
 *  [LoLA]  "LoLA: Low-Rank Linear Attention with Sparse Caching" (technical
 *          summary).
 *          Methodology 1-3: sliding window (full-rank softmax), recurrent
 *              state H_t with normaliser s_t, sparse global cache.
 *          "Self-Recall Error": SRE(k, v | H_t, s_t) =
 *              || phi(k)^T H_t / phi(k)^T s_t - v ||^2.
 *          "Inference strategy" steps 1-4.
 *
 * Readings where the pages leave a step open (each stated where it is used):
 *  R1 packing: phi(x) is the upper triangle of x x^T, row (a) major, entry
 *     (a,b) with a<=b at index a*d - a(a-1)/2 + (b-a); off-diagonal entries
 *     carry a factor sqrt(2) so that <phi(x), phi(y)> = (x.y)^2 holds exactly.
 *  R2 causality is inclusive (j <= i); a recurrent step updates the state
 *     with token i before reading it out with query i.
 *  R3 eps is added to the readout denominator and to the SRE denominator.
 */
#include <math.h>
#include <omp.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_API __attribute__((visibility("default")))

/* Threads the *_heads loops below run on (OpenMP's setting; no arithmetic). */
ORACLE_API int oracle_threads(void) { return omp_get_max_threads(); }
ORACLE_API void oracle_set_threads(int n) { if (n > 0) omp_set_num_threads(n); }

/* ---------------------------------------------------------------- phi ---- */

/* Packed feature dimension D = d(d+1)/2 (R1). */
ORACLE_API long oracle_packed_dim(int d) { return (long)d * (d + 1) / 2; }

/* Index of entry (a, b), a <= b, in the packed upper triangle (R1). */
ORACLE_API long oracle_packed_index(int d, int a, int b)
{
    return (long)a * d - (long)a * (a - 1) / 2 + (b - a);
}

/* [KATA s2.2] phi(x) = x x^T, packed with sqrt(2) on off-diagonal entries. */
ORACLE_API void oracle_phi(const double *x, int d, double *phi)
{
    const double r2 = sqrt(2.0);
    for (int a = 0; a < d; ++a)
        for (int b = a; b < d; ++b) {
            double w = (a == b) ? 1.0 : r2;
            phi[oracle_packed_index(d, a, b)] = w * x[a] * x[b];
        }
}

/* ------------------------------------------------------- quadratic form -- */

/*
 * [KATA s2.2, R2, R3] The plain definition, no feature map and no state:
 *   o_i = sum_{j<=i} (q_i . k_j)^2 v_j / (sum_{j<=i} (q_i . k_j)^2 + eps).
 * One head: q, k [T, d], v [T, dv], o [T, dv]. Rows `rows[0..nrows)` only
 * (rows == NULL means every row, written to o in order).
 */
ORACLE_API void oracle_quadratic(const double *q, const double *k, const double *v,
                                 long T, int d, int dv, double eps,
                                 const long *rows, long nrows, double *o)
{
    long n = rows ? nrows : T;
    double *num = (double *)malloc(sizeof(double) * (size_t)dv);
    for (long r = 0; r < n; ++r) {
        long i = rows ? rows[r] : r;
        double den = 0.0;
        for (int e = 0; e < dv; ++e) num[e] = 0.0;
        for (long j = 0; j <= i; ++j) {
            double dot = 0.0;
            for (int a = 0; a < d; ++a) dot += q[i * d + a] * k[j * d + a];
            double w = dot * dot;
            den += w;
            for (int e = 0; e < dv; ++e) num[e] += w * v[j * dv + e];
        }
        for (int e = 0; e < dv; ++e) o[r * dv + e] = num[e] / (den + eps);
    }
    free(num);
}

/* ------------------------------------------------------- recurrent form -- */

/*
 * [KATA s1, s2.2; LoLA Methodology 2] The literal recurrent-state form:
 *   for i = 0..T-1:  H += phi(k_i) v_i^T;  s += phi(k_i);
 *                    o_i = phi(q_i)^T H / (phi(q_i)^T s + eps)        (R2, R3)
 * One head. Hst [D, dv] and s [D] hold the initial state on entry and the
 * final state on exit. o [T, dv] may be NULL (state only).
 */
ORACLE_API void oracle_recurrent(const double *q, const double *k, const double *v,
                                 long T, int d, int dv, double eps,
                                 double *Hst, double *s, double *o)
{
    long D = oracle_packed_dim(d);
    double *pk = (double *)malloc(sizeof(double) * (size_t)D);
    double *pq = (double *)malloc(sizeof(double) * (size_t)D);
    for (long i = 0; i < T; ++i) {
        oracle_phi(k + i * d, d, pk);
        for (long r = 0; r < D; ++r) {
            for (int e = 0; e < dv; ++e) Hst[r * dv + e] += pk[r] * v[i * dv + e];
            s[r] += pk[r];
        }
        if (!o) continue;
        oracle_phi(q + i * d, d, pq);
        double den = 0.0;
        for (long r = 0; r < D; ++r) den += pq[r] * s[r];
        for (int e = 0; e < dv; ++e) {
            double num = 0.0;
            for (long r = 0; r < D; ++r) num += pq[r] * Hst[r * dv + e];
            o[i * dv + e] = num / (den + eps);
        }
    }
    free(pk);
    free(pq);
}

/* Readout of one query against a given state, no update (R3). */
ORACLE_API void oracle_readout(const double *q, int d, int dv, double eps,
                               const double *Hst, const double *s, double *o)
{
    long D = oracle_packed_dim(d);
    double *pq = (double *)malloc(sizeof(double) * (size_t)D);
    oracle_phi(q, d, pq);
    double den = 0.0;
    for (long r = 0; r < D; ++r) den += pq[r] * s[r];
    for (int e = 0; e < dv; ++e) {
        double num = 0.0;
        for (long r = 0; r < D; ++r) num += pq[r] * Hst[r * dv + e];
        o[e] = num / (den + eps);
    }
    free(pq);
}

/* -------------------------------------------------------------- LoLA ---- */

/*
 * [LoLA "Self-Recall Error"] For each candidate pair (k_j, v_j):
 *   SRE_j = || phi(k_j)^T H / (phi(k_j)^T s + eps) - v_j ||^2      (R3)
 * One head: kc [n, d], vc [n, dv], Hst [D, dv], s [D], sre [n].
 */
ORACLE_API void oracle_sre(const double *Hst, const double *s, const double *kc,
                           const double *vc, int n, int d, int dv, double eps,
                           double *sre)
{
    double *pred = (double *)malloc(sizeof(double) * (size_t)dv);
    for (int j = 0; j < n; ++j) {
        oracle_readout(kc + (long)j * d, d, dv, eps, Hst, s, pred);
        double err = 0.0;
        for (int e = 0; e < dv; ++e) {
            double diff = pred[e] - vc[(long)j * dv + e];
            err += diff * diff;
        }
        sre[j] = err;
    }
    free(pred);
}

/* Candidate x comes before y in retention order: higher SRE first, an exact
 * tie goes to the smaller token position. */
static int retained_before(const double *sc, const int *pos, int x, int y)
{
    if (sc[x] != sc[y]) return sc[x] > sc[y];
    return pos[x] < pos[y];
}

/*
 * [LoLA "Inference strategy" step 2] Keep the min(keep, n) candidates with
 * the highest SRE (exact ties: smaller position first). keep_idx receives the
 * kept candidate slots in ascending token position. Returns the kept count.
 * Plain insertion sort: n is a few hundred at most.
 */
ORACLE_API int oracle_topk(const double *sre, const int *pos, int n, int keep, int *keep_idx)
{
    int *order = (int *)malloc(sizeof(int) * (size_t)(n > 0 ? n : 1));
    for (int i = 0; i < n; ++i) {
        int j = i;
        while (j > 0 && retained_before(sre, pos, i, order[j - 1])) {
            order[j] = order[j - 1];
            --j;
        }
        order[j] = i;
    }
    int m = keep < n ? keep : n;
    for (int i = 0; i < m; ++i) {
        int j = i;
        while (j > 0 && pos[order[i]] < pos[keep_idx[j - 1]]) {
            keep_idx[j] = keep_idx[j - 1];
            --j;
        }
        keep_idx[j] = order[i];
    }
    free(order);
    return m;
}

/*
 * [LoLA "Inference strategy" step 3] Every candidate not kept is written into
 * the linear state by an outer-product update: H += phi(k_j) v_j^T,
 * s += phi(k_j). One head, in candidate order.
 */
ORACLE_API void oracle_merge(double *Hst, double *s, const double *kc, const double *vc,
                             int n, const int *keep_idx, int nkeep, int d, int dv)
{
    long D = oracle_packed_dim(d);
    double *pk = (double *)malloc(sizeof(double) * (size_t)D);
    for (int j = 0; j < n; ++j) {
        int kept = 0;
        for (int t = 0; t < nkeep; ++t) kept |= (keep_idx[t] == j);
        if (kept) continue;
        oracle_phi(kc + (long)j * d, d, pk);
        for (long r = 0; r < D; ++r) {
            for (int e = 0; e < dv; ++e) Hst[r * dv + e] += pk[r] * vc[(long)j * dv + e];
            s[r] += pk[r];
        }
    }
    free(pk);
}

/*
 * [LoLA "Inference strategy" step 4; Methodology 1-3] Hybrid readout of one
 * query q (reading R4): the window and sparse-cache pairs enter with the
 * softmax kernel exp(q.k * tau), the linear state with phi(q)^T H and
 * phi(q)^T s; one shared denominator:
 *   o = [sum_{j in W u S} exp(q.k_j tau) v_j + phi(q)^T H]
 *       / [sum_{j in W u S} exp(q.k_j tau) + phi(q)^T s + eps]
 * wk/wv [nw, d]/[nw, dv] are the window pairs, ck/cv [nc, ...] the cache.
 */
ORACLE_API void oracle_hybrid_readout(const double *q, int d, int dv, double eps, double tau,
                                      const double *wk, const double *wv, int nw,
                                      const double *ck, const double *cv, int nc,
                                      const double *Hst, const double *s, double *o)
{
    long D = oracle_packed_dim(d);
    double *pq = (double *)malloc(sizeof(double) * (size_t)D);
    double *num = (double *)malloc(sizeof(double) * (size_t)dv);
    oracle_phi(q, d, pq);
    double den = 0.0;
    for (int e = 0; e < dv; ++e) num[e] = 0.0;
    for (int pass = 0; pass < 2; ++pass) {
        const double *K = pass ? ck : wk;
        const double *V = pass ? cv : wv;
        int n = pass ? nc : nw;
        for (int j = 0; j < n; ++j) {
            double dot = 0.0;
            for (int a = 0; a < d; ++a) dot += q[a] * K[(long)j * d + a];
            double w = exp(dot * tau);
            den += w;
            for (int e = 0; e < dv; ++e) num[e] += w * V[(long)j * dv + e];
        }
    }
    for (long r = 0; r < D; ++r) {
        den += pq[r] * s[r];
        for (int e = 0; e < dv; ++e) num[e] += pq[r] * Hst[r * dv + e];
    }
    for (int e = 0; e < dv; ++e) o[e] = num[e] / (den + eps);
    free(pq);
    free(num);
}

/* ------------------------------------------------ batched over heads ----- */

ORACLE_API void oracle_quadratic_heads(int nh, const double *q, const double *k,
                                       const double *v, long T, int d, int dv, double eps,
                                       const long *rows, long nrows, double *o)
{
    long n = rows ? nrows : T;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < nh; ++h)
        oracle_quadratic(q + (long)h * T * d, k + (long)h * T * d, v + (long)h * T * dv, T,
                         d, dv, eps, rows, nrows, o + (long)h * n * dv);
}

ORACLE_API void oracle_recurrent_heads(int nh, const double *q, const double *k,
                                       const double *v, long T, int d, int dv, double eps,
                                       double *Hst, double *s, double *o)
{
    long D = oracle_packed_dim(d);
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < nh; ++h)
        oracle_recurrent(q ? q + (long)h * T * d : NULL, k + (long)h * T * d,
                         v + (long)h * T * dv, T, d, dv, eps, Hst + (long)h * D * dv,
                         s + (long)h * D, o ? o + (long)h * T * dv : NULL);
}

ORACLE_API void oracle_sre_heads(int nh, const double *Hst, const double *s, const double *kc,
                                 const double *vc, int n, int d, int dv, double eps,
                                 double *sre)
{
    long D = oracle_packed_dim(d);
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < nh; ++h)
        oracle_sre(Hst + (long)h * D * dv, s + (long)h * D, kc + (long)h * n * d,
                   vc + (long)h * n * dv, n, d, dv, eps, sre + (long)h * n);
}

ORACLE_API void oracle_merge_heads(int nh, double *Hst, double *s, const double *kc,
                                   const double *vc, int n, const int *keep_idx, int nkeep,
                                   int d, int dv)
{
    long D = oracle_packed_dim(d);
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < nh; ++h)
        oracle_merge(Hst + (long)h * D * dv, s + (long)h * D, kc + (long)h * n * d,
                     vc + (long)h * n * dv, n, keep_idx + (long)h * nkeep, nkeep, d, dv);
}

/*
 * One segment of hybrid readouts for nh heads. Query i (absolute position
 * seg0 + r, r < nq) sees window pairs at positions [w0, seg0 + r] of that
 * head's k/v [T, d] and the nc cache pairs ck/cv of that head.
 */
ORACLE_API void oracle_hybrid_segment_heads(int nh, const double *q, const double *k,
                                            const double *v, long T, int d, int dv,
                                            double eps, double tau, long w0, long seg0,
                                            int nq, const double *ck, const double *cv,
                                            int nc, int cstride, const double *Hst,
                                            const double *s, double *o)
{
    long D = oracle_packed_dim(d);
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < nh; ++h) {
        const double *qh = q + (long)h * T * d, *kh = k + (long)h * T * d;
        const double *vh = v + (long)h * T * dv;
        for (int r = 0; r < nq; ++r) {
            long i = seg0 + r;
            oracle_hybrid_readout(qh + i * d, d, dv, eps, tau, kh + w0 * d, vh + w0 * dv,
                                  (int)(i - w0 + 1), ck + (long)h * cstride * d,
                                  cv + (long)h * cstride * dv, nc, Hst + (long)h * D * dv,
                                  s + (long)h * D, o + ((long)h * T + i) * dv);
        }
    }
}

/* ------------------------------------------- multi-factor features ----- */

/*
 * [KATA s2.3 "Variants": KATA-Mg (several PSD factors) and KATA-Sigma-g
 * (summed PSD factors), which trade the state size against the packing.]
 * The page names the variants but not how the factors are formed. Reading
 * R13: the head vector u (d values) is cut into g contiguous sub-vectors
 * u_r = u[r p .. r p + p - 1], p = d / g, and each gives the rank-one PSD
 * factor u_r u_r^T of s2.2:
 *   feature 0, M1:      psi(u) = u u^T                          kernel (q.k)^2
 *   feature 1, Mg:      psi(u) = blockdiag(u_1 u_1^T, ..., u_g u_g^T)
 *                       (the g factors kept apart)              kernel sum_r (q_r.k_r)^2
 *   feature 2, Sigma-g: psi(u) = sum_r u_r u_r^T (the factors summed into
 *                       one p x p PSD matrix)                   kernel sum_{r,s} (q_r.k_s)^2
 * Both are PSD features, so every attention weight <psi(q), psi(k)>_F is
 * non-negative; g = 1 gives M1 for both. Packing: each symmetric p x p block
 * as the upper triangle with sqrt(2) on off-diagonal entries (R1); Mg's g
 * blocks one after another (block r at rows r p(p+1)/2 ...).
 */
static int oracle_feature_ok(int d, int feature, int g)
{
    if (feature == 0) return g == 1;
    return (feature == 1 || feature == 2) && g >= 1 && d % g == 0;
}

/* Feature dimension: d(d+1)/2 (M1), g p(p+1)/2 (Mg), p(p+1)/2 (Sigma-g); 0 if invalid. */
ORACLE_API long oracle_feature_dim(int d, int feature, int g)
{
    if (!oracle_feature_ok(d, feature, g)) return 0;
    if (feature == 0) return oracle_packed_dim(d);
    int p = d / g;
    return feature == 1 ? (long)g * oracle_packed_dim(p) : oracle_packed_dim(p);
}

/* psi(x) in the packed layout above (R13). */
ORACLE_API void oracle_phi_feature(const double *x, int d, int feature, int g, double *phi)
{
    if (feature == 0) {
        oracle_phi(x, d, phi);
        return;
    }
    const int p = d / g;
    const long Dp = oracle_packed_dim(p);
    const double r2 = sqrt(2.0);
    if (feature == 2)
        for (long i = 0; i < Dp; ++i) phi[i] = 0.0;
    for (int r = 0; r < g; ++r) {
        const double *xr = x + (long)r * p;
        double *dst = feature == 1 ? phi + (long)r * Dp : phi;
        for (int a = 0; a < p; ++a)
            for (int b = a; b < p; ++b) {
                double w = (a == b) ? 1.0 : r2;
                double val = w * xr[a] * xr[b];
                long at = oracle_packed_index(p, a, b);
                if (feature == 1) dst[at] = val; else dst[at] += val;
            }
    }
}

/* The kernel <psi(q), psi(k)> from the sub-vectors' dot products, no feature map (R13). */
ORACLE_API double oracle_kernel_feature(const double *q, const double *k, int d, int feature,
                                        int g)
{
    if (feature == 0) {
        double dot = 0.0;
        for (int a = 0; a < d; ++a) dot += q[a] * k[a];
        return dot * dot;
    }
    const int p = d / g;
    double sum = 0.0;
    for (int r = 0; r < g; ++r)
        for (int t = 0; t < g; ++t) {
            if (feature == 1 && t != r) continue;  /* Mg: each factor with itself only */
            double dot = 0.0;
            for (int a = 0; a < p; ++a) dot += q[(long)r * p + a] * k[(long)t * p + a];
            sum += dot * dot;
        }
    return sum;
}

/*
 * Quadratic form with a variant's kernel (R2, R3, R13), one head:
 *   o_i = sum_{j<=i} kappa(q_i, k_j) v_j / (sum_{j<=i} kappa(q_i, k_j) + eps).
 */
ORACLE_API void oracle_quadratic_feature(const double *q, const double *k, const double *v,
                                         long T, int d, int dv, double eps, int feature, int g,
                                         double *o)
{
    double *num = (double *)malloc(sizeof(double) * (size_t)dv);
    for (long i = 0; i < T; ++i) {
        double den = 0.0;
        for (int e = 0; e < dv; ++e) num[e] = 0.0;
        for (long j = 0; j <= i; ++j) {
            double w = oracle_kernel_feature(q + i * d, k + j * d, d, feature, g);
            den += w;
            for (int e = 0; e < dv; ++e) num[e] += w * v[j * dv + e];
        }
        for (int e = 0; e < dv; ++e) o[i * dv + e] = num[e] / (den + eps);
    }
    free(num);
}

/*
 * Literal recurrent form with a variant's feature (R2, R3, R13), one head:
 *   H += psi(k_i) v_i^T; s += psi(k_i); o_i = psi(q_i)^T H / (psi(q_i)^T s + eps).
 * Hst [Df, dv], s [Df] (Df = oracle_feature_dim) in and out; o may be NULL.
 */
ORACLE_API void oracle_recurrent_feature(const double *q, const double *k, const double *v,
                                         long T, int d, int dv, double eps, int feature,
                                         int g, double *Hst, double *s, double *o)
{
    long D = oracle_feature_dim(d, feature, g);
    double *pk = (double *)malloc(sizeof(double) * (size_t)D);
    double *pq = (double *)malloc(sizeof(double) * (size_t)D);
    for (long i = 0; i < T; ++i) {
        oracle_phi_feature(k + i * d, d, feature, g, pk);
        for (long r = 0; r < D; ++r) {
            for (int e = 0; e < dv; ++e) Hst[r * dv + e] += pk[r] * v[i * dv + e];
            s[r] += pk[r];
        }
        if (!o) continue;
        oracle_phi_feature(q + i * d, d, feature, g, pq);
        double den = 0.0;
        for (long r = 0; r < D; ++r) den += pq[r] * s[r];
        for (int e = 0; e < dv; ++e) {
            double num = 0.0;
            for (long r = 0; r < D; ++r) num += pq[r] * Hst[r * dv + e];
            o[i * dv + e] = num / (den + eps);
        }
    }
    free(pk);
    free(pq);
}

ORACLE_API void oracle_quadratic_feature_heads(int nh, const double *q, const double *k,
                                               const double *v, long T, int d, int dv,
                                               double eps, int feature, int g, double *o)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < nh; ++h)
        oracle_quadratic_feature(q + (long)h * T * d, k + (long)h * T * d,
                                 v + (long)h * T * dv, T, d, dv, eps, feature, g,
                                 o + (long)h * T * dv);
}

ORACLE_API void oracle_recurrent_feature_heads(int nh, const double *q, const double *k,
                                               const double *v, long T, int d, int dv,
                                               double eps, int feature, int g, double *Hst,
                                               double *s, double *o)
{
    long D = oracle_feature_dim(d, feature, g);
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < nh; ++h)
        oracle_recurrent_feature(q ? q + (long)h * T * d : NULL, k + (long)h * T * d,
                                 v + (long)h * T * dv, T, d, dv, eps, feature, g,
                                 Hst + (long)h * D * dv, s + (long)h * D,
                                 o ? o + (long)h * T * dv : NULL);
}
