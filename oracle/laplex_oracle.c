/*
 * LAPLEX fp64 oracle.  TEST INFRASTRUCTURE ONLY: tests, the smoke check and the
 * bench's CPU-baseline leg may call it; the product path never does.
 *
 * It computes, in plain sequential fp64 arithmetic from the fp32 inputs (promoted
 * exactly), what the LAPLEX operators are defined to compute ("LAPLEX: The FFT of
 * Learnable Laplace Kernels", gist.science technical summary section 2.1):
 *
 *     LAPLEX(a, b)_ij            = exp(-|a_i - b_j|)
 *     LAPLEX(a, phi; b, psi)_ij  = exp(-|a_i - b_j|) * cos(phi_i - psi_j)
 *
 * applied to vectors without forming the matrix, plus the weighted Gram apply
 * A diag(D) A^T v (section 2.2, "Gram operators") and the gradients of
 * <g, out> with respect to every input.
 *
 * The formulation deliberately differs from a prefix/suffix scan over elements:
 * the merged sorted sequence of output and input anchors is walked one DISTINCT
 * VALUE at a time, and every output receives three separate fp64 sums,
 *
 *     L = sum over inputs strictly left   exp(q - p) x
 *     T = sum over inputs at the same value         x
 *     R = sum over inputs strictly right  exp(p - q) x,
 *
 * so out = L + T + R and the anchor gradient uses R - L (sign(0) = 0 for ties,
 * the abs-derivative convention).  The step from one distinct value v' to the
 * next v is the recurrence of section 2.2 ("Exact scan algebra"), written over
 * values: L(v) = exp(v' - v) (L(v') + T(v')).
 *
 * Every function can also return the "magnitude twin" of its output: the same
 * expression with every input replaced by its absolute value and every
 * difference R - L replaced by the sum R + L.  The twin bounds the size of the
 * rounding error any correct fp32 evaluation can make, and the parity tolerance
 * is stated relative to it.
 *
 * Layout: vectors are row-major [rows][B] (row = feature, B batch columns).
 * All outputs are fp64.  Return value: 0 ok, 1 bad argument, 4 non-finite anchor,
 * 7 out of memory.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_OK = 0, OR_ERR_ARG = 1, OR_ERR_NONFINITE = 4, OR_ERR_NOMEM = 7 };

/* ------------------------------------------------------------------ sorting */

typedef struct {
    double v;
    int64_t i;
} keyidx;

static int cmp_keyidx(const void* p, const void* q) {
    const keyidx* A = (const keyidx*)p;
    const keyidx* B = (const keyidx*)q;
    if (A->v < B->v) return -1;
    if (A->v > B->v) return 1;
    return (A->i > B->i) - (A->i < B->i);
}

/* Order of the anchors: ascending value, equal values by ascending original
 * index.  -0.0 and +0.0 compare equal.  This total order makes the sorted
 * permutation unique.  s receives the sorted values (fp64), idx the indices. */
static int sort_anchors(const float* a, int64_t n, double* s, int64_t* idx) {
    keyidx* t = (keyidx*)malloc((size_t)(n > 0 ? n : 1) * sizeof(keyidx));
    if (!t) return OR_ERR_NOMEM;
    for (int64_t i = 0; i < n; ++i) {
        if (!isfinite(a[i])) {
            free(t);
            return OR_ERR_NONFINITE;
        }
        t[i].v = (double)a[i];
        t[i].i = i;
    }
    qsort(t, (size_t)n, sizeof(keyidx), cmp_keyidx);
    for (int64_t r = 0; r < n; ++r) {
        s[r] = t[r].v + 0.0; /* canonical +0 */
        idx[r] = t[r].i;
    }
    free(t);
    return OR_OK;
}

int oracle_sort(const float* a, int64_t n, float* a_sorted, uint32_t* perm) {
    if (n < 1 || !a || !a_sorted || !perm) return OR_ERR_ARG;
    double* s = (double*)malloc((size_t)n * sizeof(double));
    int64_t* idx = (int64_t*)malloc((size_t)n * sizeof(int64_t));
    int rc = (s && idx) ? sort_anchors(a, n, s, idx) : OR_ERR_NOMEM;
    if (rc == OR_OK) {
        for (int64_t r = 0; r < n; ++r) {
            a_sorted[r] = (float)s[r];
            perm[r] = (uint32_t)idx[r];
        }
    }
    free(s);
    free(idx);
    return rc;
}

/* ----------------------------------------------------------- merged sums */

/* For outputs at sorted anchors p[0..np) and inputs at sorted anchors q[0..nq)
 * with values X (row j of the input is X + j*ldx, channels [0, cb)), write
 * per output row o and channel c:
 *     L[o][c] = sum_{q_j <  p_o} exp(q_j - p_o) X[j][c]
 *     T[o][c] = sum_{q_j == p_o}                X[j][c]
 *     R[o][c] = sum_{q_j >  p_o} exp(p_o - q_j) X[j][c]
 * Any of L, T, R may be NULL.  Walks the distinct values of the merged sequence
 * once upward (L, T) and once downward (R). */
static int merged_sums(const double* p, int64_t np_, const double* q, int64_t nq, const double* X,
                       int64_t ldx, int64_t cb, double* L, double* T, double* R) {
    double* acc = (double*)calloc((size_t)cb, sizeof(double));
    double* tie = (double*)calloc((size_t)cb, sizeof(double));
    if (!acc || !tie) {
        free(acc);
        free(tie);
        return OR_ERR_NOMEM;
    }
    if (L || T) {
        int64_t i = 0, o = 0;
        int have = 0;
        double vprev = 0.0;
        while (o < np_) {
            double v = p[o];
            if (i < nq && q[i] < v) v = q[i];
            if (have) {
                double d = exp(vprev - v);
                for (int64_t c = 0; c < cb; ++c) acc[c] = d * (acc[c] + tie[c]);
            }
            for (int64_t c = 0; c < cb; ++c) tie[c] = 0.0;
            while (i < nq && q[i] == v) {
                const double* xr = X + i * ldx;
                for (int64_t c = 0; c < cb; ++c) tie[c] += xr[c];
                ++i;
            }
            while (o < np_ && p[o] == v) {
                for (int64_t c = 0; c < cb; ++c) {
                    if (L) L[o * cb + c] = acc[c];
                    if (T) T[o * cb + c] = tie[c];
                }
                ++o;
            }
            vprev = v;
            have = 1;
        }
    }
    if (R) {
        for (int64_t c = 0; c < cb; ++c) acc[c] = tie[c] = 0.0;
        int64_t i = nq - 1, o = np_ - 1;
        int have = 0;
        double vprev = 0.0;
        while (o >= 0) {
            double v = p[o];
            if (i >= 0 && q[i] > v) v = q[i];
            if (have) {
                double d = exp(v - vprev);
                for (int64_t c = 0; c < cb; ++c) acc[c] = d * (acc[c] + tie[c]);
            }
            for (int64_t c = 0; c < cb; ++c) tie[c] = 0.0;
            while (i >= 0 && q[i] == v) {
                const double* xr = X + i * ldx;
                for (int64_t c = 0; c < cb; ++c) tie[c] += xr[c];
                --i;
            }
            while (o >= 0 && p[o] == v) {
                for (int64_t c = 0; c < cb; ++c) R[o * cb + c] = acc[c];
                --o;
            }
            vprev = v;
            have = 1;
        }
    }
    free(acc);
    free(tie);
    return OR_OK;
}

/* ------------------------------------------------------------ helpers */

typedef struct {
    int64_t n;
    double* s;    /* sorted anchors */
    int64_t* idx; /* original index of sorted position r */
    double* c;    /* cos(theta) in sorted order, or NULL */
    double* sn;   /* sin(theta) in sorted order, or NULL */
} sorted_set;

static void free_set(sorted_set* S) {
    free(S->s);
    free(S->idx);
    free(S->c);
    free(S->sn);
    memset(S, 0, sizeof(*S));
}

static int make_set(const float* a, int64_t n, const float* theta, sorted_set* S) {
    memset(S, 0, sizeof(*S));
    S->n = n;
    S->s = (double*)malloc((size_t)n * sizeof(double));
    S->idx = (int64_t*)malloc((size_t)n * sizeof(int64_t));
    if (!S->s || !S->idx) {
        free_set(S);
        return OR_ERR_NOMEM;
    }
    int rc = sort_anchors(a, n, S->s, S->idx);
    if (rc != OR_OK) {
        free_set(S);
        return rc;
    }
    if (theta) {
        S->c = (double*)malloc((size_t)n * sizeof(double));
        S->sn = (double*)malloc((size_t)n * sizeof(double));
        if (!S->c || !S->sn) {
            free_set(S);
            return OR_ERR_NOMEM;
        }
        for (int64_t r = 0; r < n; ++r) {
            double t = (double)theta[S->idx[r]];
            if (!isfinite(t)) {
                free_set(S);
                return OR_ERR_NONFINITE;
            }
            S->c[r] = cos(t);
            S->sn[r] = sin(t);
        }
    }
    return OR_OK;
}

/* Gather rows of x (original order, [n][B]) into sorted order for channels
 * [c0, c0+cb), multiplied by w[r] (if w) and made absolute (if twin). */
static void gather_rows(const sorted_set* S, const float* x, int64_t B, int64_t c0, int64_t cb,
                        const double* w, int twin, double* out) {
    for (int64_t r = 0; r < S->n; ++r) {
        const float* xr = x + S->idx[r] * B + c0;
        double f = w ? w[r] : 1.0;
        if (twin) f = fabs(f);
        for (int64_t c = 0; c < cb; ++c) {
            double v = (double)xr[c] * f;
            out[r * cb + c] = twin ? fabs(v) : v;
        }
    }
}

#define CHUNK 8 /* channels per pass: bounds the oracle's memory at 8 fp64 per row per array */

static double* dalloc(int64_t count) { return (double*)calloc((size_t)(count > 0 ? count : 1), sizeof(double)); }

/* --------------------------------------------------------- symmetric */

/* y = K x, K_ij = exp(-|a_i - a_j|).  y [n][B] fp64. */
int oracle_sym_apply(const float* a, int64_t n, const float* x, int64_t B, double* y, int twin) {
    if (n < 1 || B < 1 || !a || !x || !y) return OR_ERR_ARG;
    sorted_set S;
    int rc = make_set(a, n, NULL, &S);
    if (rc) return rc;
    int64_t cbmax = B < CHUNK ? B : CHUNK;
    double *X = dalloc(n * cbmax), *L = dalloc(n * cbmax), *T = dalloc(n * cbmax), *R = dalloc(n * cbmax);
    if (!X || !L || !T || !R) rc = OR_ERR_NOMEM;
    for (int64_t c0 = 0; rc == OR_OK && c0 < B; c0 += CHUNK) {
        int64_t cb = (B - c0) < CHUNK ? (B - c0) : CHUNK;
        gather_rows(&S, x, B, c0, cb, NULL, twin, X);
        rc = merged_sums(S.s, n, S.s, n, X, cb, cb, L, T, R);
        for (int64_t r = 0; rc == OR_OK && r < n; ++r)
            for (int64_t c = 0; c < cb; ++c)
                y[S.idx[r] * B + c0 + c] = L[r * cb + c] + T[r * cb + c] + R[r * cb + c];
    }
    free(X); free(L); free(T); free(R);
    free_set(&S);
    return rc;
}

/* Gradients of <g, K x>: gx = K g and
 * ga_i = sum_c g_i (Rx_i - Lx_i) + x_i (Rg_i - Lg_i)   (strict sums, ties excluded).
 * gx [n][B], ga [n]; either may be NULL. */
int oracle_sym_backward(const float* a, int64_t n, const float* x, const float* g, int64_t B, double* gx,
                        double* ga, int twin) {
    if (n < 1 || B < 1 || !a || !x || !g) return OR_ERR_ARG;
    sorted_set S;
    int rc = make_set(a, n, NULL, &S);
    if (rc) return rc;
    int64_t cbmax = B < CHUNK ? B : CHUNK;
    int64_t m = n * cbmax;
    double *X = dalloc(m), *G = dalloc(m), *Lx = dalloc(m), *Rx = dalloc(m), *Lg = dalloc(m), *Tg = dalloc(m),
           *Rg = dalloc(m);
    if (!X || !G || !Lx || !Rx || !Lg || !Tg || !Rg) rc = OR_ERR_NOMEM;
    if (ga && rc == OR_OK)
        for (int64_t i = 0; i < n; ++i) ga[i] = 0.0;
    const double sg = twin ? 1.0 : -1.0;
    for (int64_t c0 = 0; rc == OR_OK && c0 < B; c0 += CHUNK) {
        int64_t cb = (B - c0) < CHUNK ? (B - c0) : CHUNK;
        gather_rows(&S, x, B, c0, cb, NULL, twin, X);
        gather_rows(&S, g, B, c0, cb, NULL, twin, G);
        rc = merged_sums(S.s, n, S.s, n, X, cb, cb, Lx, NULL, Rx);
        if (rc == OR_OK) rc = merged_sums(S.s, n, S.s, n, G, cb, cb, Lg, Tg, Rg);
        for (int64_t r = 0; rc == OR_OK && r < n; ++r) {
            double acc = 0.0;
            for (int64_t c = 0; c < cb; ++c) {
                int64_t e = r * cb + c;
                if (gx) gx[S.idx[r] * B + c0 + c] = Lg[e] + Tg[e] + Rg[e];
                acc += G[e] * (Rx[e] + sg * Lx[e]) + X[e] * (Rg[e] + sg * Lg[e]);
            }
            if (ga) ga[S.idx[r]] += acc;
        }
    }
    free(X); free(G); free(Lx); free(Rx); free(Lg); free(Tg); free(Rg);
    free_set(&S);
    return rc;
}

/* ------------------------------------------------------- rectangular */

/* Canonical rectangular form: outputs at the set P (anchors p, optional phases
 * tp), inputs at the set Q (anchors q, phases tq):
 *     out_i = sum_j exp(-|p_i - q_j|) cos(tp_i - tq_j) x_j
 * with cos(tp - tq) = cos tp cos tq + sin tp sin tq (the cos/sin split); without
 * phases the cosine factor is 1.  x [nq][B], out [np][B]. */
static int rect_forward_pq(const float* p, int64_t np_, const float* tp, const float* q, int64_t nq,
                           const float* tq, const float* x, int64_t B, double* out, int twin) {
    int phased = (tp != NULL);
    sorted_set P, Q;
    int rc = make_set(p, np_, tp, &P);
    if (rc) return rc;
    rc = make_set(q, nq, tq, &Q);
    if (rc) {
        free_set(&P);
        return rc;
    }
    int64_t cbmax = B < CHUNK ? B : CHUNK;
    double *X = dalloc(nq * cbmax), *L = dalloc(np_ * cbmax), *T = dalloc(np_ * cbmax), *R = dalloc(np_ * cbmax);
    if (!X || !L || !T || !R) rc = OR_ERR_NOMEM;
    int nparts = phased ? 2 : 1;
    for (int64_t i = 0; rc == OR_OK && i < np_ * B; ++i) out[i] = 0.0;
    for (int64_t c0 = 0; rc == OR_OK && c0 < B; c0 += CHUNK) {
        int64_t cb = (B - c0) < CHUNK ? (B - c0) : CHUNK;
        for (int part = 0; rc == OR_OK && part < nparts; ++part) {
            const double* wq = phased ? (part == 0 ? Q.c : Q.sn) : NULL;
            const double* wp = phased ? (part == 0 ? P.c : P.sn) : NULL;
            gather_rows(&Q, x, B, c0, cb, wq, twin, X);
            rc = merged_sums(P.s, np_, Q.s, nq, X, cb, cb, L, T, R);
            for (int64_t r = 0; rc == OR_OK && r < np_; ++r) {
                double f = wp ? (twin ? fabs(wp[r]) : wp[r]) : 1.0;
                for (int64_t c = 0; c < cb; ++c) {
                    int64_t e = r * cb + c;
                    out[P.idx[r] * B + c0 + c] += f * (L[e] + T[e] + R[e]);
                }
            }
        }
    }
    free(X); free(L); free(T); free(R);
    free_set(&P);
    free_set(&Q);
    return rc;
}

/* Gradients of <h, out> for the canonical form (h at P, x at Q):
 *   gx_j  = cos tq_j Cq_j + sin tq_j Sq_j,   Cq = E^T (cos tp h), Sq = E^T (sin tp h)
 *   gtq_j = sum_c x_j (-sin tq_j Cq_j + cos tq_j Sq_j)
 *   gtp_i = sum_c h_i (-sin tp_i Zc_i + cos tp_i Zs_i), Zc = E (cos tq x), Zs = E (sin tq x)
 *   gp_i  = sum_c h_i [cos tp_i (Zc^R - Zc^L) + sin tp_i (Zs^R - Zs^L)]_i
 *   gq_j  = sum_c x_j [cos tq_j (Cq^R - Cq^L) + sin tq_j (Sq^R - Sq^L)]_j
 * (^L / ^R: strict left / right parts; without phases cos = 1, sin = 0).
 * Each output may be NULL. */
static int rect_backward_pq(const float* p, int64_t np_, const float* tp, const float* q, int64_t nq,
                            const float* tq, const float* x, const float* h, int64_t B, double* gx, double* gp,
                            double* gq, double* gtp, double* gtq, int twin) {
    int phased = (tp != NULL);
    sorted_set P, Q;
    int rc = make_set(p, np_, tp, &P);
    if (rc) return rc;
    rc = make_set(q, nq, tq, &Q);
    if (rc) {
        free_set(&P);
        return rc;
    }
    int64_t cbmax = B < CHUNK ? B : CHUNK;
    double *Xq = dalloc(nq * cbmax), *Hp = dalloc(np_ * cbmax), *Xw = dalloc(nq * cbmax), *Hw = dalloc(np_ * cbmax);
    double *ZL = dalloc(np_ * cbmax), *ZT = dalloc(np_ * cbmax), *ZR = dalloc(np_ * cbmax);
    double *CL = dalloc(nq * cbmax), *CT = dalloc(nq * cbmax), *CR = dalloc(nq * cbmax);
    if (!Xq || !Hp || !Xw || !Hw || !ZL || !ZT || !ZR || !CL || !CT || !CR) rc = OR_ERR_NOMEM;
    const double sg = twin ? 1.0 : -1.0;
    if (rc == OR_OK) {
        if (gx) for (int64_t i = 0; i < nq * B; ++i) gx[i] = 0.0;
        if (gp) for (int64_t i = 0; i < np_; ++i) gp[i] = 0.0;
        if (gq) for (int64_t i = 0; i < nq; ++i) gq[i] = 0.0;
        if (gtp) for (int64_t i = 0; i < np_; ++i) gtp[i] = 0.0;
        if (gtq) for (int64_t i = 0; i < nq; ++i) gtq[i] = 0.0;
    }
    int nparts = phased ? 2 : 1;
    for (int64_t c0 = 0; rc == OR_OK && c0 < B; c0 += CHUNK) {
        int64_t cb = (B - c0) < CHUNK ? (B - c0) : CHUNK;
        gather_rows(&Q, x, B, c0, cb, NULL, twin, Xq);
        gather_rows(&P, h, B, c0, cb, NULL, twin, Hp);
        for (int part = 0; rc == OR_OK && part < nparts; ++part) {
            /* part 0: cosine channel, part 1: sine channel */
            const double* cq = phased ? (part == 0 ? Q.c : Q.sn) : NULL;
            const double* cp = phased ? (part == 0 ? P.c : P.sn) : NULL;
            /* derivative partners: d/dt cos t = -sin t, d/dt sin t = cos t */
            const double* dq = phased ? (part == 0 ? Q.sn : Q.c) : NULL;
            const double* dp = phased ? (part == 0 ? P.sn : P.c) : NULL;
            const double dsign = (part == 0) ? -1.0 : 1.0;
            /* Z (at P) from x weighted by this part's tq factor; C (at Q) from h weighted by tp factor */
            gather_rows(&Q, x, B, c0, cb, cq, twin, Xw);
            gather_rows(&P, h, B, c0, cb, cp, twin, Hw);
            rc = merged_sums(P.s, np_, Q.s, nq, Xw, cb, cb, ZL, ZT, ZR);
            if (rc == OR_OK) rc = merged_sums(Q.s, nq, P.s, np_, Hw, cb, cb, CL, CT, CR);
            if (rc != OR_OK) break;
            for (int64_t r = 0; r < np_; ++r) {
                double fp = cp ? (twin ? fabs(cp[r]) : cp[r]) : 1.0;
                double fd = dp ? (twin ? fabs(dp[r]) : dsign * dp[r]) : 0.0;
                double accp = 0.0, acct = 0.0;
                for (int64_t c = 0; c < cb; ++c) {
                    int64_t e = r * cb + c;
                    double hv = Hp[e];
                    accp += hv * fp * (ZR[e] + sg * ZL[e]);
                    acct += hv * fd * (ZL[e] + ZT[e] + ZR[e]);
                }
                if (gp) gp[P.idx[r]] += accp;
                if (gtp && phased) gtp[P.idx[r]] += acct;
            }
            for (int64_t r = 0; r < nq; ++r) {
                double fq = cq ? (twin ? fabs(cq[r]) : cq[r]) : 1.0;
                double fd = dq ? (twin ? fabs(dq[r]) : dsign * dq[r]) : 0.0;
                double accq = 0.0, acct = 0.0;
                for (int64_t c = 0; c < cb; ++c) {
                    int64_t e = r * cb + c;
                    double xv = Xq[e];
                    double full = CL[e] + CT[e] + CR[e];
                    if (gx) gx[Q.idx[r] * B + c0 + c] += fq * full;
                    accq += xv * fq * (CR[e] + sg * CL[e]);
                    acct += xv * fd * full;
                }
                if (gq) gq[Q.idx[r]] += accq;
                if (gtq && phased) gtq[Q.idx[r]] += acct;
            }
        }
    }
    free(Xq); free(Hp); free(Xw); free(Hw); free(ZL); free(ZT); free(ZR); free(CL); free(CT); free(CR);
    free_set(&P);
    free_set(&Q);
    return rc;
}

/* y = E x with E_ij = exp(-|a_i - b_j|) [cos(phi_i - psi_j)], x [k][B] at b, y [n][B] at a;
 * transpose: z = E^T x, x [n][B] at a, z [k][B] at b.  phi/psi NULL = unphased. */
int oracle_rect_apply(const float* a, int64_t n, const float* b, int64_t k, const float* phi, const float* psi,
                      const float* x, int64_t B, int transpose, double* out, int twin) {
    if (n < 1 || k < 1 || B < 1 || !a || !b || !x || !out) return OR_ERR_ARG;
    if ((phi == NULL) != (psi == NULL)) return OR_ERR_ARG;
    if (!transpose) return rect_forward_pq(a, n, phi, b, k, psi, x, B, out, twin);
    return rect_forward_pq(b, k, psi, a, n, phi, x, B, out, twin);
}

/* Gradients of <g, out> for oracle_rect_apply.  g lives on the output side.
 * gx has the shape of x; ga [n], gb [k], gphi [n], gpsi [k]; each may be NULL. */
int oracle_rect_backward(const float* a, int64_t n, const float* b, int64_t k, const float* phi, const float* psi,
                         const float* x, const float* g, int64_t B, int transpose, double* gx, double* ga, double* gb,
                         double* gphi, double* gpsi, int twin) {
    if (n < 1 || k < 1 || B < 1 || !a || !b || !x || !g) return OR_ERR_ARG;
    if ((phi == NULL) != (psi == NULL)) return OR_ERR_ARG;
    if (!transpose) return rect_backward_pq(a, n, phi, b, k, psi, x, g, B, gx, ga, gb, gphi, gpsi, twin);
    return rect_backward_pq(b, k, psi, a, n, phi, x, g, B, gx, gb, ga, gpsi, gphi, twin);
}

/* ---------------------------------------------------------------- Gram */

/* y = A diag(D) A^T v with A_ij = exp(-|a_i - b_j|) (section 2.2, "Gram operators"),
 * v [n][B].  Optionally w = A^T v [k][B]. */
int oracle_gram_apply(const float* a, int64_t n, const float* b, int64_t k, const float* D, const float* v, int64_t B,
                      double* y, double* w_out, int twin) {
    if (n < 1 || k < 1 || B < 1 || !a || !b || !D || !v || !y) return OR_ERR_ARG;
    double* w = dalloc(k * B);
    if (!w) return OR_ERR_NOMEM;
    int rc = rect_forward_pq(b, k, NULL, a, n, NULL, v, B, w, twin);
    if (rc == OR_OK && w_out) memcpy(w_out, w, (size_t)(k * B) * sizeof(double));
    /* second pass takes the weighted w as input; it is passed through an fp64 path */
    sorted_set Sa, Sb;
    if (rc == OR_OK) rc = make_set(a, n, NULL, &Sa);
    if (rc == OR_OK) {
        rc = make_set(b, k, NULL, &Sb);
        if (rc) free_set(&Sa);
    }
    if (rc == OR_OK) {
        int64_t cbmax = B < CHUNK ? B : CHUNK;
        double *W = dalloc(k * cbmax), *L = dalloc(n * cbmax), *T = dalloc(n * cbmax), *R = dalloc(n * cbmax);
        if (!W || !L || !T || !R) rc = OR_ERR_NOMEM;
        for (int64_t c0 = 0; rc == OR_OK && c0 < B; c0 += CHUNK) {
            int64_t cb = (B - c0) < CHUNK ? (B - c0) : CHUNK;
            for (int64_t r = 0; r < k; ++r) {
                double d = (double)D[Sb.idx[r]];
                if (twin) d = fabs(d);
                for (int64_t c = 0; c < cb; ++c) W[r * cb + c] = d * w[Sb.idx[r] * B + c0 + c];
            }
            rc = merged_sums(Sa.s, n, Sb.s, k, W, cb, cb, L, T, R);
            for (int64_t r = 0; rc == OR_OK && r < n; ++r)
                for (int64_t c = 0; c < cb; ++c) {
                    int64_t e = r * cb + c;
                    y[Sa.idx[r] * B + c0 + c] = L[e] + T[e] + R[e];
                }
        }
        free(W); free(L); free(T); free(R);
        free_set(&Sa);
        free_set(&Sb);
    }
    free(w);
    return rc;
}

/* Gradient of <g, A diag(D) A^T v> with respect to D: gD_j = sum_c (A^T g)_j (A^T v)_j. */
int oracle_gram_backward_D(const float* a, int64_t n, const float* b, int64_t k, const float* v, const float* g,
                           int64_t B, double* gD, int twin) {
    if (n < 1 || k < 1 || B < 1 || !a || !b || !v || !g || !gD) return OR_ERR_ARG;
    double *wv = dalloc(k * B), *wg = dalloc(k * B);
    int rc = (wv && wg) ? OR_OK : OR_ERR_NOMEM;
    if (rc == OR_OK) rc = rect_forward_pq(b, k, NULL, a, n, NULL, v, B, wv, twin);
    if (rc == OR_OK) rc = rect_forward_pq(b, k, NULL, a, n, NULL, g, B, wg, twin);
    for (int64_t j = 0; rc == OR_OK && j < k; ++j) {
        double acc = 0.0;
        for (int64_t c = 0; c < B; ++c) acc += wg[j * B + c] * wv[j * B + c];
        gD[j] = acc;
    }
    free(wv);
    free(wg);
    return rc;
}

/* -------------------------------------------------- sampled (windowed) */

/* For inputs too large to sort here, evaluate the symmetric operator at chosen
 * output indices directly from the definition, over the anchors within
 * distance `window` of a_i (n <= 2^32 - 1):
 *     y_i  = sum_{|a_j - a_i| <= window} exp(-|a_i - a_j|) x_j
 *     ga_i = sum_c g_i (Rx - Lx) + x_i (Rg - Lg)    (if g given)
 * Anchors are first binned by floor(a / window) (a counting sort, O(n)); each
 * sample then visits the bins within reach.  The dropped mass is at most
 * exp(-window) * sum_j |x_j|, returned in *dropped_bound (per channel maximum).
 * Outputs: y [m][B], ga [m] (NULL to skip), twins likewise.  threads > 1 shares
 * the samples out over that many host threads (when built with OpenMP). */
int oracle_sym_sampled(const float* a, int64_t n, const float* x, const float* g, int64_t B, const int64_t* samples,
                       int64_t m, double window, double* y, double* y_twin, double* ga, double* ga_twin,
                       double* dropped_bound, int threads) {
    if (n < 1 || B < 1 || m < 0 || !a || !x || !samples || !(window > 0)) return OR_ERR_ARG;
    double amin = INFINITY, amax = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
        if (!isfinite(a[i])) return OR_ERR_NONFINITE;
        if (a[i] < amin) amin = a[i];
        if (a[i] > amax) amax = a[i];
    }
    int64_t nb = (int64_t)floor((amax - amin) / window) + 1;
    if (n > (int64_t)UINT32_MAX) return OR_ERR_ARG;
    int64_t* start = (int64_t*)calloc((size_t)nb + 1, sizeof(int64_t));
    uint32_t* order = (uint32_t*)malloc((size_t)n * sizeof(uint32_t));
    if (!start || !order) {
        free(start);
        free(order);
        return OR_ERR_NOMEM;
    }
    for (int64_t i = 0; i < n; ++i) start[(int64_t)floor(((double)a[i] - amin) / window) + 1]++;
    for (int64_t t = 0; t < nb; ++t) start[t + 1] += start[t];
    {
        int64_t* fill = (int64_t*)malloc((size_t)nb * sizeof(int64_t));
        if (!fill) {
            free(start);
            free(order);
            return OR_ERR_NOMEM;
        }
        memcpy(fill, start, (size_t)nb * sizeof(int64_t));
        for (int64_t i = 0; i < n; ++i) order[fill[(int64_t)floor(((double)a[i] - amin) / window)]++] = (uint32_t)i;
        free(fill);
    }
    if (dropped_bound) {
        for (int64_t c = 0; c < B; ++c) dropped_bound[c] = 0.0;
        for (int64_t i = 0; i < n; ++i)
            for (int64_t c = 0; c < B; ++c) dropped_bound[c] += fabs((double)x[i * B + c]);
        for (int64_t c = 0; c < B; ++c) dropped_bound[c] *= exp(-window);
    }
    for (int64_t s = 0; s < m; ++s) {
        if (samples[s] < 0 || samples[s] >= n) {
            free(start);
            free(order);
            return OR_ERR_ARG;
        }
    }
    int failed = 0;
    /* the samples are independent: with threads > 1 they are shared out over host
     * threads, each with its own accumulators; the arithmetic is the same */
#pragma omp parallel for num_threads(threads > 1 ? threads : 1) schedule(dynamic, 64) reduction(| : failed)
    for (int64_t s = 0; s < m; ++s) {
        const int64_t i = samples[s];
        double* tmp = dalloc(10 * B);
        if (!tmp) {
            failed = 1;
            continue;
        }
        double ai = a[i];
        int64_t bi = (int64_t)floor((ai - amin) / window);
        double *Lx = tmp, *Rx = tmp + B, *Tx = tmp + 2 * B, *Lg = tmp + 3 * B, *Rg = tmp + 4 * B;
        double *aLx = tmp + 5 * B, *aRx = tmp + 6 * B, *aT = tmp + 7 * B, *aLg = tmp + 8 * B, *aRg = tmp + 9 * B;
        double ga_acc = 0, gat_acc = 0;
        /* the window spans bins bi-1..bi+1; two more absorb rounding in the bin index */
        for (int64_t t = bi - 2; t <= bi + 2; ++t) {
            if (t < 0 || t >= nb) continue;
            for (int64_t u = start[t]; u < start[t + 1]; ++u) {
                int64_t j = (int64_t)order[u];
                double d = (double)a[j] - ai;
                if (fabs(d) > window) continue;
                double w = exp(-fabs(d));
                for (int64_t c = 0; c < B; ++c) {
                    double xv = x[j * B + c];
                    double gv = g ? (double)g[j * B + c] : 0.0;
                    if (d < 0) {
                        Lx[c] += w * xv; aLx[c] += w * fabs(xv);
                        if (g) { Lg[c] += w * gv; aLg[c] += w * fabs(gv); }
                    } else if (d > 0) {
                        Rx[c] += w * xv; aRx[c] += w * fabs(xv);
                        if (g) { Rg[c] += w * gv; aRg[c] += w * fabs(gv); }
                    } else {
                        Tx[c] += xv; aT[c] += fabs(xv);
                    }
                }
            }
        }
        for (int64_t c = 0; c < B; ++c) {
            if (y) y[s * B + c] = Lx[c] + Tx[c] + Rx[c];
            if (y_twin) y_twin[s * B + c] = aLx[c] + aT[c] + aRx[c];
            if (g) {
                double xi = x[i * B + c], gi = g[i * B + c];
                ga_acc += gi * (Rx[c] - Lx[c]) + xi * (Rg[c] - Lg[c]);
                gat_acc += fabs(gi) * (aRx[c] + aLx[c]) + fabs(xi) * (aRg[c] + aLg[c]);
            }
        }
        if (g && ga) ga[s] = ga_acc;
        if (g && ga_twin) ga_twin[s] = gat_acc;
        free(tmp);
    }
    free(start);
    free(order);
    return failed ? OR_ERR_NOMEM : OR_OK;
}
