/*
 * milo_oracle.c -- plain, slow, fp64 CPU oracle for MILO's block-wise
 * low-rank KV-cache path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (libmilo, its
 * Python binding) may include, link or call this file; only the tests, the
 * smoke check and the bench's CPU-baseline leg use it.  It shares no code,
 * header, table or constant with the CUDA library.
 *
 * What it follows (page titles as cited in the repository docs):
 *  - "MILO: Efficient Many-shot In-Context Learning with Block-wise Low-rank
 *    Compression" (evolve.pub review), Summary: the cache is cut into blocks
 *    of several demonstrations, K (pre-RoPE) and V are each decomposed by SVD
 *    per block, and per-block ranks are chosen by greedily maximising
 *    sum log(1 + sigma^2 / eps^2) under one global rank budget (its Eqs 5-7);
 *    at inference the low-rank factors of the retrieved blocks are rebuilt
 *    before sparse attention.
 *  - same page, Strengths, "Principled, budget-feasible rank allocation":
 *    greedy marginal gains log(1 + sigma^2/eps^2) under a global budget.
 *
 * Every routine is the plain definition written out, in fp64, with the
 * steps in the order the pages give them.  Where the pages leave a point
 * open, the routine concerned states the reading it takes.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* SVD of one block: one-sided (Hestenes) Jacobi applied directly to X.     */
/* ------------------------------------------------------------------------ */
/*
 * X: T x d, row-major.  Outputs (all caller-allocated):
 *   sigma[d]    singular values, descending; entries past min(T,d) are 0,
 *   Vr[d*d]     right singular vectors as columns: Vr[j*d + k] = v_k[j],
 *   US[T*d]     X * Vr = U * diag(sigma) (column k scaled by sigma_k).
 * Columns of a working copy Y = X are rotated pairwise in cyclic order until
 * every pair is orthogonal to within tol = sqrt(T) * DBL_EPSILON (relative
 * cosine); sigma_k is the norm of column k of the converged Y.
 * Returns the number of sweeps used, or -1 when max_sweeps ran out.
 */
int oracle_svd_jacobi(const double *X, int T, int d, int max_sweeps,
                      double *sigma, double *Vr, double *US)
{
    double *Y = (double *)malloc(sizeof(double) * (size_t)T * d); /* column-major */
    double *V = (double *)malloc(sizeof(double) * (size_t)d * d); /* column-major */
    double *nrm = (double *)malloc(sizeof(double) * d);
    int *order = (int *)malloc(sizeof(int) * d);
    if (!Y || !V || !nrm || !order) { free(Y); free(V); free(nrm); free(order); return -2; }
    double normF2 = 0.0;
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < d; ++j) {
            double x = X[(size_t)t * d + j];
            Y[(size_t)j * T + t] = x;
            normF2 += x * x;
        }
    for (int j = 0; j < d; ++j)
        for (int k = 0; k < d; ++k) V[(size_t)k * d + j] = (j == k) ? 1.0 : 0.0;

    const double tol = sqrt((double)T) * DBL_EPSILON;
    /* pairs whose inner product is below this are exactly negligible */
    const double tiny = ((double)d * DBL_EPSILON) * ((double)d * DBL_EPSILON) * normF2;
    int sweeps = 0, converged = 0;
    while (sweeps < max_sweeps && !converged) {
        ++sweeps;
        int rotated = 0;
        for (int p = 0; p < d - 1; ++p) {
            for (int q = p + 1; q < d; ++q) {
                double *yp = Y + (size_t)p * T, *yq = Y + (size_t)q * T;
                double alpha = 0.0, beta = 0.0, gamma = 0.0;
                for (int t = 0; t < T; ++t) {
                    alpha += yp[t] * yp[t];
                    beta += yq[t] * yq[t];
                    gamma += yp[t] * yq[t];
                }
                if (fabs(gamma) <= tiny) continue;
                if (fabs(gamma) <= tol * sqrt(alpha) * sqrt(beta)) continue;
                /* rotation angle that makes columns p and q orthogonal */
                double zeta = (beta - alpha) / (2.0 * gamma);
                double tn = (zeta >= 0.0 ? 1.0 : -1.0) / (fabs(zeta) + sqrt(1.0 + zeta * zeta));
                double c = 1.0 / sqrt(1.0 + tn * tn);
                double s = c * tn;
                for (int t = 0; t < T; ++t) {
                    double a = yp[t], b = yq[t];
                    yp[t] = c * a - s * b;
                    yq[t] = s * a + c * b;
                }
                double *vp = V + (size_t)p * d, *vq = V + (size_t)q * d;
                for (int j = 0; j < d; ++j) {
                    double a = vp[j], b = vq[j];
                    vp[j] = c * a - s * b;
                    vq[j] = s * a + c * b;
                }
                rotated = 1;
            }
        }
        if (!rotated) converged = 1;
    }
    for (int k = 0; k < d; ++k) {
        double s2 = 0.0;
        for (int t = 0; t < T; ++t) s2 += Y[(size_t)k * T + t] * Y[(size_t)k * T + t];
        nrm[k] = sqrt(s2);
        order[k] = k;
    }
    /* stable sort of column indices by norm, descending (insertion sort) */
    for (int i = 1; i < d; ++i) {
        int v = order[i];
        int j = i - 1;
        while (j >= 0 && nrm[order[j]] < nrm[v]) { order[j + 1] = order[j]; --j; }
        order[j + 1] = v;
    }
    int m = T < d ? T : d;
    for (int k = 0; k < d; ++k) {
        int src = order[k];
        sigma[k] = (k < m) ? nrm[src] : 0.0;
        for (int j = 0; j < d; ++j) Vr[(size_t)j * d + k] = V[(size_t)src * d + j];
        for (int t = 0; t < T; ++t) US[(size_t)t * d + k] = Y[(size_t)src * T + t];
    }
    free(Y); free(V); free(nrm); free(order);
    return converged ? sweeps : -1;
}

/* ------------------------------------------------------------------------ */
/* Rank allocation (Eqs 5-7 reading): maximise sum_b sum_{k<r_b}            */
/* log(1 + sigma_{b,k}^2 / eps^2) subject to sum_b r_b = R.                 */
/* ------------------------------------------------------------------------ */
/*
 * key_{b,k} = (sigma_{b,k} / eps_{g(b)})^2, computed as q = sigma/eps then
 * q*q (two correctly rounded IEEE operations).  The marginal gain
 * log(1 + key) is strictly increasing in key, so "largest gain" is decided by
 * comparing keys; rounded log values are never compared.  eps == 0 (an
 * all-zero group) gives key 0.
 */
void oracle_keys(const double *sigma, const double *eps, const int32_t *group,
                 int n_blk, int d, double *key)
{
    for (int b = 0; b < n_blk; ++b) {
        double e = eps[group[b]];
        for (int k = 0; k < d; ++k) {
            double q = (e > 0.0) ? sigma[(size_t)b * d + k] / e : 0.0;
            key[(size_t)b * d + k] = (e > 0.0) ? q * q : 0.0;
        }
    }
}

/* sum over the chosen components of log(1 + key): the objective itself */
double oracle_objective(const double *key, const int32_t *ranks, int n_blk, int d)
{
    double f = 0.0;
    for (int b = 0; b < n_blk; ++b)
        for (int k = 0; k < ranks[b]; ++k) f += log1p(key[(size_t)b * d + k]);
    return f;
}

/* (key desc, linear index asc): returns 1 if candidate a beats candidate b */
static int beats(double ka, int64_t ia, double kb, int64_t ib)
{
    if (ka != kb) return ka > kb;
    return ia < ib;
}

/*
 * Literal greedy: every block starts at rmin_b = min(r_min, rmax_b); then,
 * R - sum rmin_b times, the block whose next component has the largest
 * marginal gain gains one rank.  Ties go to the smaller linear index
 * (block-major, then component).  A binary max-heap over blocks holds each
 * block's next candidate.  keys must be non-increasing within every block
 * (sigma sorted descending), which makes the gains concave.
 * Returns 0, or -1 if R is outside [sum rmin_b, sum rmax_b].
 */
int oracle_allocate_greedy(const double *key, const int32_t *rmax, int n_blk, int d,
                           int64_t R, int r_min, int32_t *ranks)
{
    int64_t lo = 0, hi = 0;
    for (int b = 0; b < n_blk; ++b) {
        int rb = r_min < rmax[b] ? r_min : rmax[b];
        ranks[b] = rb;
        lo += rb;
        hi += rmax[b];
    }
    if (R < lo || R > hi) return -1;
    int *heap = (int *)malloc(sizeof(int) * (n_blk + 1));
    int n = 0;
#define HKEY(b) key[(size_t)(b) * d + ranks[(b)]]
#define HIDX(b) ((int64_t)(b) * d + ranks[(b)])
#define HBEATS(x, y) beats(HKEY(x), HIDX(x), HKEY(y), HIDX(y))
    for (int b = 0; b < n_blk; ++b) {
        if (ranks[b] >= rmax[b]) continue;
        int i = n++;
        heap[i] = b;
        while (i > 0) {
            int par = (i - 1) / 2;
            if (HBEATS(heap[i], heap[par])) { int t = heap[i]; heap[i] = heap[par]; heap[par] = t; i = par; }
            else break;
        }
    }
    for (int64_t step = lo; step < R; ++step) {
        int b = heap[0];
        ranks[b] += 1;
        if (ranks[b] >= rmax[b]) { heap[0] = heap[--n]; }
        int i = 0;
        for (;;) {
            int l = 2 * i + 1, r = l + 1, best = i;
            if (l < n && HBEATS(heap[l], heap[best])) best = l;
            if (r < n && HBEATS(heap[r], heap[best])) best = r;
            if (best == i) break;
            int t = heap[i]; heap[i] = heap[best]; heap[best] = t;
            i = best;
        }
    }
#undef HKEY
#undef HIDX
#undef HBEATS
    free(heap);
    return 0;
}

typedef struct { double key; int64_t idx; } cand_t;

static int cand_cmp(const void *a, const void *b)
{
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (beats(x->key, x->idx, y->key, y->idx)) return -1;
    if (beats(y->key, y->idx, x->key, x->idx)) return 1;
    return 0;
}

/*
 * Global-sort form of the same allocation: all eligible components
 * (rmin_b <= k < rmax_b) sorted by (key desc, index asc); the first
 * R - sum rmin_b are taken.  Equal to the greedy result whenever keys are
 * non-increasing inside each block.
 */
int oracle_allocate_sort(const double *key, const int32_t *rmax, int n_blk, int d,
                         int64_t R, int r_min, int32_t *ranks)
{
    int64_t lo = 0, hi = 0, ne = 0;
    for (int b = 0; b < n_blk; ++b) {
        int rb = r_min < rmax[b] ? r_min : rmax[b];
        ranks[b] = rb;
        lo += rb;
        hi += rmax[b];
        ne += rmax[b] - rb;
    }
    if (R < lo || R > hi) return -1;
    cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (ne > 0 ? ne : 1));
    int64_t n = 0;
    for (int b = 0; b < n_blk; ++b)
        for (int k = ranks[b]; k < rmax[b]; ++k) {
            c[n].key = key[(size_t)b * d + k];
            c[n].idx = (int64_t)b * d + k;
            ++n;
        }
    qsort(c, (size_t)n, sizeof(cand_t), cand_cmp);
    for (int64_t i = 0; i < R - lo; ++i) ranks[c[i].idx / d] += 1;
    free(c);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* INT8 composition: symmetric per-column absmax codes.                      */
/* ------------------------------------------------------------------------ */
/*
 * For each column j of X (rows x cols, leading dimension ld, fp32 values):
 * s_j = absmax_j / 127 (fp32 division), q = clamp(rint(x / s_j), -127, 127)
 * with round-half-to-even; an all-zero column gets s_j = 0 and q = 0.
 * Written in float arithmetic on purpose: the codes are defined on fp32
 * factors.
 */
void oracle_quant_int8_cols(const float *X, int rows, int cols, int ld,
                            int8_t *Q, float *scale)
{
    for (int j = 0; j < cols; ++j) {
        float amax = 0.0f;
        for (int i = 0; i < rows; ++i) {
            float a = fabsf(X[(size_t)i * ld + j]);
            if (a > amax) amax = a;
        }
        float s = amax / 127.0f;
        scale[j] = s;
        for (int i = 0; i < rows; ++i) {
            float qf = (s > 0.0f) ? rintf(X[(size_t)i * ld + j] / s) : 0.0f;
            if (qf > 127.0f) qf = 127.0f;
            if (qf < -127.0f) qf = -127.0f;
            Q[(size_t)i * ld + j] = (int8_t)qf;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Decode: rebuild, RoPE at absolute positions, dense softmax attention.    */
/* ------------------------------------------------------------------------ */
/*
 * RoPE with the rotate-half pairing (i, i + d/2), theta_i = base^(-2i/d):
 *   x'_i       = x_i cos(pos*theta_i) - x_{i+d/2} sin(pos*theta_i)
 *   x'_{i+d/2} = x_{i+d/2} cos(pos*theta_i) + x_i sin(pos*theta_i)
 */
void oracle_rope(double *x, int d, double pos, double base)
{
    int h = d / 2;
    for (int i = 0; i < h; ++i) {
        double theta = pow(base, -2.0 * (double)i / (double)d);
        double a = pos * theta;
        double c = cos(a), s = sin(a);
        double x0 = x[i], x1 = x[i + h];
        x[i] = x0 * c - x1 * s;
        x[i + h] = x1 * c + x0 * s;
    }
}

/* Xhat = A * B with A: T x r, B: r x d, both row-major. */
void oracle_reconstruct(const double *A, const double *B, int T, int r, int d, double *Xhat)
{
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < d; ++j) {
            double acc = 0.0;
            for (int k = 0; k < r; ++k) acc += A[(size_t)t * r + k] * B[(size_t)k * d + j];
            Xhat[(size_t)t * d + j] = acc;
        }
}

/*
 * out[q] = softmax(Q[q] . K^T / sqrt(d)) V for each of nq queries over n
 * keys/values (keys already rotated to their positions).  Two passes: the
 * max score first, then exp(s - max), their sum and the weighted values.
 */
void oracle_attention(const double *Q, int nq, const double *K, const double *V,
                      int n, int d, double *out)
{
    double *s = (double *)malloc(sizeof(double) * (n > 0 ? n : 1));
    double scale = 1.0 / sqrt((double)d);
    for (int qi = 0; qi < nq; ++qi) {
        const double *q = Q + (size_t)qi * d;
        double m = -INFINITY;
        for (int t = 0; t < n; ++t) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j) acc += q[j] * K[(size_t)t * d + j];
            s[t] = acc * scale;
            if (s[t] > m) m = s[t];
        }
        double l = 0.0;
        double *o = out + (size_t)qi * d;
        for (int j = 0; j < d; ++j) o[j] = 0.0;
        for (int t = 0; t < n; ++t) {
            double p = exp(s[t] - m);
            l += p;
            for (int j = 0; j < d; ++j) o[j] += p * V[(size_t)t * d + j];
        }
        for (int j = 0; j < d; ++j) o[j] = (n > 0) ? o[j] / l : 0.0;
    }
    free(s);
}
