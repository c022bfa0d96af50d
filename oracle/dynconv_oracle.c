/*
 * dynconv_oracle.c -- plain fp64 CPU oracle for dynamic short convolutions.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA path.
 *
 * What it computes ("Dynamic Short Convolutions Improve Transformers",
 * gist.science technical summary, section "Dynamic Short Convolutions"):
 *
 *   filter      w[n,c,j]  generated per token from the hidden state h[n,:] by a
 *                          learned linear map (no bias, no nonlinearity):
 *                 low-rank  z[n,k] = sum_i h[n,i] A[i,k]
 *                           w[n,c,j] = sum_k z[n,k] B[k, c*K + j]
 *                 head-wise w[n,c,j] = sum_i h[n,i] W[i, (c / head_dim)*K + j]
 *                           (one filter per head, shared by its channels)
 *   conv        y[n,c] = u[n,c] + sum_{j=0}^{K-1} [n-j >= s(n)] w[n,c,j] u[n-j,c]
 *                 ("Mechanism" formula with tap 0 = current token, plus the
 *                 residual X = X + dynamicShortConv(X) of "Placement");
 *                 s(n) is the first token of n's sequence or packed document,
 *                 taps before it read zero.
 *
 *   backward (the adjoint of the above, written out term by term):
 *     dw[n,c,j] = [n-j >= s(n)] g[n,c] u[n-j,c]
 *     du[m,c]   = g[m,c] + sum_j [m+j < N, m >= s(m+j)] w[m+j,c,j] g[m+j,c]
 *     low-rank:  dz[n,k] = sum_{c,j} dw[n,c,j] B[k,c*K+j]
 *                dB[k,c*K+j] = sum_n z[n,k] dw[n,c,j]
 *                dA[i,k] = sum_n h[n,i] dz[n,k];   dh[n,i] = sum_k dz[n,k] A[i,k]
 *     head-wise: dwh[n,q,j] = sum_{c in head q} dw[n,c,j]
 *                dW[i,q*K+j] = sum_n h[n,i] dwh[n,q,j]
 *                dh[n,i] = sum_{q,j} dwh[n,q,j] W[i,q*K+j]
 *
 * Every sum runs in index order in fp64.  Loops are parallel only over
 * independent outputs (OpenMP), never over a reduction.
 *
 * Layout: every matrix is dense row-major fp64: u,g,y,du [N,C]; h,dh [N,d];
 * A,dA [d,r]; B,dB [r,C*K]; W,dW [d,H*K]; z,dz [N,r]; cu_seqlens int64 [S+1]
 * with cu_seqlens[0] = 0 and cu_seqlens[S] = N (a dense batch of B sequences
 * of length T is cu_seqlens = 0, T, 2T, ..., BT).
 *
 * Pins: see tests/test_oracle_pins.py (static-conv reduction, zero filter,
 * causality, document isolation, finite differences, adjoint identity,
 * head-wise as a low-rank special case, K = 1 closed form, a hand-worked
 * integer example, and an independent autograd restatement).
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

typedef struct {
    int64_t kind;        /* 0 = low-rank, 1 = head-wise */
    int64_t n_tokens;    /* N */
    int64_t d_model;     /* d */
    int64_t channels;    /* C */
    int64_t ksize;       /* K */
    int64_t rank;        /* r (low-rank only) */
    int64_t head_dim;    /* channels per head (head-wise only) */
    int64_t n_segs;      /* S */
    const int64_t *cu_seqlens;
} orc_problem;

#define ORC_OK 0
#define ORC_BAD 1

static int check(const orc_problem *p)
{
    if (p->n_tokens < 0 || p->d_model < 1 || p->channels < 1 || p->ksize < 1) return ORC_BAD;
    if (p->kind == 0 && p->rank < 1) return ORC_BAD;
    if (p->kind == 1 && (p->head_dim < 1 || p->channels % p->head_dim != 0)) return ORC_BAD;
    if (p->kind != 0 && p->kind != 1) return ORC_BAD;
    if (p->n_segs < 1 || p->cu_seqlens[0] != 0 || p->cu_seqlens[p->n_segs] != p->n_tokens) return ORC_BAD;
    for (int64_t s = 0; s < p->n_segs; ++s)
        if (p->cu_seqlens[s + 1] < p->cu_seqlens[s]) return ORC_BAD;
    return ORC_OK;
}

/* s(n): first token of the sequence/document holding token n. */
static int64_t *segment_starts(const orc_problem *p)
{
    int64_t *st = (int64_t *)malloc(sizeof(int64_t) * (size_t)(p->n_tokens > 0 ? p->n_tokens : 1));
    for (int64_t s = 0; s < p->n_segs; ++s)
        for (int64_t n = p->cu_seqlens[s]; n < p->cu_seqlens[s + 1]; ++n) st[n] = p->cu_seqlens[s];
    return st;
}

/* z[n,:] = h[n,:] A (low-rank stage 1). */
static void lowrank_z_row(const orc_problem *p, const double *h, const double *A, int64_t n, double *z)
{
    const int64_t d = p->d_model, r = p->rank;
    for (int64_t k = 0; k < r; ++k) {
        double acc = 0.0;
        for (int64_t i = 0; i < d; ++i) acc += h[n * d + i] * A[i * r + k];
        z[k] = acc;
    }
}

/* w[n,c,j] for every (c,j) of token n, stored at w[c*K + j]. */
static void filter_row(const orc_problem *p, const double *h, const double *A, const double *BW,
                       int64_t n, double *zscratch, double *w)
{
    const int64_t d = p->d_model, C = p->channels, K = p->ksize;
    if (p->kind == 0) {
        const int64_t r = p->rank;
        lowrank_z_row(p, h, A, n, zscratch);
        for (int64_t c = 0; c < C; ++c)
            for (int64_t j = 0; j < K; ++j) {
                double acc = 0.0;
                for (int64_t k = 0; k < r; ++k) acc += zscratch[k] * BW[k * (C * K) + c * K + j];
                w[c * K + j] = acc;
            }
    } else {
        const int64_t H = C / p->head_dim;
        for (int64_t q = 0; q < H; ++q)
            for (int64_t j = 0; j < K; ++j) {
                double acc = 0.0;
                for (int64_t i = 0; i < d; ++i) acc += h[n * d + i] * BW[i * (H * K) + q * K + j];
                for (int64_t c = q * p->head_dim; c < (q + 1) * p->head_dim; ++c) w[c * K + j] = acc;
            }
    }
}

static int64_t zdim(const orc_problem *p) { return p->kind == 0 ? p->rank : 1; }

/*
 * Forward for the listed tokens (rows == NULL: every token, in order).
 * y_out[i*C + c] = y[rows[i], c]; z_out (nullable, low-rank) [nrows, r];
 * w_out (nullable) [nrows, C*K] holds the generated filters.
 */
int orc_forward(const orc_problem *p, const double *u, const double *h, const double *A,
                const double *BW, int64_t nrows, const int64_t *rows, double *y_out,
                double *z_out, double *w_out)
{
    if (check(p) != ORC_OK) return ORC_BAD;
    const int64_t C = p->channels, K = p->ksize, N = p->n_tokens;
    if (rows == NULL) nrows = N;
    int64_t *st = segment_starts(p);
    int bad = 0;
#pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)zdim(p));
        double *w = (double *)malloc(sizeof(double) * (size_t)(C * K));
#pragma omp for schedule(static)
        for (int64_t i = 0; i < nrows; ++i) {
            const int64_t n = rows ? rows[i] : i;
            if (n < 0 || n >= N) { bad = 1; continue; }
            filter_row(p, h, A, BW, n, z, w);
            for (int64_t c = 0; c < C; ++c) {
                double acc = u[n * C + c];
                for (int64_t j = 0; j < K; ++j)
                    if (n - j >= st[n]) acc += w[c * K + j] * u[(n - j) * C + c];
                y_out[i * C + c] = acc;
            }
            if (z_out && p->kind == 0)
                for (int64_t k = 0; k < p->rank; ++k) z_out[i * p->rank + k] = z[k];
            if (w_out)
                for (int64_t e = 0; e < C * K; ++e) w_out[i * C * K + e] = w[e];
        }
        free(z);
        free(w);
    }
    free(st);
    return bad ? ORC_BAD : ORC_OK;
}

/* dw[n,c,j] for one token into dw[c*K + j]. */
static void dfilter_row(const orc_problem *p, const int64_t *st, const double *g, const double *u,
                        int64_t n, double *dw)
{
    const int64_t C = p->channels, K = p->ksize;
    for (int64_t c = 0; c < C; ++c)
        for (int64_t j = 0; j < K; ++j)
            dw[c * K + j] = (n - j >= st[n]) ? g[n * C + c] * u[(n - j) * C + c] : 0.0;
}

/* Generator-space gradient of one token: dz[n,:] (low-rank, r values) or dwh[n,:,:] (head-wise, H*K). */
static void dgen_row(const orc_problem *p, const double *BW, const double *dw, double *out)
{
    const int64_t C = p->channels, K = p->ksize;
    if (p->kind == 0) {
        for (int64_t k = 0; k < p->rank; ++k) {
            double acc = 0.0;
            for (int64_t c = 0; c < C; ++c)
                for (int64_t j = 0; j < K; ++j) acc += dw[c * K + j] * BW[k * (C * K) + c * K + j];
            out[k] = acc;
        }
    } else {
        const int64_t H = C / p->head_dim;
        for (int64_t q = 0; q < H; ++q)
            for (int64_t j = 0; j < K; ++j) {
                double acc = 0.0;
                for (int64_t c = q * p->head_dim; c < (q + 1) * p->head_dim; ++c) acc += dw[c * K + j];
                out[q * K + j] = acc;
            }
    }
}

static int64_t gdim(const orc_problem *p)
{
    return p->kind == 0 ? p->rank : (p->channels / p->head_dim) * p->ksize;
}

/*
 * Per-token backward for the listed tokens (rows == NULL: all).
 * du_out [nrows,C]; dgen_out (nullable) [nrows, r] = dz (low-rank) or
 * [nrows, H*K] = dwh (head-wise); dh_out (nullable) [nrows, d].
 */
int orc_backward_rows(const orc_problem *p, const double *g, const double *u, const double *h,
                      const double *A, const double *BW, int64_t nrows, const int64_t *rows,
                      double *du_out, double *dgen_out, double *dh_out)
{
    if (check(p) != ORC_OK) return ORC_BAD;
    const int64_t C = p->channels, K = p->ksize, N = p->n_tokens, d = p->d_model;
    if (rows == NULL) nrows = N;
    int64_t *st = segment_starts(p);
    int bad = 0;
#pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)zdim(p));
        double *w = (double *)malloc(sizeof(double) * (size_t)(C * K));
        double *dw = (double *)malloc(sizeof(double) * (size_t)(C * K));
        double *dg = (double *)malloc(sizeof(double) * (size_t)gdim(p));
#pragma omp for schedule(static)
        for (int64_t i = 0; i < nrows; ++i) {
            const int64_t m = rows ? rows[i] : i;
            if (m < 0 || m >= N) { bad = 1; continue; }
            /* du[m,c] = g[m,c] + sum_j w[m+j,c,j] g[m+j,c] over taps that reach m from its own segment */
            for (int64_t c = 0; c < C; ++c) du_out[i * C + c] = g[m * C + c];
            for (int64_t j = 0; j < K; ++j) {
                const int64_t n = m + j;
                if (n >= N || m < st[n]) continue;
                filter_row(p, h, A, BW, n, z, w);
                for (int64_t c = 0; c < C; ++c) du_out[i * C + c] += w[c * K + j] * g[n * C + c];
            }
            if (dgen_out || dh_out) {
                dfilter_row(p, st, g, u, m, dw);
                dgen_row(p, BW, dw, dg);
                if (dgen_out)
                    for (int64_t e = 0; e < gdim(p); ++e) dgen_out[i * gdim(p) + e] = dg[e];
                if (dh_out) {
                    for (int64_t a = 0; a < d; ++a) {
                        double acc = 0.0;
                        if (p->kind == 0)
                            for (int64_t k = 0; k < p->rank; ++k) acc += dg[k] * A[a * p->rank + k];
                        else
                            for (int64_t e = 0; e < gdim(p); ++e) acc += dg[e] * BW[a * gdim(p) + e];
                        dh_out[i * d + a] = acc;
                    }
                }
            }
        }
        free(z); free(w); free(dw); free(dg);
    }
    free(st);
    return bad ? ORC_BAD : ORC_OK;
}

/*
 * Parameter gradients, full: low-rank dA [d,r] and dB [r,C*K]; head-wise dW
 * [d,H*K] (dA ignored).  Each entry is one sum over tokens in order.
 */
int orc_param_grads(const orc_problem *p, const double *g, const double *u, const double *h,
                    const double *A, const double *BW, double *dA, double *dBW)
{
    if (check(p) != ORC_OK) return ORC_BAD;
    const int64_t C = p->channels, K = p->ksize, N = p->n_tokens, d = p->d_model;
    const int64_t G = gdim(p);
    int64_t *st = segment_starts(p);
    double *dgen = (double *)malloc(sizeof(double) * (size_t)(N * G + 1));
    double *zall = (double *)malloc(sizeof(double) * (size_t)(N * zdim(p) + 1));
#pragma omp parallel
    {
        double *dw = (double *)malloc(sizeof(double) * (size_t)(C * K));
#pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            dfilter_row(p, st, g, u, n, dw);
            dgen_row(p, BW, dw, dgen + n * G);
            if (p->kind == 0) lowrank_z_row(p, h, A, n, zall + n * p->rank);
        }
        free(dw);
    }
    if (p->kind == 0) {
        const int64_t r = p->rank;
#pragma omp parallel for schedule(static)
        for (int64_t e = 0; e < d * r; ++e) {
            const int64_t a = e / r, k = e % r;
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) acc += h[n * d + a] * dgen[n * r + k];
            dA[e] = acc;
        }
#pragma omp parallel for schedule(static)
        for (int64_t e = 0; e < r * C * K; ++e) {
            const int64_t k = e / (C * K), col = e % (C * K), c = col / K, j = col % K;
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n)
                if (n - j >= st[n]) acc += zall[n * r + k] * (g[n * C + c] * u[(n - j) * C + c]);
            dBW[e] = acc;
        }
    } else {
#pragma omp parallel for schedule(static)
        for (int64_t e = 0; e < d * G; ++e) {
            const int64_t a = e / G, col = e % G;
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) acc += h[n * d + a] * dgen[n * G + col];
            dBW[e] = acc;
        }
    }
    free(dgen);
    free(zall);
    free(st);
    return ORC_OK;
}

/*
 * Selected parameter-gradient entries, for sizes where the full reduction is
 * too slow: low-rank dB[k, col] (which = 1) or dA[a, k] (which = 0);
 * head-wise dW[a, col] (which = 2).  idx0/idx1 give the two indices.
 */
int orc_param_grad_entries(const orc_problem *p, const double *g, const double *u, const double *h,
                           const double *A, const double *BW, int64_t which, int64_t n_entries,
                           const int64_t *idx0, const int64_t *idx1, double *out)
{
    if (check(p) != ORC_OK) return ORC_BAD;
    const int64_t C = p->channels, K = p->ksize, N = p->n_tokens, d = p->d_model;
    int64_t *st = segment_starts(p);
    for (int64_t e = 0; e < n_entries; ++e) {
        const int64_t i0 = idx0[e], i1 = idx1[e];
        double acc = 0.0;
        if (which == 1 && p->kind == 0) {           /* dB[k=i0, col=i1] */
            const int64_t c = i1 / K, j = i1 % K;
            for (int64_t n = 0; n < N; ++n) {
                if (n - j < st[n]) continue;
                double zk = 0.0;
                for (int64_t a = 0; a < d; ++a) zk += h[n * d + a] * A[a * p->rank + i0];
                acc += zk * (g[n * C + c] * u[(n - j) * C + c]);
            }
        } else if (which == 0 && p->kind == 0) {    /* dA[a=i0, k=i1] */
            double *dzk = (double *)malloc(sizeof(double) * (size_t)(N + 1));
#pragma omp parallel for schedule(static)
            for (int64_t n = 0; n < N; ++n) {
                double s = 0.0;
                for (int64_t c = 0; c < C; ++c)
                    for (int64_t j = 0; j < K; ++j)
                        if (n - j >= st[n]) s += (g[n * C + c] * u[(n - j) * C + c]) * BW[i1 * (C * K) + c * K + j];
                dzk[n] = s;
            }
            for (int64_t n = 0; n < N; ++n) acc += h[n * d + i0] * dzk[n];
            free(dzk);
        } else if (which == 2 && p->kind == 1) {    /* dW[a=i0, col=i1] */
            const int64_t q = i1 / K, j = i1 % K;
            for (int64_t n = 0; n < N; ++n) {
                if (n - j < st[n]) continue;
                double s = 0.0;
                for (int64_t c = q * p->head_dim; c < (q + 1) * p->head_dim; ++c)
                    s += g[n * C + c] * u[(n - j) * C + c];
                acc += h[n * d + i0] * s;
            }
        } else {
            free(st);
            return ORC_BAD;
        }
        out[e] = acc;
    }
    free(st);
    return ORC_OK;
}

/*
 * One decode step for a batch of sequences (the Mechanism formula at the newest
 * token of each sequence; the K-1 previous conv inputs come from a rolling state):
 *   y[b,c] = u[b,c] + sum_{j<K} w[b,c,j] x_j[b,c],   x_0 = u[b,c],  x_j = state[b, j-1, c]
 * with w[b,:,:] the filter generated from h[b,:]; then state[b,j,c] <- x_j[b,c]
 * for j = 0 .. K-2.  p->n_tokens is the batch (one token per sequence); the
 * segment table is not used.  state is [batch, K-1, C], updated in place.
 */
int orc_decode_step(const orc_problem *p, const double *u, const double *h, const double *A, const double *BW,
                    double *state, double *y)
{
    if (p->n_tokens < 0 || p->d_model < 1 || p->channels < 1 || p->ksize < 1) return ORC_BAD;
    if (p->kind == 0 && p->rank < 1) return ORC_BAD;
    if (p->kind == 1 && (p->head_dim < 1 || p->channels % p->head_dim != 0)) return ORC_BAD;
    const int64_t C = p->channels, K = p->ksize;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t b = 0; b < p->n_tokens; ++b) {
        double *w = (double *)malloc(sizeof(double) * (size_t)(C * K));
        double *z = (double *)malloc(sizeof(double) * (size_t)(zdim(p)));
        double *x = (double *)malloc(sizeof(double) * (size_t)K);
        if (!w || !z || !x) {
            bad = 1;
        } else {
            filter_row(p, h, A, BW, b, z, w);
            for (int64_t c = 0; c < C; ++c) {
                x[0] = u[b * C + c];
                for (int64_t j = 1; j < K; ++j) x[j] = state[(b * (K - 1) + (j - 1)) * C + c];
                double acc = x[0];
                for (int64_t j = 0; j < K; ++j) acc += w[c * K + j] * x[j];
                y[b * C + c] = acc;
                for (int64_t j = 0; j + 1 < K; ++j) state[(b * (K - 1) + j) * C + c] = x[j];
            }
        }
        free(w);
        free(z);
        free(x);
    }
    return bad ? ORC_BAD : ORC_OK;
}

/*
 * Rotary position embedding applied to the conv output of the Q and K
 * channels ("Placement": the conv is applied to Q, K and V before RoPE; the
 * rotation fused after it).  The pages name RoPE without fixing a variant;
 * this is the rotation as Su et al. define it ("RoFormer: Enhanced
 * Transformer with Rotary Position Embedding", section 3.4.2): the
 * consecutive channel pairs (2i, 2i+1) of each head of hd channels turn by
 * the angle p * theta_i with theta_i = base^(-2i/hd), p being the token's
 * position in its sequence or packed document (n - s(n)).  Channels
 * c >= n_rot are left as they are.
 *   inverse = 0: (x0, x1) -> (x0 cos - x1 sin, x0 sin + x1 cos)
 *   inverse = 1: (x0, x1) -> (x0 cos + x1 sin, -x0 sin + x1 cos)   (the adjoint)
 * x is [nrows, C] for the listed tokens (rows == NULL: every token), rotated
 * in place; angles and their cosines are computed here in fp64.
 */
int orc_rope(const orc_problem *p, int64_t n_rot, int64_t hd, double base, int64_t inverse, int64_t nrows,
             const int64_t *rows, double *x)
{
    if (check(p) != ORC_OK) return ORC_BAD;
    const int64_t C = p->channels;
    if (hd < 2 || hd % 2 != 0 || n_rot < 0 || n_rot > C || n_rot % hd != 0 || !(base > 0.0)) return ORC_BAD;
    int64_t *st = segment_starts(p);
    int bad = 0;
#pragma omp parallel for schedule(static)
    for (int64_t ri = 0; ri < nrows; ++ri) {
        const int64_t n = rows ? rows[ri] : ri;
        if (n < 0 || n >= p->n_tokens) {
            bad = 1;
            continue;
        }
        const double pos = (double)(n - st[n]);
        for (int64_t c = 0; c < n_rot; c += 2) {
            const int64_t i = (c % hd) / 2;
            const double ang = pos * pow(base, -2.0 * (double)i / (double)hd);
            const double cs = cos(ang), sn = sin(ang);
            const double x0 = x[ri * C + c], x1 = x[ri * C + c + 1];
            if (!inverse) {
                x[ri * C + c] = x0 * cs - x1 * sn;
                x[ri * C + c + 1] = x0 * sn + x1 * cs;
            } else {
                x[ri * C + c] = x0 * cs + x1 * sn;
                x[ri * C + c + 1] = -x0 * sn + x1 * cs;
            }
        }
    }
    free(st);
    return bad ? ORC_BAD : ORC_OK;
}
