/*
 * Plain fp64 CPU oracle for 3D-RoPE video self-attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; it exists so that tests, the smoke check and the bench's
 * CPU-baseline leg have an independent, obviously-correct statement of what
 * the hot path computes.  It shares no code, header or table with the CUDA
 * library.
 *
 * Sources (web pages on full spatiotemporal attention):
 *  - "A video model's architecture: spatiotemporal attention and the 3D VAE"
 *    (anrans.github.io ai-infra-handbooks), section "The latents: the extra
 *    time axis" (token grid), section "How attention sees time: factorised
 *    or full" (what full, spatial and temporal attention sum over), section
 *    "Position: RoPE in three dimensions" (three contiguous head-dim ranges
 *    rotated by t, h and w; token order t-major, w fastest in the printed
 *    sequence-parallel shard listing).
 *  - "CogVideoX Architecture ..." (aifetchly-blog), section 3 "3D Rotary
 *    Position Embeddings": block-diagonal R_3D(t, y, x) and d_h = d_t+d_y+d_x.
 *  - anthology-of-the-sota record sota-390 (CogVideoX's full-vs-factorised
 *    comparison): W.A.L.T's blocks that attend inside local 3D windows.
 *  - "How AI Generates Video" (latentailabs), "What is 3D RoPE": Wan2.1 splits
 *    128 dims into 22/21/21 rotary pairs (axes_dim = [44, 42, 42]).
 *  - "04 HunyuanVideo and Wan" (note.shouss.top), section 2.5: head dim 128,
 *    RoPE split (16, 56, 56); sections 2.3/2.4: joint attention over the
 *    concatenated video+text sequence; section 3.1: a Wan block's text
 *    cross-attention (queries from the video tokens, keys and values from
 *    the text encoder's tokens, which the step does not update).
 *
 * Readings where the pages are silent:
 *  - pairs are adjacent (2j, 2j+1) inside each axis range;
 *  - each axis has its own frequency ladder theta^(-2j/d_a), theta = 10000;
 *  - ranges are ordered t, h, w at offsets 0, d_t, d_t + d_h;
 *  - positions are the integer coordinates from 0 (plus an optional offset,
 *    used only to test translation invariance);
 *  - text tokens are appended after the video tokens and are not rotated;
 *  - softmax scale defaults to 1/sqrt(head_dim).
 *
 * Arithmetic: every quantity in double precision; inputs are bf16 bit
 * patterns widened exactly; nothing is rounded back to bf16.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int T, H, W;          /* post-patch latent grid T', H', W' */
    int n_text;           /* text tokens appended after the video tokens */
    int d_t, d_h, d_w;    /* head-dim ranges rotated by t, h, w */
    double theta;         /* RoPE base */
    int off_t, off_h, off_w; /* coordinate offsets (0 for the method itself) */
} oracle_grid;

enum { ORACLE_FULL = 0, ORACLE_SPATIAL = 1, ORACLE_TEMPORAL = 2, ORACLE_WINDOW = 3 };

enum {
    ORACLE_OK = 0,
    ORACLE_EINVAL = -1,
    ORACLE_ENOMEM = -2,
};

static double bf16_bits_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Coordinates of token i.  Video tokens run t-major, then h, then w
 * (w fastest), as in the shard listing of the handbook's RoPE section.
 * Returns 0 for a video token, 1 for a text token (no coordinates). */
int oracle_token_coords(const oracle_grid *g, long i, int *t, int *h, int *w)
{
    long hw = (long)g->H * g->W;
    long nv = (long)g->T * hw;
    if (i >= nv) {
        *t = *h = *w = -1;
        return 1;
    }
    *t = (int)(i / hw);
    *h = (int)((i / g->W) % g->H);
    *w = (int)(i % g->W);
    return 0;
}

static int grid_ok(const oracle_grid *g, int head_dim)
{
    if (g->T < 1 || g->H < 1 || g->W < 1 || g->n_text < 0) return 0;
    if (g->d_t < 0 || g->d_h < 0 || g->d_w < 0) return 0;
    if ((g->d_t | g->d_h | g->d_w) & 1) return 0;
    if (g->d_t + g->d_h + g->d_w != head_dim) return 0;
    if (!(g->theta > 0.0)) return 0;
    return 1;
}

/* Rotate one head row x (length head_dim) of token i into y.
 * For each axis a in (t, h, w) with range [o_a, o_a + d_a) and each pair
 * j < d_a/2, the pair (x[o_a+2j], x[o_a+2j+1]) is turned by the angle
 * pos_a * theta^(-2j/d_a).  Text tokens are copied unchanged. */
static void rope_row(const oracle_grid *g, int head_dim, const double *x,
                     double *y, long i)
{
    int t, h, w;
    memcpy(y, x, sizeof(double) * (size_t)head_dim);
    if (oracle_token_coords(g, i, &t, &h, &w)) return;

    const int dims[3] = { g->d_t, g->d_h, g->d_w };
    const int pos[3] = { t + g->off_t, h + g->off_h, w + g->off_w };
    int offset = 0;
    for (int a = 0; a < 3; ++a) {
        const int d = dims[a];
        for (int j = 0; j < d / 2; ++j) {
            double phi = (double)pos[a] * pow(g->theta, -2.0 * (double)j / (double)d);
            double c = cos(phi), s = sin(phi);
            double x0 = x[offset + 2 * j];
            double x1 = x[offset + 2 * j + 1];
            y[offset + 2 * j] = x0 * c - x1 * s;
            y[offset + 2 * j + 1] = x0 * s + x1 * c;
        }
        offset += d;
    }
}

/* 3D RoPE of a [BH, N, head_dim] bf16 tensor into fp64 y (same shape). */
int oracle_rope3d(const uint16_t *x, double *y, long BH, long N, int head_dim,
                  const oracle_grid *g)
{
    if (!grid_ok(g, head_dim) || N != (long)g->T * g->H * g->W + g->n_text)
        return ORACLE_EINVAL;
    long rows = BH * N;
#pragma omp parallel
    {
        double *xr = (double *)malloc(sizeof(double) * (size_t)head_dim);
#pragma omp for schedule(static)
        for (long r = 0; r < rows; ++r) {
            for (int c = 0; c < head_dim; ++c)
                xr[c] = bf16_bits_to_double(x[r * head_dim + c]);
            rope_row(g, head_dim, xr, y + r * head_dim, r % N);
        }
        free(xr);
    }
    return ORACLE_OK;
}

/* The keys query token i attends to, following the handbook's section "How
 * attention sees time": full attention takes every token (joint video+text
 * too); the spatial pass takes the H'W' tokens of i's frame; the temporal pass
 * takes the T' tokens at i's spatial position (h, w), one per frame.
 * Writes the key indices to keys[] and returns their count. */
static long key_set(const oracle_grid *g, int mode, const int *win, long i, long N, long *keys)
{
    long cnt = 0;
    if (mode == ORACLE_FULL) {
        for (long j = 0; j < N; ++j) keys[cnt++] = j;
        return cnt;
    }
    int t, h, w;
    oracle_token_coords(g, i, &t, &h, &w);
    const long hw = (long)g->H * g->W;
    if (mode == ORACLE_SPATIAL) {
        for (long j = 0; j < hw; ++j) keys[cnt++] = (long)t * hw + j;
    } else if (mode == ORACLE_TEMPORAL) {
        for (long tt = 0; tt < g->T; ++tt) keys[cnt++] = tt * hw + (long)h * g->W + w;
    } else {
        /* the tokens of the query's window: coordinates in
         * [t0, t0 + wt) x [h0, h0 + wh) x [w0, w0 + ww), t0 = (t / wt) * wt, ... */
        const int t0 = t / win[0] * win[0], h0 = h / win[1] * win[1], w0 = w / win[2] * win[2];
        for (int tt = t0; tt < t0 + win[0]; ++tt)
            for (int hh = h0; hh < h0 + win[1]; ++hh)
                for (int ww = w0; ww < w0 + win[2]; ++ww)
                    keys[cnt++] = tt * hw + (long)hh * g->W + ww;
    }
    return cnt;
}

/*
 * Attention output for selected query rows:
 *   o_r = sum_j softmax_j(scale * <q~_r, k~_j>) v_j   over allowed j,
 *   lse_r = log sum_j exp(scale * <q~_r, k~_j>),
 * where q~, k~ are the 3D-RoPE-rotated rows (when rotate != 0) or the
 * inputs as given (rotate == 0).  q, k, v: bf16 bits [BH, N, head_dim].
 * rows: nrows query indices in [0, N), the same for every bh.
 * out: fp64 [BH, nrows, head_dim]; lse: fp64 [BH, nrows] or NULL.
 */
static int attention_impl(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          long BH, long N, int head_dim, const oracle_grid *g,
                          int mode, const int *win, double scale, int rotate, const long *rows,
                          long nrows, double *out, double *lse)
{
    if (!grid_ok(g, head_dim) || N != (long)g->T * g->H * g->W + g->n_text)
        return ORACLE_EINVAL;
    if (mode != ORACLE_FULL && mode != ORACLE_SPATIAL && mode != ORACLE_TEMPORAL &&
        mode != ORACLE_WINDOW)
        return ORACLE_EINVAL;
    if (mode != ORACLE_FULL && g->n_text != 0) return ORACLE_EINVAL;
    for (long r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return ORACLE_EINVAL;
    if (!(scale > 0.0)) scale = 1.0 / sqrt((double)head_dim);

    const size_t D = (size_t)head_dim;
    double *kr = (double *)malloc(sizeof(double) * (size_t)N * D);
    double *vd = (double *)malloc(sizeof(double) * (size_t)N * D);
    if (!kr || !vd) {
        free(kr);
        free(vd);
        return ORACLE_ENOMEM;
    }

    for (long bh = 0; bh < BH; ++bh) {
        const uint16_t *kb = k + (size_t)bh * N * D;
        const uint16_t *vb = v + (size_t)bh * N * D;
        const uint16_t *qb = q + (size_t)bh * N * D;

        /* rotated keys and widened values of this (batch, head) */
#pragma omp parallel
        {
            double *xr = (double *)malloc(sizeof(double) * D);
#pragma omp for schedule(static)
            for (long j = 0; j < N; ++j) {
                for (size_t c = 0; c < D; ++c) {
                    xr[c] = bf16_bits_to_double(kb[j * D + c]);
                    vd[j * D + c] = bf16_bits_to_double(vb[j * D + c]);
                }
                if (rotate)
                    rope_row(g, head_dim, xr, kr + j * D, j);
                else
                    memcpy(kr + j * D, xr, sizeof(double) * D);
            }
            free(xr);
        }

#pragma omp parallel
        {
            double *qr = (double *)malloc(sizeof(double) * D);
            double *qx = (double *)malloc(sizeof(double) * D);
            double *s = (double *)malloc(sizeof(double) * (size_t)N);
            long *keys = (long *)malloc(sizeof(long) * (size_t)N);
            double *acc = (double *)malloc(sizeof(double) * D);
#pragma omp for schedule(dynamic, 1)
            for (long r = 0; r < nrows; ++r) {
                long i = rows[r];
                for (size_t c = 0; c < D; ++c) qx[c] = bf16_bits_to_double(qb[i * D + c]);
                if (rotate)
                    rope_row(g, head_dim, qx, qr, i);
                else
                    memcpy(qr, qx, sizeof(double) * D);
                const long nk = key_set(g, mode, win, i, N, keys);

                /* scores and their maximum over the keys */
                double m = -INFINITY;
                for (long e = 0; e < nk; ++e) {
                    const double *kj = kr + keys[e] * D;
                    double dot = 0.0;
                    for (size_t c = 0; c < D; ++c) dot += qr[c] * kj[c];
                    s[e] = dot * scale;
                    if (s[e] > m) m = s[e];
                }
                /* normalised weighted sum of values */
                double z = 0.0;
                for (size_t c = 0; c < D; ++c) acc[c] = 0.0;
                for (long e = 0; e < nk; ++e) {
                    double p = exp(s[e] - m);
                    const double *vj = vd + keys[e] * D;
                    z += p;
                    for (size_t c = 0; c < D; ++c) acc[c] += p * vj[c];
                }
                double *o = out + ((size_t)bh * nrows + r) * D;
                for (size_t c = 0; c < D; ++c) o[c] = acc[c] / z;
                if (lse) lse[bh * nrows + r] = m + log(z);
            }
            free(qr);
            free(qx);
            free(s);
            free(keys);
            free(acc);
        }
    }
    free(kr);
    free(vd);
    return ORACLE_OK;
}

int oracle_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     long BH, long N, int head_dim, const oracle_grid *g,
                     int mode, double scale, int rotate, const long *rows,
                     long nrows, double *out, double *lse)
{
    if (mode == ORACLE_WINDOW) return ORACLE_EINVAL;
    return attention_impl(q, k, v, BH, N, head_dim, g, mode, NULL, scale, rotate, rows, nrows,
                          out, lse);
}

/*
 * Local 3D-window attention (anthology record sota-390, the W.A.L.T
 * comparison: blocks that attend inside local 3D windows).  The grid is cut
 * into non-overlapping windows of wt x wh x ww tokens (each dimension must
 * divide the grid's); a token attends to the tokens of its own window, with
 * the same 3D RoPE (absolute coordinates) as full attention.  No text tokens.
 */
int oracle_window_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            long BH, long N, int head_dim, const oracle_grid *g,
                            int wt, int wh, int ww, double scale, int rotate,
                            const long *rows, long nrows, double *out, double *lse)
{
    if (g->n_text != 0 || wt < 1 || wh < 1 || ww < 1) return ORACLE_EINVAL;
    if (g->T % wt != 0 || g->H % wh != 0 || g->W % ww != 0) return ORACLE_EINVAL;
    const int win[3] = {wt, wh, ww};
    return attention_impl(q, k, v, BH, N, head_dim, g, ORACLE_WINDOW, win, scale, rotate, rows,
                          nrows, out, lse);
}

/*
 * Text cross-attention of a Wan block ("04 HunyuanVideo and Wan", section
 * 3.1): every video query row attends to all Nkv text keys; neither side is
 * rotated (the 3D positions belong to the video self-attention).  Same
 * arithmetic as oracle_attention: s_j = scale * q.k_j, m = max s_j,
 * o = sum exp(s_j - m) v_j / sum exp(s_j - m), lse = m + log(sum).
 * q is [BH, Nq, D], k and v are [BH, Nkv, D] bf16 bits; rows index q.
 */
int oracle_cross_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                           long BH, long Nq, long Nkv, int head_dim, double scale,
                           const long *rows, long nrows, double *out, double *lse)
{
    if (BH < 1 || Nq < 1 || Nkv < 1 || head_dim < 1) return ORACLE_EINVAL;
    for (long r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= Nq) return ORACLE_EINVAL;
    if (!(scale > 0.0)) scale = 1.0 / sqrt((double)head_dim);
    const size_t D = (size_t)head_dim;

#pragma omp parallel
    {
        double *qx = (double *)malloc(sizeof(double) * D);
        double *s = (double *)malloc(sizeof(double) * (size_t)Nkv);
        double *acc = (double *)malloc(sizeof(double) * D);
#pragma omp for schedule(dynamic, 16) collapse(2)
        for (long bh = 0; bh < BH; ++bh) {
            for (long r = 0; r < nrows; ++r) {
                const uint16_t *qb = q + ((size_t)bh * Nq + rows[r]) * D;
                const uint16_t *kb = k + (size_t)bh * Nkv * D;
                const uint16_t *vb = v + (size_t)bh * Nkv * D;
                for (size_t c = 0; c < D; ++c) qx[c] = bf16_bits_to_double(qb[c]);
                double m = -INFINITY;
                for (long j = 0; j < Nkv; ++j) {
                    double dot = 0.0;
                    for (size_t c = 0; c < D; ++c)
                        dot += qx[c] * bf16_bits_to_double(kb[j * D + c]);
                    s[j] = dot * scale;
                    if (s[j] > m) m = s[j];
                }
                double z = 0.0;
                for (size_t c = 0; c < D; ++c) acc[c] = 0.0;
                for (long j = 0; j < Nkv; ++j) {
                    double p = exp(s[j] - m);
                    z += p;
                    for (size_t c = 0; c < D; ++c) acc[c] += p * bf16_bits_to_double(vb[j * D + c]);
                }
                double *o = out + ((size_t)bh * nrows + r) * D;
                for (size_t c = 0; c < D; ++c) o[c] = acc[c] / z;
                if (lse) lse[bh * nrows + r] = m + log(z);
            }
        }
        free(qx);
        free(s);
        free(acc);
    }
    return ORACLE_OK;
}
