/*
 * Float64 CPU oracle for the Bi-Level Routing Attention (BRA) forward pass.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library. It shares no code with the
 * CUDA path and must never be used to produce a product result.
 *
 * What it computes follows the official BRA code as walked through on the page
 * "BiFormer ... 前向传播过程" (TRANSFORMER.niftyadmin.cn/n/347023.html), section
 * "BRA模块", together with Algorithm 1 of BiFormer as described on bernice.tw
 * ("Bi-Level Routing Attention", parts one to three):
 *
 *   1. patchify: region p = j*S + i covers rows j*hr..j*hr+hr-1 and columns
 *      i*wr..i*wr+wr-1 (hr = H/S, wr = W/S); tokens inside a region are taken
 *      row-major, t = h*wr + w  (niftyadmin, Algorithm 1 "patchify" and the
 *      rearrange "n (j h) (i w) c -> n (j i) h w c");
 *   2. region queries/keys are the mean of the region's tokens over all C
 *      channels (niftyadmin, eq. 4 prelude: q.mean([2,3]));
 *   3. affinity A[p][p'] = (scale*q_r[p]) . k_r[p'] (niftyadmin, eq. 4);
 *   4. I_r = indices of the topk largest affinities of each row, in descending
 *      order; r_weight = softmax over those topk logits (niftyadmin, eq. 5 and
 *      routing_act = Softmax(dim=-1));
 *   5. for every query token and head m, softmax((scale*q) . k_j) over the
 *      union of the routed regions' tokens taken jointly, times v_j
 *      (niftyadmin, eq. 6 gather and eq. 7 attention, attn_act over the last
 *      dimension);
 *   6. plus LCE(V): a depthwise 5x5 cross-correlation of the whole V image
 *      with zero padding 2 and a per-channel bias (niftyadmin, eq. 7 LCE(V);
 *      module printout "lepe: Conv2d(C, C, 5, padding 2, groups=C)").
 *
 * Readings taken where the pages are silent: scale = d^-0.5 with d = C/heads
 * for both routing and attention; the routing uses all C channels shared by
 * all heads; r_weight is returned only and does not weight K/V; ties in the
 * top-k go to the lower region index.
 *
 * H or W not divisible by S: the bernice.tw notes (section "消融實驗") say that
 * padding the feature map costs compute, which is why S is chosen per task; the
 * pages define no padding further. Reading taken: q, k and v are zero-padded at
 * the bottom and the right to Hp = S*ceil(H/S), Wp = S*ceil(W/S); region means
 * are taken over the whole padded region (hr*wr tokens, the padding included as
 * zeros); padded tokens take part as keys (k = 0, v = 0, so their score is 0);
 * outputs are produced for the H x W real pixels only (the padding is cropped).
 * LCE(V) of a real pixel is unchanged by the padding, since the padded values
 * are the same zeros as the convolution's own border. When S divides H and W
 * every formula below reduces to the unpadded one.
 *
 * Layouts: q, k, v, out are (N,H,W,C) channels-last float64; lce_w is (C,5,5);
 * lce_b is (C); r_idx is int32 (N,S*S,topk); r_weight is (N,S*S,topk);
 * logits is (N,S*S,S*S). Channel of head m, component c is m*d + c.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define IDX4(n, y, x, c, H, W, C) ((((size_t)(n) * (H) + (y)) * (W) + (x)) * (C) + (c))

int oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int t)
{
#ifdef _OPENMP
    if (t > 0) omp_set_num_threads(t);
#else
    (void)t;
#endif
}

/* 0 if the shape is one BRA defines: C divisible by heads, 1 <= topk <= S*S
 * (H and W need not be multiples of S: see the padding reading above). */
int oracle_check_shape(int N, int H, int W, int C, int heads, int S, int topk)
{
    if (N < 0 || H <= 0 || W <= 0 || C <= 0 || heads <= 0 || S <= 0) return 1;
    if (C % heads != 0) return 1;
    if (topk < 1 || topk > S * S) return 1;
    return 0;
}

/* Region height and width of the (padded) grid: ceil(H/S), ceil(W/S). */
static int region_extent(int H, int S) { return (H + S - 1) / S; }

/* Step 2: per-region mean over the region's hr*wr tokens, every channel; tokens
 * of the zero padding (row >= H or column >= W) add nothing to the sum but count
 * in the divisor. x (N,H,W,C) -> xr (N,S*S,C). */
void oracle_region_mean(const double *x, int N, int H, int W, int C, int S, double *xr)
{
    const int hr = region_extent(H, S), wr = region_extent(W, S);
    for (int n = 0; n < N; ++n)
        for (int j = 0; j < S; ++j)
            for (int i = 0; i < S; ++i) {
                const int p = j * S + i;
                for (int c = 0; c < C; ++c) {
                    double sum = 0.0;
                    for (int h = 0; h < hr; ++h)
                        for (int w = 0; w < wr; ++w) {
                            const int y = j * hr + h, xx = i * wr + w;
                            if (y < H && xx < W) sum += x[IDX4(n, y, xx, c, H, W, C)];
                        }
                    xr[((size_t)n * S * S + p) * C + c] = sum / (double)(hr * wr);
                }
            }
}

typedef struct {
    double value;
    int index;
} scored_t;

/* Order: larger value first; equal values -> lower index first. */
static int cmp_desc(const void *a, const void *b)
{
    const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
    if (x->value > y->value) return -1;
    if (x->value < y->value) return 1;
    return (x->index > y->index) - (x->index < y->index);
}

/* Steps 2-4: region means, affinity logits, top-k indices and their softmax.
 * logits may be NULL. Returns 0, or 1 on a bad shape. */
int oracle_route(const double *q, const double *k, int N, int H, int W, int C, int heads, int S,
                 int topk, int32_t *r_idx, double *r_weight, double *logits)
{
    if (oracle_check_shape(N, H, W, C, heads, S, topk)) return 1;
    const int P = S * S;
    const double scale = 1.0 / sqrt((double)(C / heads));
    double *qr = (double *)malloc(sizeof(double) * (size_t)N * P * C);
    double *kr = (double *)malloc(sizeof(double) * (size_t)N * P * C);
    double *row = (double *)malloc(sizeof(double) * (size_t)P);
    scored_t *order = (scored_t *)malloc(sizeof(scored_t) * (size_t)P);
    oracle_region_mean(q, N, H, W, C, S, qr);
    oracle_region_mean(k, N, H, W, C, S, kr);
    for (int n = 0; n < N; ++n)
        for (int p = 0; p < P; ++p) {
            const double *qp = qr + ((size_t)n * P + p) * C;
            for (int p2 = 0; p2 < P; ++p2) {
                const double *kp = kr + ((size_t)n * P + p2) * C;
                double dot = 0.0;
                for (int c = 0; c < C; ++c) dot += (scale * qp[c]) * kp[c];
                row[p2] = dot;
                if (logits) logits[((size_t)n * P + p) * P + p2] = dot;
            }
            for (int p2 = 0; p2 < P; ++p2) {
                order[p2].value = row[p2];
                order[p2].index = p2;
            }
            qsort(order, (size_t)P, sizeof(scored_t), cmp_desc);
            /* softmax over the selected logits; order[0] holds the maximum */
            double z = 0.0;
            for (int a = 0; a < topk; ++a) z += exp(order[a].value - order[0].value);
            for (int a = 0; a < topk; ++a) {
                const size_t o = ((size_t)n * P + p) * topk + a;
                r_idx[o] = order[a].index;
                r_weight[o] = exp(order[a].value - order[0].value) / z;
            }
        }
    free(order);
    free(row);
    free(kr);
    free(qr);
    return 0;
}

/* Step 6 alone: lepe = bias + depthwise 5x5 cross-correlation of v, zero padded. */
void oracle_lce(const double *v, const double *lce_w, const double *lce_b, int N, int H, int W, int C,
                double *lepe)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int n = 0; n < N; ++n)
        for (int y = 0; y < H; ++y)
            for (int x = 0; x < W; ++x)
                for (int c = 0; c < C; ++c) {
                    double acc = 0.0;
                    for (int a = 0; a < 5; ++a)
                        for (int b = 0; b < 5; ++b) {
                            const int yy = y + a - 2, xx = x + b - 2;
                            if (yy < 0 || yy >= H || xx < 0 || xx >= W) continue;
                            acc += lce_w[(size_t)c * 25 + a * 5 + b] * v[IDX4(n, yy, xx, c, H, W, C)];
                        }
                    lepe[IDX4(n, y, x, c, H, W, C)] = acc + lce_b[c];
                }
}

/* Steps 5-6 for a given routing r_idx (N,S*S,topk): token-to-token attention over
 * the routed regions' tokens, then + LCE(V). out (N,H,W,C). Returns 0, 1 on a bad
 * shape, 2 on an out-of-range region index. */
int oracle_attend(const double *q, const double *k, const double *v, const double *lce_w,
                  const double *lce_b, int N, int H, int W, int C, int heads, int S, int topk,
                  const int32_t *r_idx, double *out)
{
    if (oracle_check_shape(N, H, W, C, heads, S, topk)) return 1;
    const int P = S * S, hr = region_extent(H, S), wr = region_extent(W, S), w2 = hr * wr, d = C / heads;
    const int L = topk * w2; /* keys per query */
    for (size_t e = 0; e < (size_t)N * P * topk; ++e)
        if (r_idx[e] < 0 || r_idx[e] >= P) return 2;
    const double scale = 1.0 / sqrt((double)d);
    double *lepe = (double *)malloc(sizeof(double) * (size_t)N * H * W * C);
    oracle_lce(v, lce_w, lce_b, N, H, W, C, lepe);

#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)L);
        int *ky = (int *)malloc(sizeof(int) * (size_t)L);
        int *kx = (int *)malloc(sizeof(int) * (size_t)L);
#pragma omp for collapse(2) schedule(dynamic)
        for (int n = 0; n < N; ++n)
            for (int p = 0; p < P; ++p) {
                /* gathered key/value tokens: routed regions in r_idx order, tokens
                 * row-major inside each region */
                for (int a = 0; a < topk; ++a) {
                    const int p2 = r_idx[((size_t)n * P + p) * topk + a];
                    const int j2 = p2 / S, i2 = p2 % S;
                    for (int t2 = 0; t2 < w2; ++t2) {
                        ky[a * w2 + t2] = j2 * hr + t2 / wr;
                        kx[a * w2 + t2] = i2 * wr + t2 % wr;
                    }
                }
                const int j = p / S, i = p % S;
                for (int t = 0; t < w2; ++t) {
                    const int y = j * hr + t / wr, x = i * wr + t % wr;
                    if (y >= H || x >= W) continue; /* a padded query: cropped */
                    for (int m = 0; m < heads; ++m) {
                        double smax = -INFINITY;
                        for (int l = 0; l < L; ++l) {
                            /* a padded key has k = 0: its score is 0 */
                            double dot = 0.0;
                            if (ky[l] < H && kx[l] < W)
                                for (int c = 0; c < d; ++c)
                                    dot += (scale * q[IDX4(n, y, x, m * d + c, H, W, C)]) *
                                           k[IDX4(n, ky[l], kx[l], m * d + c, H, W, C)];
                            s[l] = dot;
                            if (dot > smax) smax = dot;
                        }
                        double z = 0.0;
                        for (int l = 0; l < L; ++l) {
                            s[l] = exp(s[l] - smax);
                            z += s[l];
                        }
                        for (int c = 0; c < d; ++c) {
                            double o = 0.0;
                            for (int l = 0; l < L; ++l) /* a padded key has v = 0 */
                                if (ky[l] < H && kx[l] < W)
                                    o += (s[l] / z) * v[IDX4(n, ky[l], kx[l], m * d + c, H, W, C)];
                            const size_t oi = IDX4(n, y, x, m * d + c, H, W, C);
                            out[oi] = o + lepe[oi];
                        }
                    }
                }
            }
        free(kx);
        free(ky);
        free(s);
    }
    free(lepe);
    return 0;
}

/* The whole forward: route, then attend with that routing. */
int oracle_forward(const double *q, const double *k, const double *v, const double *lce_w,
                   const double *lce_b, int N, int H, int W, int C, int heads, int S, int topk,
                   double *out, int32_t *r_idx, double *r_weight)
{
    int rc = oracle_route(q, k, N, H, W, C, heads, S, topk, r_idx, r_weight, NULL);
    if (rc) return rc;
    return oracle_attend(q, k, v, lce_w, lce_b, N, H, W, C, heads, S, topk, r_idx, out);
}
