// backward.cuh — the BRA backward pass with the routing detached: gradients of q, k, v and
// of the LCE weight and bias, given dL/dout and the forward's routing r_idx.
//
// Source: the walk-through's router ("BiFormer ... 前向传播过程", niftyadmin, section
// "BRA模块", `TopkRouting`) detaches the region-level query and key when `diff_routing` is
// off (its default); the top-k index is a discrete choice and r_weight does not scale K or
// V, so gradients flow only through the token-to-token attention and the LCE:
//   per image n, query region p, head m, query token t (keys j: the tokens of the routed
//   regions r_idx[n][p][0..topk-1], each region's tokens row-major):
//     s_j = scale q_t . k_j,  a_j = softmax_j(s_j),  o_t = sum_j a_j v_j
//     ds_j = a_j (dO_t . v_j - dO_t . o_t)
//     dq_t = scale sum_j ds_j k_j,  dk_j += scale ds_j q_t,  dv_j += a_j dO_t
//   LCE (out += b + depthwise 5x5 cross-correlation of V, zero pad 2):
//     dv[y,x,c] += sum_{a,b} w[c,a,b] dout[y-a+2, x-b+2, c]
//     dw[c,a,b]  = sum_{n,y,x} dout[n,y,x,c] V[n, y+a-2, x+b-2, c],   db[c] = sum dout[..c]
//
// Work split (plain SIMT, float32 arithmetic):
//   bwd_lce_dv_kernel:    one thread per element of dv: the LCE term (initialises dv);
//   bwd_attn_kernel:      one thread per (image, region, head, query token): two passes over
//                         the gathered keys (softmax statistics and o_t, then the gradients);
//                         dq stored, dk and dv accumulated with float32 atomics;
//   bwd_lce_param_kernel: one CTA per (channel, tap) (25 weight taps and the bias): a
//                         reduction over every pixel of every image.
// The per-item arithmetic is in __host__ __device__ functions so that the same code can
// run on the host, with every memory access bounds-checked (BRA_BWD_HOST_CHECK).
#pragma once

#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

namespace bra {

struct BwdParams {
    const void *q, *k, *v, *dout;  // (N,H,W,C), bf16 or float32
    const void *lce_w;             // (C,5,5), same type
    const int32_t *r_idx;          // (N,S*S,topk)
    float *dq, *dk, *dv;           // (N,H,W,C) float32
    float *dw, *db;                // (C,5,5), (C) float32
    int *bad_index;                // set to 1 when a routed region index is out of range
    int N, H, W, C, heads, S, topk, P, hr, wr, w2, d, bf16;
    float scale;
};

#if defined(BRA_BWD_HOST_CHECK) && !defined(__CUDA_ARCH__)  // the host pass of a host-check build
void bra_bwd_host_bounds_failure(const char *what, long long i, long long n);
#define BRA_BWD_CHECK(what, i, n) \
    do { if ((long long)(i) < 0 || (long long)(i) >= (long long)(n)) bra_bwd_host_bounds_failure(what, (i), (n)); } while (0)
#else
#define BRA_BWD_CHECK(what, i, n) do { } while (0)
#endif

__host__ __device__ inline size_t bwd_elems(const BwdParams &p) { return (size_t)p.N * p.H * p.W * p.C; }

// element i of an input map or weight (bf16 or float32) as float32
__host__ __device__ inline float bwd_ld(const void *base, size_t i, int bf16) {
    if (bf16) return __bfloat162float(static_cast<const __nv_bfloat16 *>(base)[i]);
    return static_cast<const float *>(base)[i];
}
__host__ __device__ inline float bwd_map(const BwdParams &p, const void *base, size_t i) {
    BRA_BWD_CHECK("map", i, bwd_elems(p));
    return bwd_ld(base, i, p.bf16);
}

__host__ __device__ inline void bwd_add(float *dst, size_t i, size_t n, float v) {
    BRA_BWD_CHECK("accumulate", i, n);
#ifdef __CUDA_ARCH__
    atomicAdd(dst + i, v);
#else
    dst[i] += v;
#endif
}

// flat pixel index (y * W + x) of token t of region r
__host__ __device__ inline int bwd_pixel(const BwdParams &p, int r, int t) {
    const int y = (r / p.S) * p.hr + t / p.wr, x = (r % p.S) * p.wr + t % p.wr;
    return y * p.W + x;
}

// Routed region a of query region pr of image n, or -1 (and the error flag) when the
// stored index is out of range.
__host__ __device__ inline int bwd_route(const BwdParams &p, int n, int pr, int a) {
    const size_t i = ((size_t)n * p.P + pr) * p.topk + a;
    BRA_BWD_CHECK("r_idx", i, (size_t)p.N * p.P * p.topk);
    const int r = p.r_idx[i];
    if (r < 0 || r >= p.P) {
        if (p.bad_index) *p.bad_index = 1;
        return -1;
    }
    return r;
}

constexpr int kBwdMaxD = 64;  // channels per head (32 or 64)

// Gradients of one (image n, query region pr, head m, query token t).
__host__ __device__ inline void bwd_query(const BwdParams &p, int n, int pr, int m, int t) {
    const int d = p.d, c0 = m * d;
    const size_t img = (size_t)n * p.H * p.W;
    const size_t qi = (img + bwd_pixel(p, pr, t)) * p.C + c0;
    float qv[kBwdMaxD], go[kBwdMaxD], o[kBwdMaxD];
    for (int c = 0; c < d; ++c) {
        qv[c] = bwd_map(p, p.q, qi + c);
        go[c] = bwd_map(p, p.dout, qi + c);
        o[c] = 0.f;
    }
    // pass 1: running max, denominator and o_t over the gathered keys
    float mx = -INFINITY, l = 0.f;
    for (int a = 0; a < p.topk; ++a) {
        const int r = bwd_route(p, n, pr, a);
        if (r < 0) continue;
        for (int tk = 0; tk < p.w2; ++tk) {
            const size_t ki = (img + bwd_pixel(p, r, tk)) * p.C + c0;
            float s = 0.f;
            for (int c = 0; c < d; ++c) s += qv[c] * bwd_map(p, p.k, ki + c);
            s *= p.scale;
            const float mn = fmaxf(mx, s);
            const float f = expf(mx - mn), e = expf(s - mn);  // mx = -inf at the first key: f = 0
            l = l * f + e;
            for (int c = 0; c < d; ++c) o[c] = o[c] * f + e * bwd_map(p, p.v, ki + c);
            mx = mn;
        }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float god = 0.f;  // dO_t . o_t
    for (int c = 0; c < d; ++c) god += go[c] * o[c] * inv;
    // pass 2: the gradients
    float dqa[kBwdMaxD];
    for (int c = 0; c < d; ++c) dqa[c] = 0.f;
    const size_t n_el = bwd_elems(p);
    for (int a = 0; a < p.topk; ++a) {
        const int r = bwd_route(p, n, pr, a);
        if (r < 0) continue;
        for (int tk = 0; tk < p.w2; ++tk) {
            const size_t ki = (img + bwd_pixel(p, r, tk)) * p.C + c0;
            float s = 0.f, da = 0.f;
            for (int c = 0; c < d; ++c) {
                s += qv[c] * bwd_map(p, p.k, ki + c);
                da += go[c] * bwd_map(p, p.v, ki + c);
            }
            const float aj = expf(s * p.scale - mx) * inv;
            const float ds = aj * (da - god);
            for (int c = 0; c < d; ++c) {
                dqa[c] += ds * bwd_map(p, p.k, ki + c);
                bwd_add(p.dk, ki + c, n_el, p.scale * ds * qv[c]);
                bwd_add(p.dv, ki + c, n_el, aj * go[c]);
            }
        }
    }
    for (int c = 0; c < d; ++c) {
        BRA_BWD_CHECK("dq", qi + c, n_el);
        p.dq[qi + c] = p.scale * dqa[c];
    }
}

// LCE term of dv at element i = ((n * H + y) * W + x) * C + c (the full value: stored).
__host__ __device__ inline float bwd_lce_dv(const BwdParams &p, size_t i) {
    const int c = (int)(i % p.C);
    const size_t pix = i / p.C;
    const int x = (int)(pix % p.W), y = (int)((pix / p.W) % p.H);
    const size_t n = pix / ((size_t)p.W * p.H);
    float acc = 0.f;
    for (int a = 0; a < 5; ++a) {
        const int yy = y - a + 2;
        if (yy < 0 || yy >= p.H) continue;
        for (int b = 0; b < 5; ++b) {
            const int xx = x - b + 2;
            if (xx < 0 || xx >= p.W) continue;
            const size_t wi = (size_t)c * 25 + a * 5 + b;
            BRA_BWD_CHECK("lce_w", wi, (size_t)p.C * 25);
            acc += bwd_ld(p.lce_w, wi, p.bf16) * bwd_map(p, p.dout, ((n * p.H + yy) * p.W + xx) * p.C + c);
        }
    }
    return acc;
}

// Partial sum, over pixels start, start + stride, ... of all images, of the LCE parameter
// gradient `tap` of channel c: tap < 25 is weight (tap / 5, tap % 5), tap 25 the bias.
__host__ __device__ inline float bwd_lce_param_partial(const BwdParams &p, int c, int tap, size_t start,
                                                       size_t stride) {
    const size_t npix = (size_t)p.N * p.H * p.W;
    const int a = tap / 5, b = tap % 5;
    float acc = 0.f;
    for (size_t pix = start; pix < npix; pix += stride) {
        const float g = bwd_map(p, p.dout, pix * p.C + c);
        if (tap == 25) {
            acc += g;
            continue;
        }
        const int x = (int)(pix % p.W), y = (int)((pix / p.W) % p.H);
        const int yy = y + a - 2, xx = x + b - 2;
        if (yy < 0 || yy >= p.H || xx < 0 || xx >= p.W) continue;
        const size_t src = (pix + (size_t)(yy - y) * p.W + (xx - x)) * p.C + c;
        acc += g * bwd_map(p, p.v, src);
    }
    return acc;
}

// Parameters of one backward call (shapes already checked: H % S == W % S == 0,
// C % heads == 0, C / heads in {32, 64}).
__host__ inline BwdParams make_bwd_params(const void *q, const void *k, const void *v, const void *dout,
                                          const void *lce_w, const int32_t *r_idx, int N, int H, int W, int C,
                                          int heads, int S, int topk, bool bf16, float *dq, float *dk, float *dv,
                                          float *dw, float *db, int *bad_index) {
    BwdParams p;
    p.q = q;
    p.k = k;
    p.v = v;
    p.dout = dout;
    p.lce_w = lce_w;
    p.r_idx = r_idx;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.dw = dw;
    p.db = db;
    p.bad_index = bad_index;
    p.N = N;
    p.H = H;
    p.W = W;
    p.C = C;
    p.heads = heads;
    p.S = S;
    p.topk = topk;
    p.P = S * S;
    p.hr = H / S;
    p.wr = W / S;
    p.w2 = p.hr * p.wr;
    p.d = C / heads;
    p.bf16 = bf16 ? 1 : 0;
    p.scale = (float)(1.0 / sqrt((double)p.d));
    return p;
}

// Work items of the attention part: (image, region, head, query token).
__host__ __device__ inline size_t bwd_attn_items(const BwdParams &p) { return (size_t)p.N * p.P * p.heads * p.w2; }

__host__ __device__ inline void bwd_attn_item(const BwdParams &p, size_t i) {
    const int t = (int)(i % p.w2);
    const size_t r1 = i / p.w2;
    const int m = (int)(r1 % p.heads);
    const size_t r2 = r1 / p.heads;
    bwd_query(p, (int)(r2 / p.P), (int)(r2 % p.P), m, t);
}

// ----------------------------------------------------------------------------- kernels

__global__ void __launch_bounds__(256) bwd_lce_dv_kernel(const BwdParams p) {
    const size_t n = bwd_elems(p);
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        p.dv[i] = bwd_lce_dv(p, i);
}

__global__ void __launch_bounds__(128) bwd_attn_kernel(const BwdParams p) {
    const size_t items = bwd_attn_items(p);
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < items; i += (size_t)gridDim.x * blockDim.x)
        bwd_attn_item(p, i);
}

// grid: C * 26 CTAs of 256 threads, CTA = (channel, tap)
__global__ void __launch_bounds__(256) bwd_lce_param_kernel(const BwdParams p) {
    __shared__ float red[256];
    const int c = blockIdx.x / 26, tap = blockIdx.x % 26;
    red[threadIdx.x] = bwd_lce_param_partial(p, c, tap, threadIdx.x, blockDim.x);
    __syncthreads();
    for (int s = 128; s > 0; s >>= 1) {
        if ((int)threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        if (tap == 25)
            p.db[c] = red[0];
        else
            p.dw[c * 25 + tap] = red[0];
    }
}

}  // namespace bra
