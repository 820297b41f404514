// block.cuh — the BiFormer block's per-pixel steps around the attention layer and the MLP
// GEMMs: the positional embedding with its residual, and the two pre-norm LayerNorms.
//
// Source: "BiFormer ... 前向传播过程" (niftyadmin), section "2、BiFormer Block" (the block's
// forward: x = x + pos_embed(x), then x = x + drop_path(attn(norm1(x)))) and the module
// printout of section "网络结构": pos_embed = Conv2d(C, C, 3, padding 1, groups C) (with its
// bias), norm1 / norm2 = LayerNorm(C, eps 1e-6), mlp = Linear(C, 3C) -> GELU ->
// Linear(3C, C), drop_path = Identity. The MLP line is read as the same pre-norm residual
// form, x = x + mlp(norm2(x)).
//
//   pos_ln_tile_kernel:  x1 = x + b + dwconv3x3(x)  (zero pad 1)  -> stored;  h = LN1(x1) -> stored
//   add_ln_kernel:       x2 = x1 + a                               -> stored;  h = LN2(x2) -> stored
//
// LayerNorm: (x - mean) / sqrt(var + 1e-6) * gamma + beta over the C channels of a pixel,
// var the mean squared deviation (two passes over registers). Arithmetic in float32; every
// stored value is rounded once to the storage type, and each LayerNorm reads the rounded
// value that was stored (as a bf16 model stores its activations).
//
// A warp works on one pixel at a time: lane l owns channel pairs l, l + 32, ... (NP of
// them, C <= 64 * NP); loads and stores are whole pairs (bf16x2 or float2), so a warp
// moves one pixel's channels contiguously.
#pragma once

#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"

namespace bra {

constexpr int kBlockThreads = 256;
constexpr int kAddUnroll = 4;  // add_ln: pixels per warp and iteration

struct BlockParams {
    const void *x;       // pos_ln: the block input; add_ln: x1
    const void *a;       // add_ln: the attention layer's output
    const void *pos_w;   // (C, 3, 3)
    const void *pos_b;   // (C)
    const void *ln_g;    // (C)
    const void *ln_b;    // (C)
    void *xo;            // x1 (pos_ln) or x2 (add_ln)
    void *h;             // the LayerNorm output
    long long pixels;    // N * H * W
    int H, W, C;
};

template <typename T> struct PairIO;
template <> struct PairIO<__nv_bfloat16> {
    static __device__ __forceinline__ float2 ld(const void *p, size_t pair) {
        const uint32_t u = __ldg(static_cast<const unsigned int *>(p) + pair);
        return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
    }
    static __device__ __forceinline__ float2 round(float2 v) {
        return make_float2(__bfloat162float(__float2bfloat16_rn(v.x)), __bfloat162float(__float2bfloat16_rn(v.y)));
    }
    static __device__ __forceinline__ void st(void *p, size_t pair, float2 v) {  // v already representable
        const __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
        static_cast<__nv_bfloat162 *>(p)[pair] = h;
    }
    static __device__ __forceinline__ float2 lds(const void *p, int pair) {
        const uint32_t u = static_cast<const uint32_t *>(p)[pair];
        return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
    }
};
template <> struct PairIO<float> {
    static __device__ __forceinline__ float2 ld(const void *p, size_t pair) {
        return __ldg(static_cast<const float2 *>(p) + pair);
    }
    static __device__ __forceinline__ float2 round(float2 v) { return v; }
    static __device__ __forceinline__ void st(void *p, size_t pair, float2 v) { static_cast<float2 *>(p)[pair] = v; }
    static __device__ __forceinline__ float2 lds(const void *p, int pair) { return static_cast<const float2 *>(p)[pair]; }
};

// 16 bytes as floats and back (rounded to the type).
template <typename T> __device__ __forceinline__ void vec_unpack(uint4 u, float (&f)[16 / sizeof(T)]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) f[i] = __uint_as_float(w[i]);
    }
}
template <typename T> __device__ __forceinline__ uint4 vec_pack(const float (&f)[16 / sizeof(T)]) {
    uint32_t w[4];
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t *>(&h);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = __float_as_uint(f[i]);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// One parameter element (weights and per-channel vectors need only element alignment).
template <typename T> __device__ __forceinline__ float ld_elem(const void *p, int i) {
    if constexpr (sizeof(T) == 2)
        return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
    else
        return static_cast<const float *>(p)[i];
}
template <typename T> __device__ __forceinline__ float2 ld_pair_elems(const void *p, int cp) {
    return make_float2(ld_elem<T>(p, 2 * cp), ld_elem<T>(p, 2 * cp + 1));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// LayerNorm of one pixel whose channel pairs v[j] (pair lane + 32 j, valid while < C/2)
// sit in the warp's registers; writes the rounded result.
template <typename T, int NP>
__device__ __forceinline__ void ln_store(const float2 (&v)[NP], const float2 (&g)[NP], const float2 (&b)[NP],
                                         int lane, int pairs, int C, void *out, size_t pix_pair0) {
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < NP; ++j)
        if (lane + 32 * j < pairs) s += v[j].x + v[j].y;
    const float mean = warp_sum(s) / (float)C;
    float q = 0.f;
#pragma unroll
    for (int j = 0; j < NP; ++j)
        if (lane + 32 * j < pairs) {
            const float dx = v[j].x - mean, dy = v[j].y - mean;
            q = fmaf(dx, dx, fmaf(dy, dy, q));
        }
    const float rstd = rsqrtf(warp_sum(q) / (float)C + 1e-6f);
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        const int cp = lane + 32 * j;
        if (cp < pairs) {
            const float2 o = make_float2(fmaf((v[j].x - mean) * rstd, g[j].x, b[j].x),
                                         fmaf((v[j].y - mean) * rstd, g[j].y, b[j].y));
            PairIO<T>::st(out, pix_pair0 + cp, PairIO<T>::round(o));
        }
    }
}

// pos_ln_tile_kernel: one CTA per (image, tile of kPosTH x kPosTW output pixels).
// The tile's pixels with a one-pixel border, (kPosTH + 2) x (kPosTW + 2) pixels of C
// channels, are copied into shared memory once (16-byte cp.async pieces, zero outside
// the image), so the nine taps of every pixel read shared memory (a tap on the border
// adds w * 0: the convolution's zero padding); then each warp takes the tile's pixels
// w, w + 8, ...: lane l owns channel pairs l, l + 32, ... (NP of them), whose weights it
// keeps in registers.
constexpr int kPosTH = 4, kPosTW = 32;

__host__ __device__ inline int pos_tile_smem_bytes(int C, int es) { return (kPosTH + 2) * (kPosTW + 2) * C * es; }

template <typename T, int NP>
__global__ void __launch_bounds__(kBlockThreads) pos_ln_tile_kernel(const BlockParams p, int tiles_x, int tiles_y) {
    extern __shared__ __align__(16) unsigned char pos_s[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int pairs = p.C >> 1;
    int b = blockIdx.x;
    const int tx = b % tiles_x;
    b /= tiles_x;
    const int ty = b % tiles_y, n = b / tiles_y;
    const int y0 = ty * kPosTH, x0 = tx * kPosTW;
    constexpr int sp = kPosTW + 2;  // staged pixels per row
    const int pix_bytes = p.C * (int)sizeof(T), chunks = pix_bytes >> 4;
    const int total = (kPosTH + 2) * sp * chunks;
    const unsigned char *xb = static_cast<const unsigned char *>(p.x);
    for (int e = threadIdx.x; e < total; e += kBlockThreads) {
        const int pix = e / chunks, ch = e - pix * chunks;
        const int ly = pix / sp, lx = pix - ly * sp;
        const int gy = y0 - 1 + ly, gx = x0 - 1 + lx;
        const bool ok = gy >= 0 && gy < p.H && gx >= 0 && gx < p.W;
        const size_t gpix = ((size_t)n * p.H + (ok ? gy : 0)) * p.W + (ok ? gx : 0);
        cp_async16(pos_s + (size_t)e * 16, xb + gpix * pix_bytes + ch * 16, ok);
    }
    cp_async_commit();
    float2 w[NP][9], bias[NP], g[NP], bb[NP];  // loaded while the copies are in flight
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        const int cp = lane + 32 * j;
        const bool ok = cp < pairs;
        const int c = 2 * cp;
#pragma unroll
        for (int t = 0; t < 9; ++t)
            w[j][t] = ok ? make_float2(ld_elem<T>(p.pos_w, c * 9 + t), ld_elem<T>(p.pos_w, (c + 1) * 9 + t))
                         : make_float2(0.f, 0.f);
        bias[j] = ok ? ld_pair_elems<T>(p.pos_b, cp) : make_float2(0.f, 0.f);
        g[j] = ok ? ld_pair_elems<T>(p.ln_g, cp) : make_float2(0.f, 0.f);
        bb[j] = ok ? ld_pair_elems<T>(p.ln_b, cp) : make_float2(0.f, 0.f);
    }
    cp_async_wait<0>();
    __syncthreads();
    // the staged border is zero outside the image, so every tap is taken: a tap on the
    // border adds w * 0 (the convolution's zero padding)
    const int rowstep = sp * pairs;
    for (int t = warp; t < kPosTH * kPosTW; t += kBlockThreads / 32) {
        const int py = t / kPosTW, px = t - py * kPosTW;
        if (y0 + py >= p.H || x0 + px >= p.W) continue;  // the same for the whole warp
        const int c0 = (py * sp + px) * pairs + lane;     // pair `lane` of the tap at (-1, -1)
        float2 acc[NP];
#pragma unroll
        for (int j = 0; j < NP; ++j) acc[j] = bias[j];
#pragma unroll
        for (int a = 0; a < 3; ++a)
#pragma unroll
            for (int e = 0; e < 3; ++e) {
                const int q0 = c0 + a * rowstep + e * pairs;
#pragma unroll
                for (int j = 0; j < NP; ++j)
                    if (lane + 32 * j < pairs) {
                        const float2 v = PairIO<T>::lds(pos_s, q0 + 32 * j);
                        acc[j].x = fmaf(w[j][3 * a + e].x, v.x, acc[j].x);
                        acc[j].y = fmaf(w[j][3 * a + e].y, v.y, acc[j].y);
                        if (a == 1 && e == 1) {  // the residual: x itself
                            acc[j].x += v.x;
                            acc[j].y += v.y;
                        }
                    }
            }
        const size_t o0 = (((size_t)n * p.H + y0 + py) * p.W + x0 + px) * pairs;
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            acc[j] = PairIO<T>::round(acc[j]);
            if (lane + 32 * j < pairs) PairIO<T>::st(p.xo, o0 + lane + 32 * j, acc[j]);
        }
        ln_store<T, NP>(acc, g, bb, lane, pairs, p.C, p.h, o0);
    }
}

template <typename T, int NP>
__global__ void __launch_bounds__(kBlockThreads) add_ln_kernel(const BlockParams p) {
    const int lane = threadIdx.x & 31;
    const int pairs = p.C >> 1;
    float2 g[NP], bb[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
        const int cp = lane + 32 * j;
        g[j] = cp < pairs ? ld_pair_elems<T>(p.ln_g, cp) : make_float2(0.f, 0.f);
        bb[j] = cp < pairs ? ld_pair_elems<T>(p.ln_b, cp) : make_float2(0.f, 0.f);
    }
    // kAddUnroll pixels per warp and iteration: all their loads are in flight together
    const long long warps = (long long)gridDim.x * (kBlockThreads / 32);
    for (long long pix0 = (long long)blockIdx.x * (kBlockThreads / 32) + (threadIdx.x >> 5); pix0 < p.pixels;
         pix0 += warps * kAddUnroll) {
        float2 x1[kAddUnroll][NP], a[kAddUnroll][NP];
#pragma unroll
        for (int u = 0; u < kAddUnroll; ++u) {
            const long long pix = pix0 + u * warps;
            const size_t q0 = (size_t)pix * pairs;
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                const int cp = lane + 32 * j;
                x1[u][j] = a[u][j] = make_float2(0.f, 0.f);
                if (pix < p.pixels && cp < pairs) {
                    x1[u][j] = PairIO<T>::ld(p.x, q0 + cp);
                    a[u][j] = PairIO<T>::ld(p.a, q0 + cp);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kAddUnroll; ++u) {
            const long long pix = pix0 + u * warps;
            if (pix >= p.pixels) break;  // the same for the whole warp
            const size_t q0 = (size_t)pix * pairs;
            float2 v[NP];
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                const int cp = lane + 32 * j;
                v[j] = PairIO<T>::round(make_float2(x1[u][j].x + a[u][j].x, x1[u][j].y + a[u][j].y));
                if (cp < pairs) PairIO<T>::st(p.xo, q0 + cp, v[j]);
            }
            ln_store<T, NP>(v, g, bb, lane, pairs, p.C, p.h, q0);
        }
    }
}

// add_ln with 16-byte accesses, for a pixel of C channels that is a power-of-two number
// LPP <= 32 of 16-byte chunks: lane l holds chunk l mod LPP of pixel l / LPP of the
// warp's current group of 32 / LPP pixels, and the group's LayerNorm sums run over the
// LPP lanes of each pixel (xor shuffles that stay inside the pixel's lanes). kAddUnroll
// groups per warp and iteration have their loads in flight together. Same arithmetic as
// add_ln_kernel; the sums meet in another order.
template <typename T, int LPP>
__global__ void __launch_bounds__(kBlockThreads) add_ln_vec_kernel(const BlockParams p) {
    constexpr int VE = 16 / (int)sizeof(T);  // elements per chunk
    constexpr int PPW = 32 / LPP;            // pixels per warp and group
    const int lane = threadIdx.x & 31;
    const int sub = lane / LPP, ch = lane % LPP;
    float g[VE], bb[VE];
#pragma unroll
    for (int e = 0; e < VE; ++e) {
        g[e] = ld_elem<T>(p.ln_g, ch * VE + e);
        bb[e] = ld_elem<T>(p.ln_b, ch * VE + e);
    }
    const uint4 *x1p = static_cast<const uint4 *>(p.x);
    const uint4 *ap = static_cast<const uint4 *>(p.a);
    uint4 *x2p = static_cast<uint4 *>(p.xo);
    uint4 *hp = static_cast<uint4 *>(p.h);
    const long long warps = (long long)gridDim.x * (kBlockThreads / 32);
    const long long step = warps * PPW * kAddUnroll;
    for (long long pix0 = ((long long)blockIdx.x * (kBlockThreads / 32) + (threadIdx.x >> 5)) * PPW * kAddUnroll;
         pix0 < p.pixels; pix0 += step) {
        uint4 xv[kAddUnroll], av[kAddUnroll];
#pragma unroll
        for (int u = 0; u < kAddUnroll; ++u) {
            const long long pix = pix0 + u * PPW + sub;
            xv[u] = av[u] = make_uint4(0u, 0u, 0u, 0u);
            if (pix < p.pixels) {
                xv[u] = __ldg(x1p + pix * LPP + ch);
                av[u] = __ldg(ap + pix * LPP + ch);
            }
        }
#pragma unroll
        for (int u = 0; u < kAddUnroll; ++u) {
            const long long pix = pix0 + u * PPW + sub;
            float v[VE], xa[VE], aa[VE];
            vec_unpack<T>(xv[u], xa);
            vec_unpack<T>(av[u], aa);
            float s1 = 0.f;
#pragma unroll
            for (int e = 0; e < VE; ++e) {
                v[e] = PairIO<T>::round(make_float2(xa[e] + aa[e], 0.f)).x;
                s1 += v[e];
            }
#pragma unroll
            for (int o = LPP / 2; o > 0; o >>= 1) s1 += __shfl_xor_sync(0xffffffffu, s1, o);
            const float mean = s1 / (float)p.C;
            float s2 = 0.f;
#pragma unroll
            for (int e = 0; e < VE; ++e) {
                const float d = v[e] - mean;
                s2 = fmaf(d, d, s2);
            }
#pragma unroll
            for (int o = LPP / 2; o > 0; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
            const float rstd = rsqrtf(s2 / (float)p.C + 1e-6f);
            float hv[VE];
#pragma unroll
            for (int e = 0; e < VE; ++e) hv[e] = fmaf((v[e] - mean) * rstd, g[e], bb[e]);
            if (pix < p.pixels) {
                x2p[pix * LPP + ch] = vec_pack<T>(v);
                hp[pix * LPP + ch] = vec_pack<T>(hv);
            }
        }
    }
}

}  // namespace bra
