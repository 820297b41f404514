// route.cuh — steps 1-3 of BRA: region pooling, region affinity and top-k routing.
//
// Follows the BRA walk-through on "BiFormer ... 前向传播过程" (niftyadmin),
// section "BRA模块": q_win/k_win are the means of each region's tokens over all
// channels (eq. 4 prelude), attn_logit = (q_win*scale) @ k_win^T (eq. 4), then
// torch.topk over the last dimension and a softmax of the selected logits (eq. 5).
#pragma once

#include "common.cuh"

namespace bra {

constexpr int kPoolThreads = 256;

// One CTA per (image, region, tensor): blockIdx.x = n*P + p, blockIdx.y = 0 (q) / 1 (k).
// Threads own a 16-byte channel group and stride over the region's tokens; partial
// sums meet in shared memory. Output: float32 means, (N, P, C) each.
template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
region_mean_kernel(const T *__restrict__ q, const T *__restrict__ k, float *__restrict__ q_r,
                   float *__restrict__ k_r, int H, int W, int C, int S) {
    constexpr int V = Elem<T>::kVec;
    __shared__ float red[kPoolThreads * V];  // [slots][C] with slots*C == threads*V
    const int P = S * S;
    const int np = blockIdx.x;
    const int n = np / P, p = np - n * P;
    const int j = p / S, i = p - j * S;
    const int hr = H / S, wr = W / S, w2 = hr * wr;
    const T *x = blockIdx.y ? k : q;
    float *dst = blockIdx.y ? k_r : q_r;

    const int G = C / V;                   // channel groups
    const int slots = kPoolThreads / G;    // token slots
    const int g = threadIdx.x % G, s = threadIdx.x / G;
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    if (s < slots) {
        const size_t img = (size_t)n * H * W;
#pragma unroll 4
        for (int t = s; t < w2; t += slots) {
            const int th = t / wr, tw = t - th * wr;
            const size_t pix = img + (size_t)(j * hr + th) * W + (i * wr + tw);
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(x + pix * C + g * V));
            float f[V];
            unpack16(u, f, x);
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] += f[e];
        }
#pragma unroll
        for (int e = 0; e < V; ++e) red[s * C + g * V + e] = acc[e];
    }
    __syncthreads();
    const float inv_count = 1.0f / (float)w2;
    for (int c = threadIdx.x; c < C; c += kPoolThreads) {
        float sum = 0.f;
        for (int t = 0; t < slots; ++t) sum += red[t * C + c];
        dst[(size_t)np * C + c] = sum * inv_count;
    }
}

// ----------------------------------------------------------------------------- top-k

// Strict total order used by the routing: larger logit first, equal logits ->
// lower region index first.
__device__ inline bool route_before(float av, int ai, float bv, int bi) {
    return av > bv || (av == bv && ai < bi);
}

constexpr int kRouteWarps = 8;
constexpr int kRouteChunk = 64;  // channels of k_r staged in shared memory at a time

// One warp per affinity row (image n, query region p). Lane l holds columns
// l + 32e (e < E), E*32 >= P. The row is sorted with a bitonic network over
// 32*E (value, index) pairs — in registers across e, with shuffles across lanes —
// and the first topk entries are the routing. Shared memory: k_r chunk [P][65].
template <int E>
__global__ void __launch_bounds__(kRouteWarps * 32)
route_kernel(const float *__restrict__ q_r, const float *__restrict__ k_r, int C, int P, int topk,
             float scale, int32_t *__restrict__ r_idx, float *__restrict__ r_weight) {
    extern __shared__ float kr_s[];  // [P][kRouteChunk + 1]
    constexpr int PP = 32 * E;
    const int n = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int p = blockIdx.x * kRouteWarps + warp;
    const bool row_ok = p < P;
    const float *qrow = q_r + ((size_t)n * P + (row_ok ? p : 0)) * C;
    const float *kimg = k_r + (size_t)n * P * C;

    float dot[E];
#pragma unroll
    for (int e = 0; e < E; ++e) dot[e] = 0.f;

    for (int c0 = 0; c0 < C; c0 += kRouteChunk) {
        const int cw = min(kRouteChunk, C - c0);
        __syncthreads();
        for (int idx = threadIdx.x; idx < P * cw; idx += blockDim.x) {
            const int r = idx / cw, c = idx - r * cw;
            kr_s[r * (kRouteChunk + 1) + c] = kimg[(size_t)r * C + c0 + c];
        }
        __syncthreads();
        for (int c = 0; c < cw; ++c) {
            const float qv = scale * __ldg(qrow + c0 + c);
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int col = lane + 32 * e;
                if (col < P) dot[e] = fmaf(qv, kr_s[col * (kRouteChunk + 1) + c], dot[e]);
            }
        }
    }
    if (!row_ok) return;

    float val[E];
    int id[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int col = lane + 32 * e;
        val[e] = col < P ? dot[e] : -INFINITY;
        id[e] = col;  // padding columns (col >= P) carry unique indices >= P and sort last
    }

    // Bitonic sort of the PP pairs into route_before order; element index = e*32 + lane.
#pragma unroll
    for (int kk = 2; kk <= PP; kk <<= 1) {
#pragma unroll
        for (int jj = kk >> 1; jj > 0; jj >>= 1) {
            if (jj >= 32) {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int e2 = e ^ (jj >> 5);
                    if (e2 > e) {
                        const bool up = ((e * 32 + lane) & kk) == 0;
                        const bool sw = up ? route_before(val[e2], id[e2], val[e], id[e])
                                           : route_before(val[e], id[e], val[e2], id[e2]);
                        if (sw) {
                            const float tv = val[e];
                            val[e] = val[e2];
                            val[e2] = tv;
                            const int ti = id[e];
                            id[e] = id[e2];
                            id[e2] = ti;
                        }
                    }
                }
            } else {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float pv = __shfl_xor_sync(0xffffffffu, val[e], jj);
                    const int pi = __shfl_xor_sync(0xffffffffu, id[e], jj);
                    const bool up = ((e * 32 + lane) & kk) == 0;
                    const bool lower = (lane & jj) == 0;
                    const bool mine_first = route_before(val[e], id[e], pv, pi);
                    const bool keep = (up == lower) ? mine_first : !mine_first;
                    if (!keep) {
                        val[e] = pv;
                        id[e] = pi;
                    }
                }
            }
        }
    }

    // softmax over the first topk sorted logits; position 0 holds the maximum
    const float vmax = __shfl_sync(0xffffffffu, val[0], 0);
    float z = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (e * 32 + lane < topk) z += expf(val[e] - vmax);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    const float inv_z = 1.0f / z;
    const size_t base = ((size_t)n * P + p) * topk;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int pos = e * 32 + lane;
        if (pos < topk) {
            r_idx[base + pos] = id[e];
            r_weight[base + pos] = expf(val[e] - vmax) * inv_z;
        }
    }
}

}  // namespace bra
