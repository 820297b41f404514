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

// One thread per (tensor, image, region, 16-byte channel group, token slot): it sums
// the region's tokens whose column is congruent to its slot modulo `ns`, issuing its
// 16-byte loads eight at a time so that many are in flight; the ns slots of a unit
// are adjacent lanes G apart and meet by shuffles. ns divides wr and G*ns divides 32
// (or ns = 1). Output: float32 means, (N, P, C) for q and for k.
template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
region_mean_kernel(const T *__restrict__ q, const T *__restrict__ k, float *__restrict__ q_r,
                   float *__restrict__ k_r, int N, int H, int W, int C, int S, int ns_log2,
                   long long total) {
    constexpr int V = Elem<T>::kVec;
    const long long t = (long long)blockIdx.x * kPoolThreads + threadIdx.x;
    const bool valid = t < total;
    const int G = C / V, ns = 1 << ns_log2, P = S * S;
    const long long tt = valid ? t : 0;
    const int g = (int)(tt % G);
    const long long rest = tt / G;
    const int s = (int)(rest & (ns - 1));
    const long long u = rest >> ns_log2;
    const long long NP = (long long)N * P;
    const int tensor = (int)(u / NP);
    const long long np = u - tensor * NP;
    const int n = (int)(np / P), p = (int)(np - (long long)n * P);
    const int j = p / S, i = p - j * S;
    const int hr = H / S, wr = W / S;
    const T *x = tensor ? k : q;
    const T *origin = x + (((size_t)n * H + j * hr) * W + i * wr) * C + g * V;
    const int count = valid ? hr * (wr >> ns_log2) : 0;

    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    int th = 0, tw = s;
    for (int it = 0; it < count; it += 8) {
        uint4 buf[8];
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            buf[b] = make_uint4(0u, 0u, 0u, 0u);
            if (it + b < count) {
                buf[b] = __ldg(reinterpret_cast<const uint4 *>(origin + ((size_t)th * W + tw) * C));
                tw += ns;
                if (tw >= wr) {
                    tw = s;
                    ++th;
                }
            }
        }
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            float f[V];
            unpack16(buf[b], f, x);
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] += f[e];
        }
    }
    for (int off = G; off < (G << ns_log2); off <<= 1)
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    if (valid && s == 0) {
        float *dst = (tensor ? k_r : q_r) + (size_t)np * C + g * V;
        const float w2 = (float)(hr * wr);
#pragma unroll
        for (int e = 0; e < V; e += 4)
            *reinterpret_cast<float4 *>(dst + e) = make_float4(acc[e] / w2, acc[e + 1] / w2, acc[e + 2] / w2, acc[e + 3] / w2);
    }
}

// ----------------------------------------------------------------------------- top-k

// Strict total order used by the routing: larger logit first, equal logits ->
// lower region index first.
__device__ inline bool route_before(float av, int ai, float bv, int bi) {
    return av > bv || (av == bv && ai < bi);
}

constexpr int kRouteWarps = 8;

// Channels of k_r staged in shared memory per pass, for P regions: the largest
// multiple of 32 (at most C) whose [P][cc+1] tile plus 8 query rows fit in 96 KB.
inline int route_chunk(int P, int C) {
    int cc = C;
    while (cc > 32 && (P * (cc + 1) + 4 + kRouteWarps * cc) * 4 > 96 * 1024) cc -= 32;
    return cc;
}
inline int route_qoff(int P, int cc) { return (P * (cc + 1) + 3) & ~3; }  // 16-byte aligned query rows
inline int route_smem_bytes(int P, int cc) { return (route_qoff(P, cc) + kRouteWarps * cc) * 4; }

// One warp per affinity row (image n, query region p). Lane l holds columns
// l + 32e (e < E), E*32 >= P. The row is sorted with a bitonic network over
// 32*E (value, index) pairs — in registers across e, with shuffles across lanes —
// and the first topk entries are the routing. Shared memory: k_r chunk [P][cc+1]
// (odd pitch: conflict-free column reads) and the CTA's 8 query rows [8][cc].
template <int E>
__global__ void __launch_bounds__(kRouteWarps * 32)
route_kernel(const float *__restrict__ q_r, const float *__restrict__ k_r, int C, int P, int topk, int cc,
             float scale, int32_t *__restrict__ r_idx, float *__restrict__ r_weight) {
    extern __shared__ float kr_s[];
    float *q_s = kr_s + ((P * (cc + 1) + 3) & ~3);
    constexpr int PP = 32 * E;
    griddep_wait();               // pooled means come from the preceding kernel
    griddep_launch_dependents();  // the attention kernel may start its prologue
    const int n = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int p0 = blockIdx.x * kRouteWarps;
    const int p = p0 + warp;
    const bool row_ok = p < P;
    const float *kimg = k_r + (size_t)n * P * C;
    const float *qimg = q_r + (size_t)n * P * C;

    float dot[E];
#pragma unroll
    for (int e = 0; e < E; ++e) dot[e] = 0.f;

    for (int c0 = 0; c0 < C; c0 += cc) {
        const int cw = min(cc, C - c0);  // multiple of 4
        const int q4 = cw >> 2;
        __syncthreads();
        for (int idx = threadIdx.x; idx < P * q4; idx += blockDim.x) {
            const int r = idx / q4, c = (idx - r * q4) * 4;
            const float4 v = __ldg(reinterpret_cast<const float4 *>(kimg + (size_t)r * C + c0 + c));
            float *d = kr_s + r * (cc + 1) + c;
            d[0] = v.x;
            d[1] = v.y;
            d[2] = v.z;
            d[3] = v.w;
        }
        for (int idx = threadIdx.x; idx < kRouteWarps * q4; idx += blockDim.x) {
            const int r = idx / q4, c = (idx - r * q4) * 4;
            const int pr = min(p0 + r, P - 1);
            *reinterpret_cast<float4 *>(q_s + r * cc + c) =
                __ldg(reinterpret_cast<const float4 *>(qimg + (size_t)pr * C + c0 + c));
        }
        __syncthreads();
        for (int c = 0; c < cw; ++c) {
            const float qv = scale * q_s[warp * cc + c];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int col = lane + 32 * e;
                if (col < P) dot[e] = fmaf(qv, kr_s[col * (cc + 1) + c], dot[e]);
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
