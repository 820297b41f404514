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

// One thread per (image, region, 16-byte channel group, token slot), for q and k
// together: it sums the region's tokens whose column is congruent to its slot modulo
// `ns`, issuing its 16-byte loads four per tensor at a time (eight in flight); the ns
// slots of a unit are adjacent lanes G apart and meet by shuffles. ns divides wr and
// G*ns divides 32 (or ns = 1). Output: float32 means, (N, P, C) for q and for k.
template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
region_mean_kernel(const T *__restrict__ q, const T *__restrict__ k, float *__restrict__ q_r,
                   float *__restrict__ k_r, int N, int H, int W, int C, int S, int ns_log2, int total) {
    constexpr int V = Elem<T>::kVec;
    const int t = blockIdx.x * kPoolThreads + threadIdx.x;  // total < 2^31 (checked by the host)
    const bool valid = t < total;
    const int G = C / V, ns = 1 << ns_log2, P = S * S;
    const int tt = valid ? t : 0;
    const int rest = tt / G;
    const int g = tt - rest * G;
    const int s = rest & (ns - 1);
    const int np = rest >> ns_log2;
    const int n = np / P, p = np - n * P;
    const int j = p / S, i = p - j * S;
    const int hr = H / S, wr = W / S;
    const size_t org = (((size_t)n * H + j * hr) * W + i * wr) * C + g * V;
    const T *oq = q + org, *ok = k + org;
    const int count = valid ? hr * (wr >> ns_log2) : 0;

    float aq[V], ak[V];
#pragma unroll
    for (int e = 0; e < V; ++e) aq[e] = ak[e] = 0.f;
    int th = 0, tw = s;
    for (int it = 0; it < count; it += 4) {
        uint4 bq[4], bk[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            bq[b] = bk[b] = make_uint4(0u, 0u, 0u, 0u);
            if (it + b < count) {
                const size_t off = ((size_t)th * W + tw) * C;
                bq[b] = __ldg(reinterpret_cast<const uint4 *>(oq + off));
                bk[b] = __ldg(reinterpret_cast<const uint4 *>(ok + off));
                tw += ns;
                if (tw >= wr) {
                    tw = s;
                    ++th;
                }
            }
        }
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            float f[V];
            unpack16(bq[b], f, q);
#pragma unroll
            for (int e = 0; e < V; ++e) aq[e] += f[e];
            unpack16(bk[b], f, k);
#pragma unroll
            for (int e = 0; e < V; ++e) ak[e] += f[e];
        }
    }
    for (int off = G; off < (G << ns_log2); off <<= 1)
#pragma unroll
        for (int e = 0; e < V; ++e) {
            aq[e] += __shfl_xor_sync(0xffffffffu, aq[e], off);
            ak[e] += __shfl_xor_sync(0xffffffffu, ak[e], off);
        }
    if (valid && s == 0) {
        const size_t o = (size_t)np * C + g * V;
        const float w2 = (float)(hr * wr);
#pragma unroll
        for (int e = 0; e < V; e += 4) {
            *reinterpret_cast<float4 *>(q_r + o + e) = make_float4(aq[e] / w2, aq[e + 1] / w2, aq[e + 2] / w2, aq[e + 3] / w2);
            *reinterpret_cast<float4 *>(k_r + o + e) = make_float4(ak[e] / w2, ak[e + 1] / w2, ak[e + 2] / w2, ak[e + 3] / w2);
        }
    }
}

// Large regions (w2 >= 64): one CTA per (image, region). Thread = (16-byte channel
// group g, token slot s) over q and k; slots stride the region's tokens with four
// independent loads of each tensor in flight (few registers, so four CTAs share an
// SM); partial sums meet in shared memory.
template <typename T>
__global__ void __launch_bounds__(kPoolThreads, 4)
region_mean_big_kernel(const T *__restrict__ q, const T *__restrict__ k, float *__restrict__ q_r,
                       float *__restrict__ k_r, int H, int W, int C, int S, FastDiv div_wr) {
    constexpr int V = Elem<T>::kVec;
    __shared__ float red[2][kPoolThreads * V];  // [tensor][slots][C]
    const int P = S * S, np = blockIdx.x;
    const int n = np / P, p = np - n * P;
    const int j = p / S, i = p - j * S;
    const int hr = H / S, wr = W / S, w2 = hr * wr;
    const int G = C / V, slots = kPoolThreads / G;
    const int g = threadIdx.x % G, sl = threadIdx.x / G;
    const size_t org = (((size_t)n * H + j * hr) * W + i * wr) * C + g * V;
    float aq[V], ak[V];
#pragma unroll
    for (int e = 0; e < V; ++e) aq[e] = ak[e] = 0.f;
    if (sl < slots) {
        for (int t0 = sl; t0 < w2; t0 += 4 * slots) {
            uint4 bq[4], bk[4];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int t = t0 + b * slots;
                bq[b] = bk[b] = make_uint4(0u, 0u, 0u, 0u);
                if (t < w2) {
                    uint32_t twu;
                    const int th = (int)div_wr.divmod((uint32_t)t, twu), tw = (int)twu;
                    const size_t off = org + ((size_t)th * W + tw) * C;
                    bq[b] = __ldg(reinterpret_cast<const uint4 *>(q + off));
                    bk[b] = __ldg(reinterpret_cast<const uint4 *>(k + off));
                }
            }
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                float f[V];
                unpack16(bq[b], f, q);
#pragma unroll
                for (int e = 0; e < V; ++e) aq[e] += f[e];
                unpack16(bk[b], f, k);
#pragma unroll
                for (int e = 0; e < V; ++e) ak[e] += f[e];
            }
        }
#pragma unroll
        for (int e = 0; e < V; ++e) {
            red[0][sl * C + g * V + e] = aq[e];
            red[1][sl * C + g * V + e] = ak[e];
        }
    }
    __syncthreads();
    for (int c = threadIdx.x; c < 2 * C; c += kPoolThreads) {
        const int tensor = c >= C, cc = c - tensor * C;
        float sum = 0.f;
        for (int t = 0; t < slots; ++t) sum += red[tensor][t * C + cc];
        (tensor ? k_r : q_r)[(size_t)np * C + cc] = sum / (float)w2;
    }
}

// ----------------------------------------------------------------------------- top-k

// Strict total order used by the routing: larger logit first, equal logits ->
// lower region index first.
__device__ inline bool route_before(float av, int ai, float bv, int bi) {
    return av > bv || (av == bv && ai < bi);
}

constexpr int kRouteWarps = 8;

// Channels of k_r staged in shared memory per pass: the largest multiple of 32 (at
// most C) whose [32E][cc+4] tile and [8*RPW][cc] query rows fit in 160 KB.
inline int route_chunk(int PP, int rows, int C) {
    int cc = C;
    while (cc > 32 && (PP * (cc + 4) + rows * cc) * 4 > 160 * 1024) cc -= 32;
    return cc;
}
inline int route_smem_bytes(int PP, int rows, int cc) {
    const int dots = rows * PP;  // reuses the k_r tile when it fits
    const int tile = PP * (cc + 4) + rows * cc;
    return (tile > dots ? tile : dots) * 4;
}

// Shared memory of route_cols_kernel: the scaled query means and the logits of its rows.
inline int route_cols_smem_bytes(int rows, int C) { return (rows * C + rows * 256) * 4; }

// Top-k selection and softmax of one affinity row (dots: the row's PP = 32E logits in
// shared memory), run by one warp; writes topk (index, weight) pairs at out_idx /
// out_w. topk <= 8 by repeated warp argmax, larger topk by a bitonic sort of all 32E
// (value, index) pairs. Order: larger logit first, equal logits -> lower index first.
template <int E>
__device__ __forceinline__ void route_select_row(const float *dots, int P, int topk, int lane, int32_t *out_idx,
                                                 float *out_w) {
    constexpr int PP = 32 * E;
    float val[E];
    int id[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int col = lane + 32 * e;
        val[e] = col < P ? dots[col] : -INFINITY;
        id[e] = col;  // padding columns carry unique indices >= P and lose every comparison
    }
    if (topk <= 8) {
        // topk rounds of warp argmax; lane `round` keeps that round's winner
        unsigned taken = 0;
        float my_v = 0.f;
        int my_i = 0;
        float v0 = 0.f;
        for (int round = 0; round < topk; ++round) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int e = 0; e < E; ++e)
                if (!(taken & (1u << e)) && (id[e] < P) && route_before(val[e], id[e], bv, bi)) {
                    bv = val[e];
                    bi = id[e];
                }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (route_before(ov, oi, bv, bi)) {
                    bv = ov;
                    bi = oi;
                }
            }
            if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
            if (lane == round) {
                my_v = bv;
                my_i = bi;
            }
            if (round == 0) v0 = bv;
        }
        const float ex = lane < topk ? expf(my_v - v0) : 0.f;
        float z = ex;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        if (lane < topk) {
            out_idx[lane] = my_i;
            out_w[lane] = ex / z;
        }
        return;
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
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int pos = e * 32 + lane;
        if (pos < topk) {
            out_idx[pos] = id[e];
            out_w[pos] = expf(val[e] - vmax) * inv_z;
        }
    }
}

// One CTA per (image n, block of 8*RPW affinity rows). Each warp owns RPW rows and each
// lane the columns lane + 32e (e < E, 32E >= P): per four channels it loads RPW
// query float4s (broadcast) and E key float4s and issues 4*RPW*E FMAs. k_r rows
// have a pitch of cc+4 floats (an odd number of 16-byte units: conflict-free float4
// reads across lanes); rows past P are zero. The dot products then go through shared
// memory to one warp per row for the selection: topk <= 8 by repeated warp argmax,
// larger topk by a bitonic sort of all 32E (value, index) pairs. Order: larger logit
// first, equal logits -> lower region index first.
template <int E, int RPW>
__global__ void __launch_bounds__(kRouteWarps * 32)
route_kernel(const float *__restrict__ q_r, const float *__restrict__ k_r, int C, int P, int topk, int cc,
             float scale, int32_t *__restrict__ r_idx, float *__restrict__ r_weight, FastDiv div_q4) {
    extern __shared__ __align__(16) float route_s[];
    constexpr int PP = 32 * E;
    constexpr int ROWS = kRouteWarps * RPW;
    griddep_wait();               // pooled means come from the preceding kernel
    griddep_launch_dependents();  // the attention kernel may start its prologue
    const int n = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int p0 = blockIdx.x * ROWS;
    const float *kimg = k_r + (size_t)n * P * C;
    const float *qimg = q_r + (size_t)n * P * C;
    const int kp = cc + 4;                 // k_r tile pitch (floats)
    float *kr_s = route_s;                 // [PP][kp]
    float *q_s = route_s + PP * kp;        // [ROWS][cc]

    float dot[RPW][E];
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int e = 0; e < E; ++e) dot[r][e] = 0.f;

    for (int c0 = 0; c0 < C; c0 += cc) {
        const int cw = min(cc, C - c0), q4 = cw >> 2;
        __syncthreads();
        // staging: eight independent float4 loads per thread in flight, then the stores
        // (element idx -> row idx / q4, column 4 * (idx % q4); q4 = cw / 4 is div_q4's
        // divisor, the same for every pass since C is a multiple of cc)
        for (int i0 = threadIdx.x; i0 < (PP + ROWS) * q4; i0 += 8 * blockDim.x) {
            float4 buf[8];
            int rr[8], cc4[8];
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                const int idx = i0 + b * blockDim.x;
                uint32_t cm;
                rr[b] = (int)div_q4.divmod((uint32_t)idx, cm);
                cc4[b] = (int)cm * 4;
                buf[b] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (rr[b] < P) {
                    buf[b] = __ldg(reinterpret_cast<const float4 *>(kimg + (size_t)rr[b] * C + c0 + cc4[b]));
                } else if (rr[b] >= PP && rr[b] < PP + ROWS) {
                    buf[b] = __ldg(reinterpret_cast<const float4 *>(qimg + (size_t)min(p0 + rr[b] - PP, P - 1) * C + c0 +
                                                                   cc4[b]));
                }
            }
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                if (rr[b] < PP) {
                    *reinterpret_cast<float4 *>(kr_s + rr[b] * kp + cc4[b]) = buf[b];
                } else if (rr[b] < PP + ROWS) {
                    float4 v = buf[b];
                    v.x *= scale;  // the walk-through scales the region query before the product
                    v.y *= scale;
                    v.z *= scale;
                    v.w *= scale;
                    *reinterpret_cast<float4 *>(q_s + (rr[b] - PP) * cc + cc4[b]) = v;
                }
            }
        }
        __syncthreads();
        for (int c = 0; c < cw; c += 4) {
            float4 qv[RPW], kv[E];
#pragma unroll
            for (int r = 0; r < RPW; ++r) qv[r] = *reinterpret_cast<const float4 *>(q_s + (warp * RPW + r) * cc + c);
#pragma unroll
            for (int e = 0; e < E; ++e) kv[e] = *reinterpret_cast<const float4 *>(kr_s + (lane + 32 * e) * kp + c);
#pragma unroll
            for (int r = 0; r < RPW; ++r)
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    dot[r][e] = fmaf(qv[r].x, kv[e].x, dot[r][e]);
                    dot[r][e] = fmaf(qv[r].y, kv[e].y, dot[r][e]);
                    dot[r][e] = fmaf(qv[r].z, kv[e].z, dot[r][e]);
                    dot[r][e] = fmaf(qv[r].w, kv[e].w, dot[r][e]);
                }
        }
    }

    // every row's logits to one warp: dots[row][col]
    __syncthreads();
    float *dots = route_s;
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int e = 0; e < E; ++e) dots[(warp * RPW + r) * PP + lane + 32 * e] = dot[r][e];
    __syncthreads();

    for (int r = 0; r < RPW; ++r) {
        const int row = warp * RPW + r, p = p0 + row;
        if (p >= P) break;
        const size_t base = ((size_t)n * P + p) * topk;
        route_select_row<E>(dots + row * PP, P, topk, lane, r_idx + base, r_weight + base);
    }
}

// Many regions (32E = 256 columns): one CTA per (image n, block of ROWS affinity rows),
// eight warps; thread t owns column t for all ROWS rows. It loads its own column's key
// means straight into registers, 64 channels at a time (16 independent float4 loads in
// flight), and multiplies them with the ROWS scaled query means broadcast from shared
// memory; no key mean is staged. Selection as in route_kernel.
template <int ROWS>
__global__ void __launch_bounds__(kRouteWarps * 32)
route_cols_kernel(const float *__restrict__ q_r, const float *__restrict__ k_r, int C, int P, int topk, float scale,
                  int32_t *__restrict__ r_idx, float *__restrict__ r_weight) {
    extern __shared__ __align__(16) float route_s[];
    constexpr int E = 8, PP = 32 * E;
    griddep_wait();               // pooled means come from the preceding kernel
    griddep_launch_dependents();  // the attention kernel may start its prologue
    const int n = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int p0 = blockIdx.x * ROWS;
    const float *kimg = k_r + (size_t)n * P * C;
    const float *qimg = q_r + (size_t)n * P * C;
    float *q_s = route_s;              // [ROWS][C]
    float *dots = route_s + ROWS * C;  // [ROWS][PP]
    const int col = threadIdx.x;
    const float4 *kc = reinterpret_cast<const float4 *>(kimg + (size_t)min(col, P - 1) * C);
    float4 kv[16];
#pragma unroll
    for (int b = 0; b < 16; ++b) kv[b] = 4 * b < C ? __ldg(kc + b) : make_float4(0.f, 0.f, 0.f, 0.f);
    const int c4n = C >> 2;
    for (int i = threadIdx.x; i < ROWS * c4n; i += blockDim.x) {
        const int r = i / c4n, c4 = i - r * c4n;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p0 + r < P) v = __ldg(reinterpret_cast<const float4 *>(qimg + (size_t)(p0 + r) * C) + c4);
        v.x *= scale;  // the walk-through scales the region query before the product
        v.y *= scale;
        v.z *= scale;
        v.w *= scale;
        reinterpret_cast<float4 *>(q_s + r * C)[c4] = v;
    }
    __syncthreads();
    float dot[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) dot[r] = 0.f;
    for (int c0 = 0; c0 < C; c0 += 64) {
        if (c0 > 0) {
#pragma unroll
            for (int b = 0; b < 16; ++b) kv[b] = c0 + 4 * b < C ? __ldg(kc + c0 / 4 + b) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int b = 0; b < 16; ++b) {
            if (c0 + 4 * b >= C) break;
#pragma unroll
            for (int r = 0; r < ROWS; ++r) {
                const float4 qv = *reinterpret_cast<const float4 *>(q_s + r * C + c0 + 4 * b);
                dot[r] = fmaf(qv.x, kv[b].x, dot[r]);
                dot[r] = fmaf(qv.y, kv[b].y, dot[r]);
                dot[r] = fmaf(qv.z, kv[b].z, dot[r]);
                dot[r] = fmaf(qv.w, kv[b].w, dot[r]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < ROWS; ++r) dots[r * PP + col] = dot[r];
    __syncthreads();
    for (int row = warp; row < ROWS; row += kRouteWarps) {
        const int p = p0 + row;
        if (p >= P) break;
        const size_t base = ((size_t)n * P + p) * topk;
        route_select_row<E>(dots + row * PP, P, topk, lane, r_idx + base, r_weight + base);
    }
}

}  // namespace bra
