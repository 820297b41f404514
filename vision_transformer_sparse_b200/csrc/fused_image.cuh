// fused_image.cuh — the whole BRA forward in one kernel, for images small enough that
// one head's K, V and Q slices of a whole image fit in one CTA's shared memory (the
// classification stages: 28x28 and 14x14 maps).
//
// Computation (BRA walk-through on "BiFormer ... 前向传播过程", niftyadmin, section
// "BRA模块", eqs. 4-7): region means of q and k over all C channels, affinity
// (scale*q_r) k_r^T, top-k per row and the softmax of the selected logits; then for
// every query token and head, softmax((scale*q).k) v over the routed regions' tokens
// jointly, plus LCE(V): depthwise 5x5 convolution of the whole V image, zero padded,
// with bias.
//
// Work split. One CTA per (image n, head m); the `heads` CTAs of an image form a
// thread-block cluster (cluster rank = head).
//   1. One thread issues three tensor-copy boxes (64-byte rows: the head's 32
//      channels of every pixel) for Q, K (both 64-byte swizzled, for ldmatrix) and V
//      (unswizzled, for the LCE) onto one mbarrier.
//   2. Region means of the head's channels of q and k, and the partial affinity
//      A_m[p][p'] = sum over the head's channels of (scale*q_r[p]) k_r[p'].
//   3. Cluster barrier; the CTAs share the affinity rows (rank m takes rows m, m +
//      heads, ...): for each, the `heads` partial rows are summed from the peers'
//      shared memory (distributed shared memory, fixed order 0..heads-1), the top-k
//      selected, r_idx and r_weight written, and the row's indices stored into every
//      peer's index table; a second cluster barrier publishes the full routing.
//   4. Each warp takes regions p = warp, warp + nwarps, ...: mma.sync attention of the
//      region's 16-token query tile over its routed keys (rows looked up per key), O
//      to a per-warp staging tile, then the LCE of the region's pixels for the head's
//      channels from the resident V, added to O and stored.
// Global traffic: q, k, v read once, out written once; no scratch memory.
#pragma once

#include <cuda.h>

#include "attn_tma.cuh"
#include "route.cuh"

namespace bra {

struct ImageParams {
    CUtensorMap tmQ, tmK;  // box (32, W, H, 1), 64-byte swizzle
    CUtensorMap tmV;       // box (32, W + 4, H + 4, 1) from (-2, -2), no swizzle
    const __nv_bfloat16 *lce_w, *lce_b;
    __nv_bfloat16 *out;
    int32_t *r_idx;
    float *r_weight;
    int N, H, W, C, heads, S, topk, P;
    float scale, scale_log2;
    unsigned wait_limit;
    FastDiv div_S, div_W;
};

struct ImageSmem {
    int q, k, v, qr, kr, a, ridx, base, keyrow, o, bar, total;
};

// Byte offsets from a 1024-aligned base. Q and K: H*W pixels of 64 bytes; V: the
// (H+4) x (W+4) zero-bordered image (the convolution's padding comes with the copy).
// routed: the routing comes from global memory, so no pooling or affinity buffers.
__host__ __device__ inline ImageSmem image_smem_layout(int H, int W, int P, int topk, int w2, int nwarps,
                                                       bool routed = false) {
    ImageSmem s;
    const int tile = ((H * W * 64 + 1023) / 1024) * 1024;
    const int vtile = (((H + 4) * (W + 4) * 64 + 1023) / 1024) * 1024;
    const int L = topk * w2, kpad = (L + kKC - 1) / kKC * kKC;
    s.q = 0;
    s.k = s.q + tile;
    s.v = s.k + tile;
    int end = s.v + vtile;
    const int rp = routed ? 0 : P;
    s.qr = end;  // [P][32] fp32 region means of the head's q channels
    end += align16(rp * 32 * 4);
    s.kr = end;  // [P][36]: pitch of 9 16-byte units, conflict-free float4 reads
    end += align16(rp * 36 * 4);
    s.a = end;  // [P][P] partial affinity of this head (read by the cluster peers)
    end += align16(rp * P * 4);
    s.ridx = end;  // [P][topk]
    end += align16(P * topk * 4);
    s.base = end;  // [P] first pixel row of each region
    end += align16(P * 4);
    s.keyrow = end;  // [nwarps][kpad] pixel row of each key of the warp's current region
    end += align16(nwarps * kpad * 4);
    s.o = end;  // [nwarps][16][34] fp32 attention output staging
    end += align16(nwarps * 16 * 34 * 4);
    s.bar = end;
    end += 16;
    s.total = end + 1024;
    return s;
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void st_dsmem_s32(uint32_t local_addr, uint32_t rank, int v) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(ra) : "r"(local_addr), "r"(rank));
    asm volatile("st.shared::cluster.s32 [%0], %1;\n" ::"r"(ra), "r"(v) : "memory");
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t local_addr, uint32_t rank) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(ra) : "r"(local_addr), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];\n" : "=f"(v) : "r"(ra) : "memory");
    return v;
}
// 16-byte chunk `ck` (0..3) of 64-byte row `row` in a 64-byte-swizzled tile.
__device__ __forceinline__ uint32_t swz64(uint32_t tile, int row, int ck) {
    return tile + row * 64 + (((ck ^ (row >> 1)) & 3) << 4);
}

// HR x WR regions, 32 channels per head. kRouted: steps 1-3 ran in the routing kernels
// before this one (launched with programmatic dependent launch): the kernel copies its
// tiles while they finish, then takes r_idx from global memory and runs step 4-5 only;
// no cluster, no pooling, no affinity.
template <int HR, int WR, bool kRouted>
__global__ void __launch_bounds__(512, 1) bra_image_kernel(const __grid_constant__ ImageParams prm) {
    constexpr int D = 32, W2 = HR * WR;
    static_assert(W2 <= 16, "a region's queries fill at most one 16-row tile");
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (sbase - raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nwarps = blockDim.x >> 5;
    const int H = prm.H, W = prm.W, HW = H * W, P = prm.P, topk = prm.topk;
    const int L = topk * W2, kpad = (L + kKC - 1) / kKC * kKC;
    const ImageSmem Ls = image_smem_layout(H, W, P, topk, W2, nwarps, kRouted);
    const int WP = W + 4;  // padded V row pitch (pixels)
    const int m = kRouted ? (int)(blockIdx.x % prm.heads) : (int)cluster_ctarank();
    const int n = blockIdx.x / prm.heads;
    const int c0 = m * D;
    float *qr = reinterpret_cast<float *>(sm + Ls.qr);
    float *kr = reinterpret_cast<float *>(sm + Ls.kr);
    float *A = reinterpret_cast<float *>(sm + Ls.a);
    int *ridx = reinterpret_cast<int *>(sm + Ls.ridx);
    int *rbase = reinterpret_cast<int *>(sm + Ls.base);
    int *keyrow = reinterpret_cast<int *>(sm + Ls.keyrow) + warp * kpad;
    float *sOw = reinterpret_cast<float *>(sm + Ls.o) + warp * 16 * 34;
    const uint32_t tQ = sbase + Ls.q, tK = sbase + Ls.k, tV = sbase + Ls.v;
    const uint32_t bar = sbase + Ls.bar;

    // ---------------------------------------------------------------- 1. load
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        mbar_arrive_expect_tx(bar, (2u * HW + (uint32_t)(H + 4) * (W + 4)) * 64u);
        tma_load_4d(tQ, &prm.tmQ, c0, 0, 0, n, bar);
        tma_load_4d(tK, &prm.tmK, c0, 0, 0, n, bar);
        tma_load_4d(tV, &prm.tmV, c0, -2, -2, n, bar);
    }
    for (int p = tid; p < P; p += blockDim.x) {
        uint32_t i;
        const int j = (int)prm.div_S.divmod((uint32_t)p, i);
        rbase[p] = j * HR * W + (int)i * WR;
    }
    // LCE weights and bias of this lane's channel pair (fixed for the whole kernel)
    const int cp = lane & 15;
    float2 wt[25], bias;
    {
        const int c = c0 + 2 * cp;
        const uint32_t *wp = reinterpret_cast<const uint32_t *>(prm.lce_w + (size_t)c * 25);
        uint32_t wv[25];
#pragma unroll
        for (int t = 0; t < 25; ++t) wv[t] = __ldg(wp + t);
#pragma unroll
        for (int t = 0; t < 25; ++t) {
            const int e0 = t, e1 = 25 + t;
            const uint32_t u0 = wv[e0 >> 1], u1 = wv[e1 >> 1];
            wt[t].x = __uint_as_float((e0 & 1) ? (u0 & 0xFFFF0000u) : (u0 << 16));
            wt[t].y = __uint_as_float((e1 & 1) ? (u1 & 0xFFFF0000u) : (u1 << 16));
        }
        bias = bf16x2_to_float2(__ldg(reinterpret_cast<const uint32_t *>(prm.lce_b + c)));
    }
    if constexpr (kRouted) {
        griddep_wait();  // r_idx comes from the preceding routing kernel
        const int32_t *src = prm.r_idx + (size_t)n * P * topk;
        for (int i = tid; i < P * topk; i += blockDim.x) {
            const int r = __ldcg(src + i);
            ridx[i] = r >= 0 && r < P ? r : 0;  // the routing kernels only write indices in range
        }
    }
    const bool ok = __syncthreads_and(mbar_wait_bounded(bar, 0, prm.wait_limit));
    if (!ok) {
        if (tid == 0) atomicExch(&g_bra_timeout_flag, 1);
        mbar_wait_bounded(bar, 0, prm.wait_limit);
        if constexpr (!kRouted) {
            // keep the cluster's barrier sequence intact before leaving
            cluster_arrive();
            cluster_wait();
            cluster_arrive();
            cluster_wait();
        }
        return;
    }

    if constexpr (!kRouted) {
        // ---------------------------------------------------------------- 2. means, partial affinity
        // region sums as column sums on the tensor cores: one warp per (tensor, region),
        // D[16 x 32] = ones[16 x W2] * X[W2 x 32] (bf16 in, fp32 accumulate: exact products,
        // fp32 sums), X read with ldmatrix.trans like the V operand of the attention; every
        // row of D holds the sums, lanes 0-3 write row 0.
        {
            const int kc = 2 * (lane & 3);  // this lane's k (token) pair in the A fragment
            const uint32_t one2 = 0x3F803F80u;
            uint32_t a1[4];
            a1[0] = a1[1] = kc < W2 ? one2 : 0u;          // tokens kc, kc+1
            a1[2] = a1[3] = kc + 8 < W2 ? one2 : 0u;      // tokens kc+8, kc+9
            const int tl = (lane & 7) + ((lane >> 3) & 1) * 8;  // token row this lane addresses
            const int tt = tl < W2 ? tl : 0;                     // rows past W2 meet zeros in A
            const int toff = (tt / WR) * W + (tt % WR);
            for (int it = warp; it < 2 * P; it += nwarps) {
                const int tensor = it >= P, p = it - tensor * P;
                const uint32_t tile = tensor ? tK : tQ;
                const int row = rbase[p] + toff;
                float d[4][4];
#pragma unroll
                for (int t = 0; t < 4; ++t) d[t][0] = d[t][1] = d[t][2] = d[t][3] = 0.f;
#pragma unroll
                for (int dp = 0; dp < 2; ++dp) {
                    uint32_t b0, b1, b2, b3;
                    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                                 : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3)
                                 : "r"(swz64(tile, row, dp * 2 + ((lane >> 4) & 1))));
                    mma_bf16_16816(d[2 * dp], a1, b0, b1);
                    mma_bf16_16816(d[2 * dp + 1], a1, b2, b3);
                }
                if (lane < 4) {
                    const float inv = 1.f / (float)W2;
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int c = 8 * t + kc;
                        if (tensor) {
                            *reinterpret_cast<float2 *>(kr + p * 36 + c) = make_float2(d[t][0] * inv, d[t][1] * inv);
                        } else {  // scale * q_r, as the walk-through
                            *reinterpret_cast<float2 *>(qr + p * 32 + c) =
                                make_float2(prm.scale * (d[t][0] * inv), prm.scale * (d[t][1] * inv));
                        }
                    }
                }
            }
        }
        __syncthreads();
        // affinity rows two at a time per warp (they share the key loads), lane = columns
        // lane and lane + 32; one partial sum per float4 component keeps the chains short
        for (int p = 2 * warp; p < P; p += 2 * nwarps) {
            const int p2 = p + 1 < P ? p + 1 : p;
            float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0, b0 = a0, b1 = a0;
            const int c1 = lane < P ? lane : 0, cB = lane + 32 < P ? lane + 32 : lane;
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
                const float4 qv = *reinterpret_cast<const float4 *>(qr + p * 32 + c);
                const float4 qw = *reinterpret_cast<const float4 *>(qr + p2 * 32 + c);
                const float4 k0 = *reinterpret_cast<const float4 *>(kr + c1 * 36 + c);
                const float4 k1 = *reinterpret_cast<const float4 *>(kr + cB * 36 + c);
                a0.x = fmaf(qv.x, k0.x, a0.x);
                a0.y = fmaf(qv.y, k0.y, a0.y);
                a0.z = fmaf(qv.z, k0.z, a0.z);
                a0.w = fmaf(qv.w, k0.w, a0.w);
                a1.x = fmaf(qv.x, k1.x, a1.x);
                a1.y = fmaf(qv.y, k1.y, a1.y);
                a1.z = fmaf(qv.z, k1.z, a1.z);
                a1.w = fmaf(qv.w, k1.w, a1.w);
                b0.x = fmaf(qw.x, k0.x, b0.x);
                b0.y = fmaf(qw.y, k0.y, b0.y);
                b0.z = fmaf(qw.z, k0.z, b0.z);
                b0.w = fmaf(qw.w, k0.w, b0.w);
                b1.x = fmaf(qw.x, k1.x, b1.x);
                b1.y = fmaf(qw.y, k1.y, b1.y);
                b1.z = fmaf(qw.z, k1.z, b1.z);
                b1.w = fmaf(qw.w, k1.w, b1.w);
            }
            if (lane < P) A[p * P + lane] = (a0.x + a0.y) + (a0.z + a0.w);
            if (lane + 32 < P) A[p * P + lane + 32] = (a1.x + a1.y) + (a1.z + a1.w);
            if (p2 != p) {
                if (lane < P) A[p2 * P + lane] = (b0.x + b0.y) + (b0.z + b0.w);
                if (lane + 32 < P) A[p2 * P + lane + 32] = (b1.x + b1.y) + (b1.z + b1.w);
            }
        }

        // ---------------------------------------------------------------- 3. routing
        cluster_arrive();  // our partial affinity is complete and visible to the peers
        cluster_wait();
        const uint32_t Aloc = sbase + Ls.a;
        const uint32_t Rloc = sbase + Ls.ridx;
        // the cluster's CTAs share the rows: this CTA selects rows m, m + heads, ... and
        // writes each row's routing into every peer's index table
        for (int p = m + warp * prm.heads; p < P; p += nwarps * prm.heads) {
            float val[2];
            int id[2];
            {
                // every peer's partial first (independent remote loads), then the sums in rank order
                float part[2][8];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int col = min(lane + 32 * e, P - 1);
#pragma unroll
                    for (int r = 0; r < 8; ++r) part[e][r] = r < prm.heads ? ld_dsmem_f32(Aloc + (p * P + col) * 4, r) : 0.f;
                }
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int col = lane + 32 * e;
                    float s = 0.f;
#pragma unroll
                    for (int r = 0; r < 8; ++r)
                        if (r < prm.heads) s += part[e][r];
                    id[e] = col;
                    val[e] = col < P ? s : -INFINITY;
                }
            }
            // topk rounds of warp argmax (larger logit first, ties to the lower region index);
            // round r's winner is kept by lane r % 32 in slot r / 32 (topk <= 64)
            unsigned taken = 0;
            float my_v[2] = {0.f, 0.f}, v0 = 0.f;
            int my_i[2] = {0, 0};
            for (int round = 0; round < topk; ++round) {
                float bv = -INFINITY;
                int bi = 0x7fffffff;
#pragma unroll
                for (int e = 0; e < 2; ++e)
                    if (!(taken & (1u << e)) && id[e] < P && route_before(val[e], id[e], bv, bi)) {
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
                if (lane == (round & 31)) {
                    my_v[round >> 5] = bv;
                    my_i[round >> 5] = bi;
                }
                if (round == 0) v0 = bv;
            }
            // r_weight: softmax of the selected logits
            float ex[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) ex[e] = lane + 32 * e < topk ? expf(my_v[e] - v0) : 0.f;
            float z = ex[0] + ex[1];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int slot = lane + 32 * e;
                if (slot < topk) {
                    const size_t o = ((size_t)n * P + p) * topk + slot;
                    prm.r_idx[o] = my_i[e];
                    prm.r_weight[o] = ex[e] / z;
                    for (int r = 0; r < prm.heads; ++r)
                        st_dsmem_s32(Rloc + (p * topk + slot) * 4, (uint32_t)r, my_i[e]);
                }
            }
        }
        cluster_arrive();  // every row's routing is in every CTA; the partial affinities are no longer read
        cluster_wait();
    }

    // ---------------------------------------------------------------- 4. attention + LCE
    const int nchunks = kpad / kKC;
    const bool need_mask = (L % kKC) != 0;
    const float sl2 = prm.scale_log2;
    // LCE item of this lane: channel pair cp, columns xh, xh + 2, ... of the region
    const int xh = lane >> 4;
    for (int p = warp; p < P; p += nwarps) {
        const int *rp = ridx + p * topk;
        // key j -> pixel row of its routed region's token (K tile); the V tile row is
        // the same pixel in the bordered image: row + 2*WP + 2 + 4*(row / W)
        for (int jj = lane; jj < kpad; jj += 32) {
            int row = rbase[rp[0]];
            if (jj < L) {
                const int a = jj / W2, t = jj - a * W2;
                row = rbase[rp[a]] + (t / WR) * W + (t % WR);
            }
            keyrow[jj] = row;
        }
        __syncwarp();
        // Q tile: tokens t < W2 of region p (rows beyond W2 repeat token 0 and are unused)
        uint32_t qa[2][4];
        {
            const int t = (lane & 7) + ((lane >> 3) & 1) * 8;
            const int tt = t < W2 ? t : 0;
            const int row = rbase[p] + (tt / WR) * W + (tt % WR);
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                const int ck = kk * 2 + ((lane >> 4) & 1);
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                             : "=r"(qa[kk][0]), "=r"(qa[kk][1]), "=r"(qa[kk][2]), "=r"(qa[kk][3])
                             : "r"(swz64(tQ, row, ck)));
            }
        }
        float m_i[2] = {-INFINITY, -INFINITY}, l_i[2] = {0.f, 0.f};
        float acc[4][4];
#pragma unroll
        for (int t = 0; t < 4; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
        for (int ch = 0; ch < nchunks; ++ch) {
            float sc[8][4];
#pragma unroll
            for (int t = 0; t < 8; ++t) sc[t][0] = sc[t][1] = sc[t][2] = sc[t][3] = 0.f;
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                const int row = keyrow[ch * kKC + np * 16 + (lane & 7) + ((lane >> 4) & 1) * 8];
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    uint32_t b0, b1, b2, b3;
                    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                                 : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3)
                                 : "r"(swz64(tK, row, kk * 2 + ((lane >> 3) & 1))));
                    mma_bf16_16816(sc[2 * np], qa[kk], b0, b1);
                    mma_bf16_16816(sc[2 * np + 1], qa[kk], b2, b3);
                }
            }
            float rmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int t = 0; t < 8; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (need_mask && ch * kKC + t * 8 + 2 * (lane & 3) + (e & 1) >= L) sc[t][e] = -INFINITY;
                    rmax[e >> 1] = fmaxf(rmax[e >> 1], sc[t][e]);
                }
            float mneg[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                rmax[r] = fmaxf(rmax[r], __shfl_xor_sync(0xffffffffu, rmax[r], 1));
                rmax[r] = fmaxf(rmax[r], __shfl_xor_sync(0xffffffffu, rmax[r], 2));
                const float m_new = fmaxf(m_i[r], rmax[r]);
                const float mref = m_new == -INFINITY ? 0.f : m_new;
                if (ch > 0) {
                    const float alpha = fast_exp2((m_i[r] - mref) * sl2);
                    l_i[r] *= alpha;
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        acc[t][2 * r] *= alpha;
                        acc[t][2 * r + 1] *= alpha;
                    }
                }
                m_i[r] = m_new;
                mneg[r] = -mref * sl2;
            }
#pragma unroll
            for (int t = 0; t < 8; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float pe = fast_exp2(fmaf(sc[t][e], sl2, mneg[e >> 1]));
                    sc[t][e] = pe;
                    l_i[e >> 1] += pe;
                }
#pragma unroll
            for (int kt = 0; kt < 4; ++kt) {
                uint32_t pa[4];
                pa[0] = pack_bf16x2(sc[2 * kt][0], sc[2 * kt][1]);
                pa[1] = pack_bf16x2(sc[2 * kt][2], sc[2 * kt][3]);
                pa[2] = pack_bf16x2(sc[2 * kt + 1][0], sc[2 * kt + 1][1]);
                pa[3] = pack_bf16x2(sc[2 * kt + 1][2], sc[2 * kt + 1][3]);
                const int prow = keyrow[ch * kKC + kt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8];
                const int row = prow + 2 * WP + 2 + 4 * (int)prm.div_W.div((uint32_t)prow);  // same pixel, bordered V
#pragma unroll
                for (int dp = 0; dp < 2; ++dp) {
                    uint32_t b0, b1, b2, b3;
                    // V is unswizzled: 16-byte chunk ck of row r at r*64 + ck*16
                    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                                 : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3)
                                 : "r"(tV + row * 64 + (dp * 2 + ((lane >> 4) & 1)) * 16));
                    mma_bf16_16816(acc[2 * dp], pa, b0, b1);
                    mma_bf16_16816(acc[2 * dp + 1], pa, b2, b3);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            l_i[r] += __shfl_xor_sync(0xffffffffu, l_i[r], 1);
            l_i[r] += __shfl_xor_sync(0xffffffffu, l_i[r], 2);
        }
        const float inv0 = l_i[0] > 0.f ? 1.f / l_i[0] : 0.f;
        const float inv1 = l_i[1] > 0.f ? 1.f / l_i[1] : 0.f;
        {
            const int r0 = lane >> 2;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int col = t * 8 + 2 * (lane & 3);
                *reinterpret_cast<float2 *>(sOw + r0 * 34 + col) = make_float2(acc[t][0] * inv0, acc[t][1] * inv0);
                *reinterpret_cast<float2 *>(sOw + (r0 + 8) * 34 + col) = make_float2(acc[t][2] * inv1, acc[t][3] * inv1);
            }
        }
        __syncwarp();

        // LCE of region p for the head's channels: lane = (pair cp, first column xh);
        // columns xh, xh + 2, ... of the region, all HR rows, from the resident V.
        uint32_t x0u;
        const int y0 = (int)prm.div_W.divmod((uint32_t)rbase[p], x0u), x0 = (int)x0u;
        constexpr int NX = (WR + 1) / 2;        // columns per lane
        constexpr int SPAN = 2 * (NX - 1) + 5;  // pixels per halo row covering them
        float2 out2[HR][NX];
#pragma unroll
        for (int r = 0; r < HR; ++r)
#pragma unroll
            for (int xi = 0; xi < NX; ++xi) out2[r][xi] = bias;
        // bordered V: pixel (y, x) of the image is row (y+2)*WP + x+2, zero outside
        const uint32_t vrow0 = tV + ((y0 * WP) + x0 + xh) * 64 + cp * 4;
#pragma unroll
        for (int hy = 0; hy < HR + 4; ++hy) {
            float2 v[SPAN];
#pragma unroll
            for (int b = 0; b < SPAN; ++b) v[b] = bf16x2_to_float2(ld_shared_u32(vrow0 + (hy * WP + b) * 64));
#pragma unroll
            for (int r = 0; r < HR; ++r) {
                const int a = hy - r;
                if (a < 0 || a >= 5) continue;
#pragma unroll
                for (int xi = 0; xi < NX; ++xi)
#pragma unroll
                    for (int b = 0; b < 5; ++b) out2[r][xi] = ffma2(wt[a * 5 + b], v[2 * xi + b], out2[r][xi]);
            }
        }
#pragma unroll
        for (int r = 0; r < HR; ++r)
#pragma unroll
            for (int xi = 0; xi < NX; ++xi) {
                const int x = xh + 2 * xi;
                if (x >= WR) continue;
                const float2 o = *reinterpret_cast<const float2 *>(sOw + (r * WR + x) * 34 + 2 * cp);
                __nv_bfloat16 *dst = prm.out + (((size_t)n * H + y0 + r) * W + x0 + x) * prm.C + c0 + 2 * cp;
                *reinterpret_cast<__nv_bfloat162 *>(dst) = __floats2bfloat162_rn(o.x + out2[r][xi].x, o.y + out2[r][xi].y);
            }
        __syncwarp();
    }
}

}  // namespace bra
