// backward_tc.cuh — the BRA backward with the routing detached, on the tensor cores
// (warp-level mma.sync, bf16 operands, float32 accumulation) and deterministic: every
// output element is written by exactly one thread, in a fixed order, without atomics.
//
// Source: the walk-through's router ("BiFormer ... 前向传播过程", niftyadmin, section
// "BRA模块", `TopkRouting`) detaches the region-level query and key when `diff_routing` is
// off, its default; the top-k index is a discrete choice and r_weight does not scale K or
// V, so gradients flow through the token-to-token attention and the LCE only. Per image
// n, query region p and head m, with the routed keys j (the tokens of r_idx[n][p][*]):
//     s_ij = scale q_i . k_j,   A = softmax_j(s),   D_i = sum_j A_ij dA_ij = dO_i . o_i
//     dA_ij = dO_i . v_j,       dS_ij = A_ij (dA_ij - D_i)
//     dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,  dv_j = sum_i A_ij dO_i
//
// Kernels (bf16 maps, 32 channels per head):
//   bwd_tc_transpose_kernel: per image, the transposed routing: for every key region the
//       list of (query region, slot) entries e = p * topk + a that route to it, ascending
//       (one warp ranks the entries 32 at a time);
//   bwd_tc_query_kernel: one CTA per (image, query region, head), a warp per 16 queries.
//       Up to 64 keys: S = Q K^T and dA = dO V^T of both 32-key chunks in registers, the
//       row statistics and A from one set of exponentials, D = sum A dA, then dS and
//       dQ = scale dS K. More keys: two passes over the chunks, recomputing S: the row
//       statistics and O' = sum 2^(s - m) V (online), hence D = dO . O' / l = sum A dA;
//       then dA, dS and dQ. Stores dq and, per query, (lse, D) for the key side;
//   bwd_tc_key_kernel: one CTA per (image, key region, head), a warp per 16 keys. For each
//       entry of the key region's list (in list order) it recomputes S^T = K Q^T and
//       dA^T = V dO^T for the entry's queries, then dK += dS^T Q and dV += A^T dO in
//       registers; it stores dk and adds dv to the LCE part already stored (so no key is
//       written by two CTAs).
// A and dS enter their products split into a bf16 high part and a bf16 low part (two
// MMAs, about 16 mantissa bits), so that the float32 result is not limited by one bf16
// rounding of the probabilities; S and dA are exact products of the bf16 inputs.
//
// Shared-memory tiles hold rows of 32 channels (64 bytes) with the 64-byte swizzle (16-byte
// chunk c of row r at c ^ ((r >> 1) & 3)), so that ldmatrix reads of 8 rows are
// conflict-free. Masked keys (an r_idx entry outside [0, S*S), or padding of the last
// chunk) take no part in the softmax; padded query rows carry lse = +inf, so their
// probabilities and gradients are zero.
#pragma once

#include "common.cuh"

namespace bra {

constexpr int kBwdTcMaxWarps = 16;  // 256 tokens per region

struct BwdTcParams {
    const __nv_bfloat16 *q, *k, *v, *dout;  // (N,H,W,C)
    const int32_t *r_idx;                   // (N,P,topk)
    int *kv_off;                            // (N, P+1): start of each key region's list
    int *kv_list;                           // (N, P*topk): entries p*topk + a by key region
    float *dq, *dk, *dv;                    // (N,H,W,C) float32; dv holds the LCE part
    float *stats;                           // (N,P,heads,w2,2): lse (base 2) and D per query
    int *bad;                               // set to 1 when an r_idx entry is out of range
    int N, H, W, C, heads, S, topk, P, hr, wr, w2, L, nw;
    float scale, sl2;                       // scale and scale * log2(e)
    FastDiv div_S, div_wr, div_w2, div_topk, div_heads, div_P;  // the index arithmetic's divisors
};

__device__ __forceinline__ uint32_t tc_sw64(int row, int chunk) {
    return (uint32_t)(row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4));
}

// Element offset of channel 0 of token t of region r of image n.
__device__ __forceinline__ size_t tc_pix(const BwdTcParams &p, int n, int r, int t) {
    uint32_t ri, ti;
    const int ry = (int)p.div_S.divmod((uint32_t)r, ri), ty = (int)p.div_wr.divmod((uint32_t)t, ti);
    const int y = ry * p.hr + ty, x = (int)ri * p.wr + (int)ti;
    return (((size_t)n * p.H + y) * p.W + x) * p.C;
}

// 8-byte global -> shared copy (asynchronous; completes with the thread's cp.async group).
__device__ __forceinline__ void tc_cp_async8(uint32_t smem_dst, const void *gmem_src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(smem_dst), "l"(gmem_src) : "memory");
}

__device__ __forceinline__ void tc_split(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

// ----------------------------------------------------------------------------- routing

// One CTA per image: kv_off[n][pk] .. kv_off[n][pk+1] index the entries e = p * topk + a
// with r_idx[n][p][a] == pk, in ascending e. One warp walks the image's entries in order,
// 32 at a time, so the order does not depend on scheduling.
__global__ void __launch_bounds__(256) bwd_tc_transpose_kernel(const BwdTcParams p) {
    extern __shared__ int tr_s[];  // [P] counts, then running list positions
    const int n = blockIdx.x, E = p.P * p.topk;
    const int32_t *ri = p.r_idx + (size_t)n * E;
    int *cnt = tr_s;
    for (int k = threadIdx.x; k < p.P; k += blockDim.x) cnt[k] = 0;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int r = ri[e];
        if (r < 0 || r >= p.P) atomicExch(p.bad, 1);
    }
    __syncthreads();
    if (threadIdx.x >= 32) return;
    // one warp, entries in order, 32 at a time: the lanes holding the same key region find
    // each other (match_any); the group's leader adds its size to the region's count, and a
    // lane's rank in its group is its order among the chunk's entries of that region, so
    // every list comes out ascending in e, as a serial walk would write it
    const int lane = threadIdx.x;
    const unsigned below = (1u << lane) - 1u;
    for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        const int r = e < E ? ri[e] : -1;
        const bool ok = r >= 0 && r < p.P;
        const unsigned grp = __match_any_sync(0xffffffffu, ok ? r : -1);
        if (ok && (grp & below) == 0u) cnt[r] += __popc(grp);
        __syncwarp();
    }
    // exclusive prefix sum of the counts: lane l takes regions [l * per, (l + 1) * per)
    const int per = (p.P + 31) / 32;
    int local = 0;
    for (int k = lane * per; k < p.P && k < (lane + 1) * per; ++k) local += cnt[k];
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    int run = incl - local;  // entries of the regions before this lane's first one
    int *off = p.kv_off + (size_t)n * (p.P + 1);
    for (int k = lane * per; k < p.P && k < (lane + 1) * per; ++k) {
        const int c = cnt[k];
        off[k] = run;
        cnt[k] = run;
        run += c;
    }
    if (lane == 31) off[p.P] = incl;
    __syncwarp();
    int *list = p.kv_list + (size_t)n * E;
    for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        const int r = e < E ? ri[e] : -1;
        const bool ok = r >= 0 && r < p.P;
        const unsigned grp = __match_any_sync(0xffffffffu, ok ? r : -1);
        if (ok) list[cnt[r] + __popc(grp & below)] = e;
        __syncwarp();
        if (ok && (grp & below) == 0u) cnt[r] += __popc(grp);
        __syncwarp();
    }
}

// ----------------------------------------------------------------------------- query side

// Shared memory of the query kernel: Q and dO tiles (nw*16 rows), K and V tiles (L
// rounded up to 32 rows), the routed regions, the per-chunk key masks.
__host__ __device__ inline int bwd_tc_query_smem(int nw, int L, int topk) {
    const int Lp = (L + 31) & ~31;
    return 2 * nw * 16 * 64 + 2 * Lp * 64 + topk * 4 + (Lp / 32) * 4 + 128;
}

__global__ void __launch_bounds__(32 * kBwdTcMaxWarps) bwd_tc_query_kernel(const BwdTcParams p) {
    extern __shared__ __align__(128) unsigned char tc_q_s[];
    const int unit = blockIdx.x;
    uint32_t m_, pr_;
    const int npr = (int)p.div_heads.divmod((uint32_t)unit, m_), n = (int)p.div_P.divmod((uint32_t)npr, pr_);
    const int m = (int)m_, pr = (int)pr_;
    const int Rp = p.nw * 16, Lp = (p.L + 31) & ~31, nch = Lp / 32;
    unsigned char *sQ = tc_q_s, *sO = sQ + Rp * 64, *sK = sO + Rp * 64, *sV = sK + Lp * 64;
    int *sRoute = reinterpret_cast<int *>(sV + Lp * 64);
    uint32_t *sMask = reinterpret_cast<uint32_t *>(sRoute + p.topk);
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int c0 = m * 32;
    for (int a = tid; a < p.topk; a += nthr) {
        int r = p.r_idx[(size_t)npr * p.topk + a];
        if (r < 0 || r >= p.P) r = -1;  // flagged by the transpose kernel
        sRoute[a] = r;
    }
    __syncthreads();
    if (tid < 32)  // warp 0: one key per lane, one ballot per 32-key chunk
        for (int w = 0; w < nch; ++w) {
            const int j = w * 32 + tid;
            const bool live = j < p.L && sRoute[p.div_w2.div((uint32_t)j)] >= 0;
            const uint32_t mk = __ballot_sync(0xffffffffu, live);
            if (tid == 0) sMask[w] = mk;
        }
    const uint32_t q_s = smem_u32(sQ), o_s = smem_u32(sO), k_s = smem_u32(sK), v_s = smem_u32(sV);
    for (int i = tid; i < Rp * 2; i += nthr) {  // two 16-byte pieces of a row per step
        const int row = i >> 1, ch = 2 * (i & 1);
        const bool ok = row < p.w2;
        const size_t g = ok ? tc_pix(p, n, pr, row) + c0 + 8 * ch : 0;
        cp_async16_s(q_s + tc_sw64(row, ch), p.q + g, ok);
        cp_async16_s(q_s + tc_sw64(row, ch + 1), p.q + g + 8, ok);
        cp_async16_s(o_s + tc_sw64(row, ch), p.dout + g, ok);
        cp_async16_s(o_s + tc_sw64(row, ch + 1), p.dout + g + 8, ok);
    }
    // two 16-byte pieces of a key row per step: one address for four copies
    for (int i = tid; i < Lp * 2; i += nthr) {
        const int j = i >> 1, ch = 2 * (i & 1);
        const int a = (int)p.div_w2.div((uint32_t)j), t = j - a * p.w2;
        const int r = j < p.L ? sRoute[a] : -1;
        const bool ok = r >= 0;
        const size_t g = ok ? tc_pix(p, n, r, t) + c0 + 8 * ch : 0;
        cp_async16_s(k_s + tc_sw64(j, ch), p.k + g, ok);
        cp_async16_s(k_s + tc_sw64(j, ch + 1), p.k + g + 8, ok);
        cp_async16_s(v_s + tc_sw64(j, ch), p.v + g, ok);
        cp_async16_s(v_s + tc_sw64(j, ch + 1), p.v + g + 8, ok);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, tq = lane & 3, mat = lane >> 3;
    const int r0 = warp * 16;
    uint32_t aq[2][4], ado[2][4];
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        const int row = r0 + (lane & 7) + 8 * (mat & 1), chunk = 2 * kk + (mat >> 1);
        ldsm_x4(aq[kk][0], aq[kk][1], aq[kk][2], aq[kk][3], sQ + tc_sw64(row, chunk));
        ldsm_x4(ado[kk][0], ado[kk][1], ado[kk][2], ado[kk][3], sO + tc_sw64(row, chunk));
    }
    // S (or dA) of the 32-key chunk kc: acc[n-tile][c0..c3], rows g / g + 8, key 8 nt + 2 tq (+1)
    auto chunk_mma = [&](const uint32_t (&af)[2][4], const unsigned char *tile, int kc, float (&acc)[4][4]) {
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
#pragma unroll
            for (int hp = 0; hp < 2; ++hp) {
                const int key = kc * 32 + 16 * hp + (lane & 7) + 8 * (mat >> 1), chunk = 2 * kk + (mat & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(b0, b1, b2, b3, tile + tc_sw64(key, chunk));
                mma_bf16_16816(acc[2 * hp], af[kk], b0, b1);
                mma_bf16_16816(acc[2 * hp + 1], af[kk], b2, b3);
            }
    };
    // scaled logits (base 2) of the chunk, -inf where the key is masked
    auto logits = [&](int kc, float (&s)[4][4]) {
        chunk_mma(aq, sK, kc, s);
        const uint32_t mk = sMask[kc];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                s[nt][e] = ((mk >> (8 * nt + 2 * tq + (e & 1))) & 1u) ? s[nt][e] * p.sl2 : -INFINITY;
    };
    // dQ += dS K over chunk kc (keys as the contraction index), dS = A (dA - D)
    auto dq_chunk = [&](int kc, const float (&a)[4][4], const float (&da)[4][4], const float (&Dr)[2],
                        float (&dq)[4][4]) {
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int nt = 2 * ks + u;
                tc_split(a[nt][0] * (da[nt][0] - Dr[0]), a[nt][1] * (da[nt][1] - Dr[0]), hi[2 * u], lo[2 * u]);
                tc_split(a[nt][2] * (da[nt][2] - Dr[1]), a[nt][3] * (da[nt][3] - Dr[1]), hi[2 * u + 1], lo[2 * u + 1]);
            }
#pragma unroll
            for (int cp2 = 0; cp2 < 2; ++cp2) {
                const int key = kc * 32 + 16 * ks + (lane & 7) + 8 * (mat & 1), chunk = 2 * cp2 + (mat >> 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(b0, b1, b2, b3, sK + tc_sw64(key, chunk));
                mma_bf16_16816(dq[2 * cp2], hi, b0, b1);
                mma_bf16_16816(dq[2 * cp2], lo, b0, b1);
                mma_bf16_16816(dq[2 * cp2 + 1], hi, b2, b3);
                mma_bf16_16816(dq[2 * cp2 + 1], lo, b2, b3);
            }
        }
    };
    float lse[2], D[2], dqa[4][4];
#pragma unroll
    for (int ct = 0; ct < 4; ++ct)
#pragma unroll
        for (int e = 0; e < 4; ++e) dqa[ct][e] = 0.f;
    if (nch <= 2) {
        // at most 64 keys per query: the logits and dA of both chunks stay in registers, the
        // exponentials are taken once relative to the exact row maximum, and D = sum_j A dA
        // is summed from them directly (no O' product)
        float sc[2][4][4], da[2][4][4];
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int kc = 0; kc < 2; ++kc) {
            if (kc >= nch) break;
            logits(kc, sc[kc]);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) mx[h] = fmaxf(mx[h], fmaxf(sc[kc][nt][2 * h], sc[kc][nt][2 * h + 1]));
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
        }
        float sm[2] = {0.f, 0.f};
#pragma unroll
        for (int kc = 0; kc < 2; ++kc) {
            if (kc >= nch) break;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float mr = mx[e >> 1];
                    const float pe = mr == -INFINITY ? 0.f : fast_exp2(sc[kc][nt][e] - mr);
                    sc[kc][nt][e] = pe;
                    sm[e >> 1] += pe;
                }
        }
        float inv[2], dd[2] = {0.f, 0.f};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            sm[h] += __shfl_xor_sync(0xffffffffu, sm[h], 1);
            sm[h] += __shfl_xor_sync(0xffffffffu, sm[h], 2);
            lse[h] = sm[h] > 0.f ? mx[h] + log2f(sm[h]) : INFINITY;  // no valid key: probabilities 0
            inv[h] = sm[h] > 0.f ? 1.0f / sm[h] : 0.f;
        }
#pragma unroll
        for (int kc = 0; kc < 2; ++kc) {
            if (kc >= nch) break;
            chunk_mma(ado, sV, kc, da[kc]);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    sc[kc][nt][e] *= inv[e >> 1];  // A
                    dd[e >> 1] = fmaf(sc[kc][nt][e], da[kc][nt][e], dd[e >> 1]);
                }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            dd[h] += __shfl_xor_sync(0xffffffffu, dd[h], 1);
            dd[h] += __shfl_xor_sync(0xffffffffu, dd[h], 2);
            D[h] = dd[h];
        }
#pragma unroll
        for (int kc = 0; kc < 2; ++kc) {
            if (kc >= nch) break;
            dq_chunk(kc, sc[kc], da[kc], D, dqa);
        }
    } else {
        // pass 1 (online over the chunks): row max m, row sum l and O' = sum_j 2^(s_j - m) v_j
        // (this thread holds rows g (e < 2) and g + 8 (e >= 2)); then D = dO . O' / l, which is
        // sum_j A dA
        float mx[2] = {-INFINITY, -INFINITY}, sm[2] = {0.f, 0.f};
        float oa[4][4];  // O' rows g / g + 8, channels 8 ct + 2 tq (+1)
#pragma unroll
        for (int ct = 0; ct < 4; ++ct)
#pragma unroll
            for (int e = 0; e < 4; ++e) oa[ct][e] = 0.f;
        for (int kc = 0; kc < nch; ++kc) {
            float s[4][4];
            logits(kc, s);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float cm = -INFINITY;
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) cm = fmaxf(cm, fmaxf(s[nt][2 * h], s[nt][2 * h + 1]));
                cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 1));
                cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 2));
                const float mn = fmaxf(mx[h], cm);
                // the rescale of what was summed relative to the old max (0 before any valid key)
                const float f = mn == -INFINITY || mx[h] == -INFINITY ? 0.f : fast_exp2(mx[h] - mn);
                float acc = sm[h] * f;
#pragma unroll
                for (int ct = 0; ct < 4; ++ct) {
                    oa[ct][2 * h] *= f;
                    oa[ct][2 * h + 1] *= f;
                }
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    // 2^(s - m); a masked key (-inf) or a row without a valid key yet gives 0
                    const float p0 = mn == -INFINITY ? 0.f : fast_exp2(s[nt][2 * h] - mn);
                    const float p1 = mn == -INFINITY ? 0.f : fast_exp2(s[nt][2 * h + 1] - mn);
                    s[nt][2 * h] = p0;
                    s[nt][2 * h + 1] = p1;
                    acc += p0 + p1;
                }
                sm[h] = acc;
                mx[h] = mn;
            }
            // O' += P V over this chunk's 32 keys (P as bf16 high + low parts)
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int nt = 2 * ks + u;
                    tc_split(s[nt][0], s[nt][1], hi[2 * u], lo[2 * u]);
                    tc_split(s[nt][2], s[nt][3], hi[2 * u + 1], lo[2 * u + 1]);
                }
#pragma unroll
                for (int cp2 = 0; cp2 < 2; ++cp2) {
                    const int key = kc * 32 + 16 * ks + (lane & 7) + 8 * (mat & 1), chunk = 2 * cp2 + (mat >> 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(b0, b1, b2, b3, sV + tc_sw64(key, chunk));
                    mma_bf16_16816(oa[2 * cp2], hi, b0, b1);
                    mma_bf16_16816(oa[2 * cp2], lo, b0, b1);
                    mma_bf16_16816(oa[2 * cp2 + 1], hi, b2, b3);
                    mma_bf16_16816(oa[2 * cp2 + 1], lo, b2, b3);
                }
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float t = sm[h];
            t += __shfl_xor_sync(0xffffffffu, t, 1);
            t += __shfl_xor_sync(0xffffffffu, t, 2);
            lse[h] = t > 0.f ? mx[h] + log2f(t) : INFINITY;  // no valid key: probabilities 0
            // dO . O' of row g + 8 h, this thread's 8 channels, then the quad
            const int row = r0 + g + 8 * h;
            float dd = 0.f;
#pragma unroll
            for (int ct = 0; ct < 4; ++ct) {
                // channels 8 ct + 2 tq, + 1: 16-byte chunk ct of the row, bytes 4 tq .. 4 tq + 3
                const __nv_bfloat162 d2 = *reinterpret_cast<const __nv_bfloat162 *>(sO + tc_sw64(row, ct) + 4 * tq);
                const float2 df = __bfloat1622float2(d2);
                dd = fmaf(df.x, oa[ct][2 * h], fmaf(df.y, oa[ct][2 * h + 1], dd));
            }
            dd += __shfl_xor_sync(0xffffffffu, dd, 1);
            dd += __shfl_xor_sync(0xffffffffu, dd, 2);
            D[h] = t > 0.f ? dd / t : 0.f;
        }
        // probabilities and dA of chunk kc
        auto probs = [&](int kc, float (&a)[4][4], float (&da)[4][4]) {
            logits(kc, a);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) a[nt][e] = fast_exp2(a[nt][e] - lse[e >> 1]);
            chunk_mma(ado, sV, kc, da);
        };
        // pass 2: dS and dQ += dS K (keys as the contraction index)
        for (int kc = 0; kc < nch; ++kc) {
            float a[4][4], da[4][4];
            probs(kc, a, da);
            dq_chunk(kc, a, da, D, dqa);
        }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int row = r0 + g + 8 * h;
        if (row >= p.w2) continue;
        float *dst = p.dq + tc_pix(p, n, pr, row) + c0;
#pragma unroll
        for (int ct = 0; ct < 4; ++ct)
            *reinterpret_cast<float2 *>(dst + 8 * ct + 2 * tq) =
                make_float2(p.scale * dqa[ct][2 * h], p.scale * dqa[ct][2 * h + 1]);
        if (tq == 0)
            *reinterpret_cast<float2 *>(p.stats + (((size_t)npr * p.heads + m) * p.w2 + row) * 2) =
                make_float2(lse[h], D[h]);
    }
}

// ----------------------------------------------------------------------------- key side

// Shared memory of the key kernel: K and V tiles (nw*16 rows), two stages of the
// entry's Q and dO tiles (Rp = w2 rounded up to 16 rows) and its per-query (lse, D).
__host__ __device__ inline int bwd_tc_key_smem(int nw, int w2) {
    const int Rp = (w2 + 15) & ~15;
    return 2 * nw * 16 * 64 + 2 * (2 * Rp * 64 + Rp * 8) + nw * 16 * 128 + 128;
}

__global__ void __launch_bounds__(32 * kBwdTcMaxWarps) bwd_tc_key_kernel(const BwdTcParams p) {
    extern __shared__ __align__(128) unsigned char tc_k_s[];
    const int unit = blockIdx.x;
    uint32_t m_, pk_;
    const int npk = (int)p.div_heads.divmod((uint32_t)unit, m_), n = (int)p.div_P.divmod((uint32_t)npk, pk_);
    const int m = (int)m_, pk = (int)pk_;
    const int Kp = p.nw * 16, Rp = (p.w2 + 15) & ~15;
    unsigned char *sK = tc_k_s, *sV = sK + Kp * 64, *stage0 = sV + Kp * 64;
    const int stage_bytes = 2 * Rp * 64 + Rp * 8;
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int c0 = m * 32;
    const int *off = p.kv_off + (size_t)n * (p.P + 1);
    const int e0 = off[pk], cnt = off[pk + 1] - e0;
    const int *list = p.kv_list + (size_t)n * p.P * p.topk + e0;
    const uint32_t k_s = smem_u32(sK), v_s = smem_u32(sV);
    for (int i = tid; i < Kp * 2; i += nthr) {  // two 16-byte pieces of a row per step
        const int row = i >> 1, ch = 2 * (i & 1);
        const bool ok = row < p.w2;
        const size_t g = ok ? tc_pix(p, n, pk, row) + c0 + 8 * ch : 0;
        cp_async16_s(k_s + tc_sw64(row, ch), p.k + g, ok);
        cp_async16_s(k_s + tc_sw64(row, ch + 1), p.k + g + 8, ok);
        cp_async16_s(v_s + tc_sw64(row, ch), p.v + g, ok);
        cp_async16_s(v_s + tc_sw64(row, ch + 1), p.v + g + 8, ok);
    }
    // the LCE part of dv already stored for these keys (nw * 16 rows of 32 floats after the
    // two entry stages), copied now and added to the attention part at the end
    const uint32_t l_s = smem_u32(stage0 + 2 * stage_bytes);
    for (int i = tid; i < Kp * 2; i += nthr) {  // four 16-byte pieces of a row per step
        const int row = i >> 1, ch = 4 * (i & 1);
        const bool ok = row < p.w2;
        const size_t g = ok ? tc_pix(p, n, pk, row) + c0 + 4 * ch : 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) cp_async16_s(l_s + row * 128 + (ch + u) * 16, p.dv + g + 4 * u, ok);
    }
    // the entry's queries (query region pr): Q and dO rows, (lse, D) per row, all as
    // asynchronous copies (padding rows: lse = +inf, D = 0, written directly)
    auto load_entry = [&](int pr, int s) {
        unsigned char *st = stage0 + s * stage_bytes;
        const uint32_t sq = smem_u32(st), so = sq + Rp * 64;
        float2 *sst = reinterpret_cast<float2 *>(st + 2 * Rp * 64);
        for (int i = tid; i < Rp * 2; i += nthr) {  // two 16-byte pieces of a row per step
            const int row = i >> 1, ch = 2 * (i & 1);
            const bool ok = row < p.w2;
            const size_t g = ok ? tc_pix(p, n, pr, row) + c0 + 8 * ch : 0;
            cp_async16_s(sq + tc_sw64(row, ch), p.q + g, ok);
            cp_async16_s(sq + tc_sw64(row, ch + 1), p.q + g + 8, ok);
            cp_async16_s(so + tc_sw64(row, ch), p.dout + g, ok);
            cp_async16_s(so + tc_sw64(row, ch + 1), p.dout + g + 8, ok);
        }
        for (int row = tid; row < Rp; row += nthr) {
            if (row < p.w2)
                tc_cp_async8(smem_u32(sst + row), p.stats + ((((size_t)n * p.P + pr) * p.heads + m) * p.w2 + row) * 2);
            else
                sst[row] = make_float2(INFINITY, 0.f);
        }
    };
    // the query region of entry idx + 1 is read one entry ahead, so that its load overlaps
    // the current entry's work instead of stalling the next copies
    int pr_next = cnt > 0 ? (int)p.div_topk.div((uint32_t)list[0]) : 0;
    if (cnt > 0) load_entry(pr_next, 0);
    pr_next = cnt > 1 ? (int)p.div_topk.div((uint32_t)list[1]) : 0;
    cp_async_commit();

    const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, tq = lane & 3, mat = lane >> 3;
    const int k0 = warp * 16;
    float dka[4][4], dva[4][4];
#pragma unroll
    for (int ct = 0; ct < 4; ++ct)
#pragma unroll
        for (int e = 0; e < 4; ++e) dka[ct][e] = dva[ct][e] = 0.f;
    uint32_t ak[2][4], av[2][4];
    for (int idx = 0; idx < cnt; ++idx) {
        if (idx + 1 < cnt) load_entry(pr_next, (idx + 1) & 1);  // the other stage is free
        const int pr_after = idx + 2 < cnt ? (int)p.div_topk.div((uint32_t)list[idx + 2]) : 0;
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        if (idx == 0) {
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                const int row = k0 + (lane & 7) + 8 * (mat & 1), chunk = 2 * kk + (mat >> 1);
                ldsm_x4(ak[kk][0], ak[kk][1], ak[kk][2], ak[kk][3], sK + tc_sw64(row, chunk));
                ldsm_x4(av[kk][0], av[kk][1], av[kk][2], av[kk][3], sV + tc_sw64(row, chunk));
            }
        }
        pr_next = pr_after;
        const unsigned char *sQ = stage0 + (idx & 1) * stage_bytes, *sO = sQ + Rp * 64;
        const float2 *sst = reinterpret_cast<const float2 *>(sQ + 2 * Rp * 64);
        for (int qc = 0; qc < Rp / 16; ++qc) {
            // S^T and dA^T of these 16 keys x 16 queries: rows = keys g / g + 8, columns =
            // queries 16 qc + 8 nt + 2 tq (+1)
            float sT[2][4], dT[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) sT[nt][e] = dT[nt][e] = 0.f;
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                const int row = qc * 16 + (lane & 7) + 8 * (mat >> 1), chunk = 2 * kk + (mat & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(b0, b1, b2, b3, sQ + tc_sw64(row, chunk));
                mma_bf16_16816(sT[0], ak[kk], b0, b1);
                mma_bf16_16816(sT[1], ak[kk], b2, b3);
                ldsm_x4(b0, b1, b2, b3, sO + tc_sw64(row, chunk));
                mma_bf16_16816(dT[0], av[kk], b0, b1);
                mma_bf16_16816(dT[1], av[kk], b2, b3);
            }
            uint32_t dh[4], dl[4], ah[4], al[4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const float2 st0 = sst[qc * 16 + 8 * nt + 2 * tq], st1 = sst[qc * 16 + 8 * nt + 2 * tq + 1];
                float a[4], ds[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 st = (e & 1) ? st1 : st0;
                    a[e] = fast_exp2(sT[nt][e] * p.sl2 - st.x);
                    ds[e] = a[e] * (dT[nt][e] - st.y);
                }
                // A fragments (keys x queries, k = queries): this tile's columns are k 8 nt + 2 tq
                tc_split(ds[0], ds[1], dh[2 * nt], dl[2 * nt]);
                tc_split(ds[2], ds[3], dh[2 * nt + 1], dl[2 * nt + 1]);
                tc_split(a[0], a[1], ah[2 * nt], al[2 * nt]);
                tc_split(a[2], a[3], ah[2 * nt + 1], al[2 * nt + 1]);
            }
#pragma unroll
            for (int cp2 = 0; cp2 < 2; ++cp2) {
                const int row = qc * 16 + (lane & 7) + 8 * (mat & 1), chunk = 2 * cp2 + (mat >> 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(b0, b1, b2, b3, sQ + tc_sw64(row, chunk));
                mma_bf16_16816(dka[2 * cp2], dh, b0, b1);
                mma_bf16_16816(dka[2 * cp2], dl, b0, b1);
                mma_bf16_16816(dka[2 * cp2 + 1], dh, b2, b3);
                mma_bf16_16816(dka[2 * cp2 + 1], dl, b2, b3);
                ldsm_x4_t(b0, b1, b2, b3, sO + tc_sw64(row, chunk));
                mma_bf16_16816(dva[2 * cp2], ah, b0, b1);
                mma_bf16_16816(dva[2 * cp2], al, b0, b1);
                mma_bf16_16816(dva[2 * cp2 + 1], ah, b2, b3);
                mma_bf16_16816(dva[2 * cp2 + 1], al, b2, b3);
            }
        }
        __syncthreads();  // the stage is read: the next prefetch may overwrite it
    }
    cp_async_wait<0>();
    __syncthreads();  // every thread's copy of the LCE part has landed
    const float *sL = reinterpret_cast<const float *>(stage0 + 2 * stage_bytes);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int row = k0 + g + 8 * h;
        if (row >= p.w2) continue;
        const size_t o = tc_pix(p, n, pk, row) + c0;
#pragma unroll
        for (int ct = 0; ct < 4; ++ct) {
            const int c = 8 * ct + 2 * tq;
            *reinterpret_cast<float2 *>(p.dk + o + c) = make_float2(p.scale * dka[ct][2 * h], p.scale * dka[ct][2 * h + 1]);
            const float2 lce = *reinterpret_cast<const float2 *>(sL + row * 32 + c);
            *reinterpret_cast<float2 *>(p.dv + o + c) = make_float2(lce.x + dva[ct][2 * h], lce.y + dva[ct][2 * h + 1]);
        }
    }
}

// ----------------------------------------------------------------------------- LCE gradients

// The LCE term out[y,x,c] += b[c] + sum_{a,b} w[c][a][b] V[y+a-2, x+b-2, c] (zero outside) gives
//   dv[y,x,c]   = sum_{a,b} w[c][a][b] dout[y-a+2, x-b+2, c]      (the LCE part of dv)
//   dw[c][a][b] = sum_{n,y,x} dout[n,y,x,c] V[n, y+a-2, x+b-2, c],  db[c] = sum dout[..., c].
// bwd_tc_lce_kernel: tiles of kLceTH x kLceTW pixels and a group of PG <= kLceGroup channel
// pairs (PG divides the pairs); the CTA stages the tile's dout and V with a 2-pixel zero
// border (bf16 pairs, 16-byte cp.async pieces coalesced across channels, the next tile's in
// flight while this one is summed), thread = (channel pair, slot), slot = a row segment of
// the tile that the thread walks left to right with a 5 x 5 window of the staging in
// registers (one new column of five values per pixel). Each thread writes the dv of its
// pixels and keeps the 25 dw taps and db of its channel pair in registers over every tile
// of its CTA; CTA (g, j) takes the tiles j, j + G, ... of channel group g, in that order.
// The slots then meet in shared memory and the CTA writes its partial sums;
// bwd_tc_lce_final_kernel adds the G partials of each (channel, tap) with one warp, in a
// fixed order (lane stride, then a shuffle tree): no atomics, the same bits every call.
constexpr int kLceTH = 4, kLceTW = 16, kLceGroup = 64, kLceThreads = 256;

// Two stages of the staged tile (bf16 pairs of dout and of V), and after the last tile the
// per-thread partial sums (the same memory).
__host__ __device__ inline int bwd_tc_lce_smem(int pairs_g) {
    const int stage = 2 * 2 * (kLceTH + 4) * (kLceTW + 4) * pairs_g * 4, red = kLceThreads * 52 * 4;
    return stage > red ? stage : red;
}

// PG: channel pairs of the group (16, 32, 48 or 64), a constant so that every tap's shared
// address is the thread's base plus an immediate offset.
template <int PG>
__global__ void __launch_bounds__(kLceThreads) bwd_tc_lce_kernel(const BwdTcParams p, const __nv_bfloat16 *lce_w,
                                                                 float *part, int G) {
    extern __shared__ __align__(16) uint32_t lce_s[];
    const int pairs = p.C >> 1;
    const int g = blockIdx.x / G, j0 = blockIdx.x - g * G;
    constexpr int pg = PG;
    const int cp0 = g * pg;  // the group's first channel pair
    constexpr int HW = (kLceTH + 4) * (kLceTW + 4);
    float *red = reinterpret_cast<float *>(lce_s);  // [threads][52], over the staging after the tiles
    constexpr int slots = kLceThreads / pg;
    // slot = (row of the tile, segment of that row): kParts segments of kSeg pixels per row
    constexpr int SW = kLceTW + 4, kParts = slots / kLceTH, kSeg = kLceTW / kParts;
    static_assert(kParts >= 1 && kLceTW % kParts == 0, "tile rows and segments must cover the slots");
    const int cpl = threadIdx.x % pg, slot = threadIdx.x / pg;
    const bool active = slot < kLceTH * kParts;
    const int cp = cp0 + cpl, c = 2 * cp;
    float2 w[25];
#pragma unroll
    for (int t = 0; t < 25; ++t)
        w[t] = active ? make_float2(__bfloat162float(lce_w[c * 25 + t]), __bfloat162float(lce_w[(c + 1) * 25 + t]))
                      : make_float2(0.f, 0.f);
    float2 dw[25], db = make_float2(0.f, 0.f);
#pragma unroll
    for (int t = 0; t < 25; ++t) dw[t] = make_float2(0.f, 0.f);
    const int nrb = (p.H + kLceTH - 1) / kLceTH, ncb = (p.W + kLceTW - 1) / kLceTW;
    const int tiles = p.N * nrb * ncb;
    const uint4 *dout16 = reinterpret_cast<const uint4 *>(p.dout);  // 4 channel pairs per 16 bytes
    const uint4 *v16 = reinterpret_cast<const uint4 *>(p.v);
    constexpr int pg4 = pg >> 2;
    const int pairs4 = pairs >> 2;
    // stage st: dout pairs [HW][pg] at lce_s + st * 2 * HW * pg, then V's
    auto issue = [&](int tile, int st) {
        const int n = tile / (nrb * ncb), rc = tile - n * nrb * ncb, rb = rc / ncb, cb = rc - rb * ncb;
        const int y0 = rb * kLceTH, x0 = cb * kLceTW;
        uint32_t *sD = lce_s + st * 2 * HW * pg, *sV = sD + HW * pg;
        for (int i = threadIdx.x; i < HW * pg4; i += kLceThreads) {
            const int px = i / pg4, q4 = i - px * pg4;
            const int hy = px / SW, hx = px - hy * SW;
            const int y = y0 + hy - 2, x = x0 + hx - 2;
            const bool ok = y >= 0 && y < p.H && x >= 0 && x < p.W;  // outside: zero fill
            const size_t o = ok ? (((size_t)n * p.H + y) * p.W + x) * pairs4 + (cp0 >> 2) + q4 : 0;
            cp_async16(sD + px * pg + 4 * q4, dout16 + o, ok);
            cp_async16(sV + px * pg + 4 * q4, v16 + o, ok);
        }
        cp_async_commit();
    };
    // tiles j0, j0 + G, ...: the next tile's copies are in flight while this one is summed
    if (j0 < tiles) issue(j0, 0);
    int k = 0;
    for (int tile = j0; tile < tiles; tile += G, ++k) {
        const int st = k & 1;
        if (tile + G < tiles) {
            issue(tile + G, st ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();  // every thread's copies of this tile have landed
        const int n = tile / (nrb * ncb), rc = tile - n * nrb * ncb, rb = rc / ncb, cb = rc - rb * ncb;
        const int y0 = rb * kLceTH, x0 = cb * kLceTW;
        // slot = (row of the tile, segment of that row); the slot walks its segment left to
        // right with a 5 x 5 window in registers, first of V (for dw and db), then of dout
        // (for dv): each step loads one new column of five values instead of all 25 taps.
        // Staged (hy, hx) is pixel (y0 + hy - 2, x0 + hx - 2), so the window of pixel
        // (ly, lx) is rows ly .. ly + 4, columns lx .. lx + 4 of the staging.
        const int ly = slot % kLceTH, xs = (slot / kLceTH) * kSeg;
        if (active && y0 + ly < p.H) {
            const uint32_t *sD = lce_s + st * 2 * HW * pg, *sV = sD + HW * pg;
            const uint32_t *vw = sV + (ly * SW + xs) * pg + cpl;             // V window origin
            const uint32_t *dw0 = sD + (ly * SW + xs) * pg + cpl;            // dout window origin
            const uint32_t *dc = sD + ((ly + 2) * SW + xs + 2) * pg + cpl;   // dout at the pixel
            float2 win[5][5];
#pragma unroll
            for (int a = 0; a < 5; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) win[a][b] = bf16x2_to_float2(vw[(a * SW + b) * pg]);
#pragma unroll
            for (int i = 0; i < kSeg; ++i) {
#pragma unroll
                for (int a = 0; a < 5; ++a) win[a][(i + 4) % 5] = bf16x2_to_float2(vw[(a * SW + i + 4) * pg]);
                if (x0 + xs + i < p.W) {
                    const float2 d = bf16x2_to_float2(dc[i * pg]);
                    db.x += d.x;
                    db.y += d.y;
#pragma unroll
                    for (int a = 0; a < 5; ++a)
#pragma unroll
                        for (int b = 0; b < 5; ++b) dw[a * 5 + b] = ffma2(d, win[a][(i + b) % 5], dw[a * 5 + b]);
                }
            }
            // dv(y, x) = sum_{a,b} w[a][b] dout(y - a + 2, x - b + 2): dout at window (4 - a, 4 - b)
#pragma unroll
            for (int a = 0; a < 5; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) win[a][b] = bf16x2_to_float2(dw0[(a * SW + b) * pg]);
            float2 *dvp = reinterpret_cast<float2 *>(p.dv + (((size_t)n * p.H + y0 + ly) * p.W + x0 + xs) * p.C + c);
#pragma unroll
            for (int i = 0; i < kSeg; ++i) {
#pragma unroll
                for (int a = 0; a < 5; ++a) win[a][(i + 4) % 5] = bf16x2_to_float2(dw0[(a * SW + i + 4) * pg]);
                if (x0 + xs + i < p.W) {
                    float2 acc[5];  // one chain per window row, summed at the end
#pragma unroll
                    for (int a = 0; a < 5; ++a) {
                        acc[a] = make_float2(0.f, 0.f);
#pragma unroll
                        for (int b = 0; b < 5; ++b) acc[a] = ffma2(w[a * 5 + b], win[4 - a][(i + 4 - b) % 5], acc[a]);
                    }
                    dvp[(size_t)i * pairs] = make_float2(((acc[0].x + acc[1].x) + (acc[2].x + acc[3].x)) + acc[4].x,
                                                         ((acc[0].y + acc[1].y) + (acc[2].y + acc[3].y)) + acc[4].y);
                }
            }
        }
        __syncthreads();  // this stage is read: the copies of tile k + 2 may overwrite it
    }
    // the slots of a channel pair meet in shared memory, then the CTA writes its partial
    __syncthreads();  // every thread is done with the staged tile
    float *mine = red + threadIdx.x * 52;
#pragma unroll
    for (int t = 0; t < 25; ++t) {
        mine[2 * t] = dw[t].x;
        mine[2 * t + 1] = dw[t].y;
    }
    mine[50] = db.x;
    mine[51] = db.y;
    __syncthreads();
    float *dst = part + (size_t)blockIdx.x * kLceGroup * 2 * 26;  // [pairs of the group][2][26]
    for (int i = threadIdx.x; i < pg * 52; i += kLceThreads) {
        const int q = i / 52, e = i - q * 52;  // e: tap * 2 + channel, or 50 / 51 for db
        float s2 = 0.f;
        for (int sl = 0; sl < slots; ++sl) s2 += red[(sl * pg + q) * 52 + e];
        const int ch = e & 1, tap = e >> 1;  // tap 25 = db
        dst[(q * 2 + ch) * 26 + tap] = s2;
    }
}

// dw[c][t] (t < 25) and db[c] (t = 25): one warp per (c, t) adds the G partials of c's group
// (groups of pg channel pairs; each CTA's partials sit in a block of kLceGroup pairs).
__global__ void __launch_bounds__(256) bwd_tc_lce_final_kernel(const float *part, int G, int C, int pg, float *dw,
                                                                float *db) {
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (gw >= C * 26) return;
    const int c = gw / 26, t = gw - c * 26;
    const int cp = c >> 1, g = cp / pg, ql = (cp - g * pg) * 2 + (c & 1);
    float s = 0.f;
    for (int j = lane; j < G; j += 32) s += part[((size_t)(g * G + j) * kLceGroup * 2 + ql) * 26 + t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) {
        if (t < 25)
            dw[c * 25 + t] = s;
        else
            db[c] = s;
    }
}

}  // namespace bra
