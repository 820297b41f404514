// attn.cuh — steps 4-5 of BRA: token-to-token attention over the routed regions,
// with the LCE depthwise 5x5 convolution of V fused into the epilogue.
//
// Follows the BRA walk-through on "BiFormer ... 前向传播过程" (niftyadmin), section
// "BRA模块": kv_gather collects the topk routed regions' K/V tokens (eq. 6), each
// query attends per head over all topk*w2 gathered keys jointly, attn_act being a
// softmax over the last dimension (eq. 7), and lepe = Conv2d(C, C, 5, pad 2,
// groups=C) of the un-patchified V is added to the re-assembled output (eq. 7,
// LCE(V)).
//
// Work split: one CTA per (image n, query region p, block of RB region rows, group of
// HG heads). The gathered keys are never materialised in global memory: each CTA
// streams them, KC tokens at a time, straight from the (N,H,W,C) K and V maps into
// shared memory (16-byte cp.async, double-buffered), reading the region index of
// every key from the routing.
#pragma once

#include "common.cuh"

namespace bra {

struct AttnParams {
    const void *q, *k, *v, *lce_w, *lce_b;
    void *out;
    const int32_t *r_idx;
    int *err_flag;  // optional: set to 1 when a region index is out of range
    int N, H, W, C, heads, S, topk;
    int hr, wr, w2, P;
    int RB;    // region rows per CTA
    int HG;    // heads per CTA
    int QT;    // 16-row query tiles per CTA (tensor-core kernel)
    int n_rb;  // hr / RB
    int n_hg;  // heads / HG
    int stages;        // K/V chunk buffers (1 or 2)
    float scale_log2;  // d^-0.5 * log2(e)
};

__host__ __device__ constexpr int align16(int b) { return (b + 15) & ~15; }

// ----------------------------------------------------------------------------- shared pieces

// Region indices of this (n, p) into shared memory; an index outside [0, P) becomes -1
// and raises the error flag. Returns true if any index was bad.
__device__ inline bool load_route(const AttnParams &prm, int n, int p, int *sIdx) {
    int bad = 0;
    for (int a = threadIdx.x; a < prm.topk; a += blockDim.x) {
        int r = __ldg(prm.r_idx + ((size_t)n * prm.P + p) * prm.topk + a);
        if (r < 0 || r >= prm.P) {
            r = -1;
            bad = 1;
        }
        sIdx[a] = r;
    }
    bad = __syncthreads_or(bad);
    if (bad && threadIdx.x == 0 && prm.err_flag) atomicExch(prm.err_flag, 1);
    return bad != 0;
}

// Copy keys [k0, k0+KC) of the gathered list (routed regions in r_idx order, tokens
// row-major inside each) into sK/sV rows of `ld` elements; keys past the end or in a
// bad region are zero-filled. Channels [c0, c0+CH).
template <typename T>
__device__ inline void load_kv_chunk(const AttnParams &prm, const T *__restrict__ kg,
                                     const T *__restrict__ vg, const int *sIdx, int n, int k0,
                                     int KC, int c0, int CH, int ld, T *sK, T *sV) {
    constexpr int V = Elem<T>::kVec;
    const int pieces = CH / V;
    const int L = prm.topk * prm.w2;
    const size_t img = (size_t)n * prm.H * prm.W;
    for (int idx = threadIdx.x; idx < KC * pieces; idx += blockDim.x) {
        const int row = idx / pieces, pc = idx - row * pieces;
        const int key = k0 + row;
        bool ok = key < L;
        size_t off = 0;
        if (ok) {
            const int a = key / prm.w2, t = key - a * prm.w2;
            const int p2 = sIdx[a];
            ok = p2 >= 0;
            if (ok) {
                const int j2 = p2 / prm.S, i2 = p2 - j2 * prm.S;
                const int th = t / prm.wr, tw = t - th * prm.wr;
                off = ((img + (size_t)(j2 * prm.hr + th) * prm.W + (i2 * prm.wr + tw)) * prm.C) + c0 +
                      pc * V;
            }
        }
        cp_async16(sK + row * ld + pc * V, kg + off, ok);
        cp_async16(sV + row * ld + pc * V, vg + off, ok);
    }
}

// V pixels rows y0-2 .. y0+RB+1, columns x0-2 .. x0+wr+1, channels [c0, c0+CH),
// zero outside the image: the 2-pixel halo that the 5x5 LCE of the CTA's outputs reads.
template <typename T>
__device__ inline void load_halo(const AttnParams &prm, const T *__restrict__ vg, int n, int y0,
                                 int x0, int c0, int CH, T *sHalo) {
    constexpr int V = Elem<T>::kVec;
    const int pieces = CH / V;
    const int hw = prm.wr + 4, hh = prm.RB + 4;
    const size_t img = (size_t)n * prm.H * prm.W;
    for (int idx = threadIdx.x; idx < hh * hw * pieces; idx += blockDim.x) {
        const int pix = idx / pieces, pc = idx - pix * pieces;
        const int hy = pix / hw, hx = pix - hy * hw;
        const int y = y0 - 2 + hy, x = x0 - 2 + hx;
        const bool ok = y >= 0 && y < prm.H && x >= 0 && x < prm.W;
        const size_t off = ok ? ((img + (size_t)y * prm.W + x) * prm.C + c0 + pc * V) : 0;
        cp_async16(sHalo + pix * CH + pc * V, vg + off, ok);
    }
}

// out = O + lce_b + sum_{a,b} lce_w[c][a][b] * V[y+a-2][x+b-2][c] for the CTA's
// RB x wr pixels and CH channels. O is float32 in shared memory, [token][o_ld];
// the V halo is in shared memory. One thread handles a channel pair of one pixel
// column and slides a 5x5 register window down the RB rows.
template <typename T>
__device__ inline void lce_epilogue(const AttnParams &prm, const float *sO, int o_ld,
                                    const T *sHalo, int n, int y0, int x0, int c0, int CH) {
    const T *__restrict__ wg = static_cast<const T *>(prm.lce_w);
    const T *__restrict__ bg = static_cast<const T *>(prm.lce_b);
    T *__restrict__ og = static_cast<T *>(prm.out);
    const int npairs = CH / 2, wr = prm.wr, hw = wr + 4;
    for (int item = threadIdx.x; item < npairs * wr; item += blockDim.x) {
        const int cp = item % npairs, xx = item / npairs;
        const int c = c0 + 2 * cp;
        float w0[25], w1[25];
#pragma unroll
        for (int t = 0; t < 25; ++t) {
            w0[t] = Elem<T>::to_f(wg[(size_t)c * 25 + t]);
            w1[t] = Elem<T>::to_f(wg[(size_t)(c + 1) * 25 + t]);
        }
        const float b0 = Elem<T>::to_f(bg[c]), b1 = Elem<T>::to_f(bg[c + 1]);
        float2 win[5][5];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 5; ++b) win[a + 1][b] = Elem<T>::load2(sHalo + (a * hw + xx + b) * CH + 2 * cp);
        for (int r = 0; r < prm.RB; ++r) {
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 5; ++b) win[a][b] = win[a + 1][b];
#pragma unroll
            for (int b = 0; b < 5; ++b) win[4][b] = Elem<T>::load2(sHalo + ((r + 4) * hw + xx + b) * CH + 2 * cp);
            float a0 = b0, a1 = b1;
#pragma unroll
            for (int a = 0; a < 5; ++a)
#pragma unroll
                for (int b = 0; b < 5; ++b) {
                    a0 = fmaf(w0[a * 5 + b], win[a][b].x, a0);
                    a1 = fmaf(w1[a * 5 + b], win[a][b].y, a1);
                }
            const float2 o = *reinterpret_cast<const float2 *>(sO + (r * wr + xx) * o_ld + 2 * cp);
            const size_t gi = (((size_t)n * prm.H + y0 + r) * prm.W + x0 + xx) * prm.C + c;
            Elem<T>::store2(og + gi, o.x + a0, o.y + a1);
        }
    }
}

// ----------------------------------------------------------------------------- bf16, tensor cores

constexpr int kKC = 64;  // keys per chunk

struct Bf16Smem {
    int idx, q, halo, kv, total;
    int ld;    // row pitch of Q/K/V tiles (elements)
    int o_ld;  // row pitch of the float32 O tile
};

__host__ __device__ inline Bf16Smem bf16_smem_layout(int topk, int QT, int RB, int wr, int CH,
                                                     int stages) {
    Bf16Smem s;
    s.ld = CH + 8;
    s.o_ld = CH + 4;
    s.idx = 0;
    s.q = align16(topk * 4);
    s.halo = s.q + align16(QT * 16 * s.ld * 2);
    s.kv = s.halo + align16((RB + 4) * (wr + 4) * CH * 2);
    int kv_bytes = stages * 2 * kKC * s.ld * 2;
    const int o_bytes = QT * 16 * s.o_ld * 4;
    if (o_bytes > kv_bytes) kv_bytes = o_bytes;
    s.total = s.kv + align16(kv_bytes);
    return s;
}

// Each warp owns one (head, 16-query tile): S = Q K^T and O += P V with
// mma.sync m16n8k16 (bf16 in, fp32 accumulate), online softmax in fp32 registers.
template <int D>
__global__ void __launch_bounds__(256)
attn_bf16_kernel(const AttnParams prm) {
    using T = __nv_bfloat16;
    extern __shared__ __align__(16) unsigned char smem[];
    const int CH = prm.HG * D;
    const Bf16Smem L = bf16_smem_layout(prm.topk, prm.QT, prm.RB, prm.wr, CH, prm.stages);
    int *sIdx = reinterpret_cast<int *>(smem + L.idx);
    T *sQ = reinterpret_cast<T *>(smem + L.q);
    T *sHalo = reinterpret_cast<T *>(smem + L.halo);
    T *sKV = reinterpret_cast<T *>(smem + L.kv);
    float *sO = reinterpret_cast<float *>(smem + L.kv);  // reused after the key loop

    int bid = blockIdx.x;
    const int hg = bid % prm.n_hg;
    bid /= prm.n_hg;
    const int rb = bid % prm.n_rb;
    bid /= prm.n_rb;
    const int p = bid % prm.P, n = bid / prm.P;
    const int j = p / prm.S, i = p - j * prm.S;
    const int y0 = j * prm.hr + rb * prm.RB, x0 = i * prm.wr;
    const int c0 = hg * CH;
    const int nq = prm.RB * prm.wr;
    const T *qg = static_cast<const T *>(prm.q);
    const T *kg = static_cast<const T *>(prm.k);
    const T *vg = static_cast<const T *>(prm.v);

    const bool bad = load_route(prm, n, p, sIdx);

    // group 0: Q tile, V halo, key chunk 0
    {
        constexpr int V = Elem<T>::kVec;
        const int pieces = CH / V;
        for (int idx = threadIdx.x; idx < prm.QT * 16 * pieces; idx += blockDim.x) {
            const int row = idx / pieces, pc = idx - row * pieces;
            const bool ok = row < nq;
            const int th = row / prm.wr, tw = row - th * prm.wr;
            const size_t off =
                ok ? (((size_t)n * prm.H + y0 + th) * prm.W + x0 + tw) * prm.C + c0 + pc * V : 0;
            cp_async16(sQ + row * L.ld + pc * V, qg + off, ok);
        }
    }
    load_halo<T>(prm, vg, n, y0, x0, c0, CH, sHalo);
    const int stage_elems = 2 * kKC * L.ld;
    load_kv_chunk<T>(prm, kg, vg, sIdx, n, 0, kKC, c0, CH, L.ld, sKV, sKV + kKC * L.ld);
    cp_async_commit();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hl = warp / prm.QT, mt = warp - hl * prm.QT;
    const int Lk = prm.topk * prm.w2;
    const int nchunks = (Lk + kKC - 1) / kKC;
    const bool need_mask = bad || (Lk % kKC) != 0;

    uint32_t qa[D / 16][4];
    float m_i[2] = {-INFINITY, -INFINITY}, l_i[2] = {0.f, 0.f};
    float acc[D / 8][4];
#pragma unroll
    for (int t = 0; t < D / 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

    for (int ch = 0; ch < nchunks; ++ch) {
        if (ch + 1 < nchunks) {
            T *nb = sKV + ((ch + 1) % prm.stages) * stage_elems;
            load_kv_chunk<T>(prm, kg, vg, sIdx, n, (ch + 1) * kKC, kKC, c0, CH, L.ld, nb, nb + kKC * L.ld);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const T *sK = sKV + (ch % prm.stages) * stage_elems;
        const T *sV = sK + kKC * L.ld;
        if (ch == 0) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int row = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int col = hl * D + kk * 16 + ((lane >> 4) & 1) * 8;
                ldsm_x4(qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], sQ + row * L.ld + col);
            }
        }
        // S = Q K^T for 16 queries x KC keys
        float s[kKC / 8][4];
#pragma unroll
        for (int t = 0; t < kKC / 8; ++t) s[t][0] = s[t][1] = s[t][2] = s[t][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
            for (int np = 0; np < kKC / 16; ++np) {
                uint32_t b0, b1, b2, b3;
                const int key = np * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
                const int col = hl * D + kk * 16 + ((lane >> 3) & 1) * 8;
                ldsm_x4(b0, b1, b2, b3, sK + key * L.ld + col);
                mma_bf16_16816(s[2 * np], qa[kk], b0, b1);
                mma_bf16_16816(s[2 * np + 1], qa[kk], b2, b3);
            }
        // scale into the log2 domain, mask keys past the end / in bad regions
        float rmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int t = 0; t < kKC / 8; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float x = s[t][e] * prm.scale_log2;
                if (need_mask) {
                    const int key = ch * kKC + t * 8 + 2 * (lane & 3) + (e & 1);
                    const bool ok = key < Lk && sIdx[key / prm.w2] >= 0;
                    if (!ok) x = -INFINITY;
                }
                s[t][e] = x;
                rmax[e >> 1] = fmaxf(rmax[e >> 1], x);
            }
        float alpha[2], mref[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            rmax[r] = fmaxf(rmax[r], __shfl_xor_sync(0xffffffffu, rmax[r], 1));
            rmax[r] = fmaxf(rmax[r], __shfl_xor_sync(0xffffffffu, rmax[r], 2));
            const float m_new = fmaxf(m_i[r], rmax[r]);
            mref[r] = m_new == -INFINITY ? 0.f : m_new;
            alpha[r] = fast_exp2(m_i[r] - mref[r]);
            m_i[r] = m_new;
            l_i[r] *= alpha[r];
        }
#pragma unroll
        for (int t = 0; t < kKC / 8; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float pe = fast_exp2(s[t][e] - mref[e >> 1]);
                s[t][e] = pe;
                l_i[e >> 1] += pe;
            }
#pragma unroll
        for (int t = 0; t < D / 8; ++t) {
            acc[t][0] *= alpha[0];
            acc[t][1] *= alpha[0];
            acc[t][2] *= alpha[1];
            acc[t][3] *= alpha[1];
        }
        // O += P V
#pragma unroll
        for (int kt = 0; kt < kKC / 16; ++kt) {
            uint32_t pa[4];
            pa[0] = pack_bf16x2(s[2 * kt][0], s[2 * kt][1]);
            pa[1] = pack_bf16x2(s[2 * kt][2], s[2 * kt][3]);
            pa[2] = pack_bf16x2(s[2 * kt + 1][0], s[2 * kt + 1][1]);
            pa[3] = pack_bf16x2(s[2 * kt + 1][2], s[2 * kt + 1][3]);
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                uint32_t b0, b1, b2, b3;
                const int key = kt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int col = hl * D + dp * 16 + ((lane >> 4) & 1) * 8;
                ldsm_x4_t(b0, b1, b2, b3, sV + key * L.ld + col);
                mma_bf16_16816(acc[2 * dp], pa, b0, b1);
                mma_bf16_16816(acc[2 * dp + 1], pa, b2, b3);
            }
        }
        __syncthreads();
    }

    // normalise and park O (fp32) in shared memory for the LCE epilogue
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        l_i[r] += __shfl_xor_sync(0xffffffffu, l_i[r], 1);
        l_i[r] += __shfl_xor_sync(0xffffffffu, l_i[r], 2);
    }
    const float inv0 = l_i[0] > 0.f ? 1.f / l_i[0] : 0.f;
    const float inv1 = l_i[1] > 0.f ? 1.f / l_i[1] : 0.f;
    {
        const int r0 = mt * 16 + (lane >> 2);
#pragma unroll
        for (int t = 0; t < D / 8; ++t) {
            const int col = hl * D + t * 8 + 2 * (lane & 3);
            *reinterpret_cast<float2 *>(sO + r0 * L.o_ld + col) = make_float2(acc[t][0] * inv0, acc[t][1] * inv0);
            *reinterpret_cast<float2 *>(sO + (r0 + 8) * L.o_ld + col) =
                make_float2(acc[t][2] * inv1, acc[t][3] * inv1);
        }
    }
    __syncthreads();
    lce_epilogue<T>(prm, sO, L.o_ld, sHalo, n, y0, x0, c0, CH);
}

// ----------------------------------------------------------------------------- float32, SIMT

constexpr int kKCF = 32;  // keys per chunk, float32 kernel

struct F32Smem {
    int idx, halo, kv, o, total;
    int o_ld;
};

__host__ __device__ inline F32Smem f32_smem_layout(int topk, int nq, int RB, int wr, int CH) {
    F32Smem s;
    s.o_ld = CH + 4;
    s.idx = 0;
    s.halo = align16(topk * 4);
    s.kv = s.halo + align16((RB + 4) * (wr + 4) * CH * 4);
    s.o = s.kv + align16(2 * kKCF * CH * 4);
    s.total = s.o + align16(nq * s.o_ld * 4);
    return s;
}

// F32Lanes<D>::n lanes per (query, head), each taking every n-th key of a chunk with
// its own online softmax; the lanes' partial states (max, sum, O) merge by shuffles at
// the end. One lane at d = 64, whose q and O rows already fill the registers.
// float32 FMA throughout (exact enough for 1e-4).
template <int D> struct F32Lanes {
    static constexpr int n = D == 32 ? 2 : 1;
    static constexpr int max_threads = 256;
};

template <int D>
__global__ void __launch_bounds__(F32Lanes<D>::max_threads)
attn_f32_kernel(const AttnParams prm) {
    constexpr int kKSF = F32Lanes<D>::n;
    using T = float;
    extern __shared__ __align__(16) unsigned char smem[];
    const int CH = prm.HG * D;
    const int nq = prm.RB * prm.wr;
    const F32Smem L = f32_smem_layout(prm.topk, nq, prm.RB, prm.wr, CH);
    int *sIdx = reinterpret_cast<int *>(smem + L.idx);
    T *sHalo = reinterpret_cast<T *>(smem + L.halo);
    T *sK = reinterpret_cast<T *>(smem + L.kv);
    T *sV = sK + kKCF * CH;
    float *sO = reinterpret_cast<float *>(smem + L.o);

    int bid = blockIdx.x;
    const int hg = bid % prm.n_hg;
    bid /= prm.n_hg;
    const int rb = bid % prm.n_rb;
    bid /= prm.n_rb;
    const int p = bid % prm.P, n = bid / prm.P;
    const int j = p / prm.S, i = p - j * prm.S;
    const int y0 = j * prm.hr + rb * prm.RB, x0 = i * prm.wr;
    const int c0 = hg * CH;
    const T *qg = static_cast<const T *>(prm.q);
    const T *kg = static_cast<const T *>(prm.k);
    const T *vg = static_cast<const T *>(prm.v);

    const bool bad = load_route(prm, n, p, sIdx);
    load_halo<T>(prm, vg, n, y0, x0, c0, CH, sHalo);
    cp_async_commit();

    const int sub = threadIdx.x % kKSF, qh = threadIdx.x / kKSF;  // the kKSF lanes of a query are adjacent
    const int tq = qh % nq, hl = qh / nq;
    const bool active = hl < prm.HG;
    float qv[D], acc[D];
    float m_i = -INFINITY, l_i = 0.f;
    {
        const int th = tq / prm.wr, tw = tq - th * prm.wr;
        const T *qrow = qg + (((size_t)n * prm.H + y0 + th) * prm.W + x0 + tw) * prm.C + c0 +
                        (active ? hl : 0) * D;
#pragma unroll
        for (int c = 0; c < D; ++c) {
            qv[c] = active ? __ldg(qrow + c) : 0.f;
            acc[c] = 0.f;
        }
    }
    const int Lk = prm.topk * prm.w2;
    for (int k0 = 0; k0 < Lk; k0 += kKCF) {
        __syncthreads();
        load_kv_chunk<T>(prm, kg, vg, sIdx, n, k0, kKCF, c0, CH, CH, sK, sV);
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        if (active) {
            float s[kKCF / kKSF];
            float cmax = -INFINITY;
#pragma unroll
            for (int kq = 0; kq < kKCF / kKSF; ++kq) {
                const int kk = kq * kKSF + sub;
                const float *kr = sK + kk * CH + hl * D;
                float dot = 0.f;
#pragma unroll
                for (int c = 0; c < D; ++c) dot = fmaf(qv[c], kr[c], dot);
                const int key = k0 + kk;
                const bool ok = key < Lk && (!bad || sIdx[key / prm.w2] >= 0);
                s[kq] = ok ? dot * prm.scale_log2 : -INFINITY;
                cmax = fmaxf(cmax, s[kq]);
            }
            const float m_new = fmaxf(m_i, cmax);
            const float mref = m_new == -INFINITY ? 0.f : m_new;
            const float alpha = exp2f(m_i - mref);
            m_i = m_new;
            l_i *= alpha;
#pragma unroll
            for (int c = 0; c < D; ++c) acc[c] *= alpha;
#pragma unroll
            for (int kq = 0; kq < kKCF / kKSF; ++kq) {
                const float pe = exp2f(s[kq] - mref);
                l_i += pe;
                const float *vr = sV + (kq * kKSF + sub) * CH + hl * D;
#pragma unroll
                for (int c = 0; c < D; ++c) acc[c] = fmaf(pe, vr[c], acc[c]);
            }
        }
    }
    // merge the lanes' partial states: common max, rescaled sums and O
    float m = m_i;
#pragma unroll
    for (int o = 1; o < kKSF; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float f = m_i == -INFINITY ? 0.f : exp2f(m_i - m);
    float l = l_i * f;
#pragma unroll
    for (int o = 1; o < kKSF; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
#pragma unroll
    for (int c = 0; c < D; ++c) {
        float a = acc[c] * f;
#pragma unroll
        for (int o = 1; o < kKSF; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        acc[c] = a;
    }
    if (active && sub == 0) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int c = 0; c < D; ++c) sO[tq * L.o_ld + hl * D + c] = acc[c] * inv;
    }
    __syncthreads();
    lce_epilogue<T>(prm, sO, L.o_ld, sHalo, n, y0, x0, c0, CH);
}

}  // namespace bra
