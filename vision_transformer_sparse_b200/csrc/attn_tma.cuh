// attn_tma.cuh — steps 4-5 of BRA with tensor-memory-accelerator (TMA) tile loads.
//
// Same computation as attn_bf16_kernel (attn.cuh): for each query token and head,
// softmax((scale*q) . k) v over the tokens of the topk routed regions taken jointly
// (eqs. 6-7 of the niftyadmin walk-through, section "BRA模块"), plus LCE(V), the
// depthwise 5x5 convolution of the whole V image with bias (eq. 7).
//
// What changes is how tiles reach shared memory. A routed region's K (or V) tile for
// a 64-channel slice is one rectangular box of the (N,H,W,C) map — (64, wr, hr, 1) —
// so one thread issues one cp.async.bulk.tensor per (routed region, tensor, 64-channel
// half), with no per-element address arithmetic. The Q tile and the 2-pixel V halo of
// the CTA's output rows are boxes too (the halo box starts at negative coordinates at
// the image border; the TMA unit fills those with zeros, which is the convolution's
// zero padding). All copies complete on one mbarrier; every wait is bounded.
//
// Shared-memory tiles use the 128-byte swizzle: row r of a tile holds 64 channels
// (128 bytes) and its 16-byte chunk c sits at chunk position c ^ (r & 7), so that the
// ldmatrix reads of 8 rows hit 8 different bank groups. Every tile starts on a
// 1024-byte boundary (a routed region occupies w2 rounded up to 8 rows).
//
// The Q tile and halo do not depend on the routing, so they are requested before
// griddepcontrol.wait: under programmatic dependent launch they overlap the tail of
// the routing kernel.
#pragma once

#include <cuda.h>

#include "attn.cuh"

namespace bra {

struct TmaAttnParams {
    CUtensorMap tmQ;  // q, box (64, wr, RB, 1)
    CUtensorMap tmK;  // k, box (64, wr, hr, 1)
    CUtensorMap tmV;  // v, box (64, wr, hr, 1)
    CUtensorMap tmH;  // v, box (64, wr + 4, RB + 4, 1), unswizzled: the LCE halo
    const __nv_bfloat16 *lce_w, *lce_b;
    __nv_bfloat16 *out;
    const int32_t *r_idx;
    int *err_flag;  // optional: set to 1 when a region index is out of range
    int N, H, W, C, heads, S, topk, hr, wr, w2, P;
    int RB, HG, QT, n_rb, n_hg;
    int slot;  // shared-memory rows per routed region: w2 rounded up to 8
    float scale_log2;
    unsigned wait_limit;  // mbarrier polls before giving up
};

struct TmaSmem {
    int q, halo, k, v, o, rowmap, idx, flags, bar, total;
    int q_half, halo_half, kv_half;
};

// Byte offsets from a 1024-aligned base; `total` includes the alignment slack.
__host__ __device__ inline TmaSmem tma_smem_layout(int topk, int w2, int QT, int RB, int wr, int CH) {
    TmaSmem s;
    const int nh = CH / 64;
    const int slot = (w2 + 7) & ~7;
    const int kpad = (topk * w2 + kKC - 1) / kKC * kKC;
    s.q_half = QT * 16 * 128;
    s.halo_half = (((RB + 4) * (wr + 4) + 7) & ~7) * 128;
    s.kv_half = topk * slot * 128;
    s.q = 0;
    s.halo = s.q + nh * s.q_half;
    s.k = s.halo + nh * s.halo_half;
    s.v = s.k + nh * s.kv_half;
    int end = s.v + nh * s.kv_half;
    const int o_bytes = QT * 16 * (CH + 4) * 4;  // float32 O tile for the epilogue
    if (o_bytes <= 2 * nh * s.kv_half) {
        s.o = s.k;  // K/V are dead by then
    } else {
        s.o = end;
        end += align16(o_bytes);
    }
    s.rowmap = end;
    end += align16(kpad * 4);
    s.idx = end;
    end += align16(topk * 4);
    s.flags = end;
    end += 16;
    s.bar = end;
    end += 16;
    s.total = end + 1024;
    return s;
}

__device__ inline uint32_t ld_shared_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(addr));
    return v;
}

// Address of the 16-byte chunk holding channel `col` (within a 64-channel half) of
// swizzled row `row` of the tile at `tile`.
__device__ inline uint32_t swz(uint32_t tile, int row, int col) {
    return tile + row * 128 + ((((col >> 3) ^ row) & 7) << 4) + (col & 7) * 2;
}

constexpr int kRowInvalid = 0x40000000;  // rowmap flag: key masked out of the softmax

// LCE epilogue rows for one (channel pair, pixel column, group of RT output rows).
// The halo tile is unswizzled: pixel (hy, hx) is the 128-byte row hy*(wr+4)+hx of its
// 64-channel half, so the five taps of a row sit at immediate offsets of one address.
// acc[r] collects bias + sum_{a,b} w[a][b] * V[r0+r+a][xx+b]; every loaded halo row
// feeds each output row it touches, with RT fixed at compile time (no register moves).
template <int RT>
__device__ __forceinline__ void lce_rows(uint32_t tH, int hw, int xx, int r0, int chl, const float2 *wt,
                                         float2 bias, const float *sO, int o_ld, int wr, int cl,
                                         __nv_bfloat16 *orow, size_t row_stride) {
    float2 acc[RT];
#pragma unroll
    for (int r = 0; r < RT; ++r) acc[r] = bias;
#pragma unroll
    for (int hy = 0; hy < RT + 4; ++hy) {
        const uint32_t ra = tH + ((r0 + hy) * hw + xx) * 128 + chl * 2;
        float2 v[5];
#pragma unroll
        for (int b = 0; b < 5; ++b) v[b] = bf16x2_to_float2(ld_shared_u32(ra + b * 128));
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            const int a = hy - r;
            if (a >= 0 && a < 5) {
#pragma unroll
                for (int b = 0; b < 5; ++b) acc[r] = ffma2(wt[a * 5 + b], v[b], acc[r]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < RT; ++r) {
        const float2 o = *reinterpret_cast<const float2 *>(sO + ((r0 + r) * wr + xx) * o_ld + cl);
        *reinterpret_cast<__nv_bfloat162 *>(orow + (size_t)(r0 + r) * row_stride) =
            __floats2bfloat162_rn(o.x + acc[r].x, o.y + acc[r].y);
    }
}

// Rows per epilogue item: 4 when RB allows, else 2, else 1.
__host__ __device__ inline int lce_row_span(int RB) { return RB % 4 == 0 ? 4 : (RB % 2 == 0 ? 2 : 1); }

// The whole LCE epilogue of a unit: items = (channel pair, column, row group), spread
// over `nthreads` threads starting at `t0`. `load_weights(cp)` refreshes the thread's
// weight registers when its channel pair changes.
// out_px0 points at out[n][y0][x0][c0]; C is the pixel pitch, row_stride = W*C.
template <typename LoadW>
__device__ __forceinline__ void lce_epilogue_tma(uint32_t halo_tile, int halo_half, int CH, int wr, int RB,
                                                 const float *sO, int o_ld, __nv_bfloat16 *out_px0, int C,
                                                 size_t row_stride, int t0, int nthreads, int &w_pair,
                                                 const float2 *wt, const float2 &bias, LoadW &&load_weights) {
    const int npairs = CH / 2, hw = wr + 4, RT = lce_row_span(RB);
    const int items = npairs * wr * (RB / RT);
    for (int item = t0; item < items; item += nthreads) {
        const int cp = item & (npairs - 1);
        const int rest = item / npairs;
        const int xx = rest % wr, rg = rest / wr;
        if (cp != w_pair) load_weights(cp);
        const int cl = 2 * cp;
        const uint32_t tH = halo_tile + (cl >> 6) * halo_half;
        const int chl = cl & 63;
        __nv_bfloat16 *orow = out_px0 + (size_t)xx * C + cl;
        if (RT == 4)
            lce_rows<4>(tH, hw, xx, rg * 4, chl, wt, bias, sO, o_ld, wr, cl, orow, row_stride);
        else if (RT == 2)
            lce_rows<2>(tH, hw, xx, rg * 2, chl, wt, bias, sO, o_ld, wr, cl, orow, row_stride);
        else
            lce_rows<1>(tH, hw, xx, rg, chl, wt, bias, sO, o_ld, wr, cl, orow, row_stride);
    }
}

template <int D>
__global__ void __launch_bounds__(256) attn_tma_kernel(const __grid_constant__ TmaAttnParams prm) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);
    const int CH = prm.HG * D, nh = CH / 64;
    const TmaSmem L = tma_smem_layout(prm.topk, prm.w2, prm.QT, prm.RB, prm.wr, CH);
    int *sRow = reinterpret_cast<int *>(sm + L.rowmap);
    int *sIdx = reinterpret_cast<int *>(sm + L.idx);
    int *sFlags = reinterpret_cast<int *>(sm + L.flags);
    float *sO = reinterpret_cast<float *>(sm + L.o);
    const uint32_t bar = base + L.bar;
    const int o_ld = CH + 4;

    int bid = blockIdx.x;
    const int hg = bid % prm.n_hg;
    bid /= prm.n_hg;
    const int rb = bid % prm.n_rb;
    bid /= prm.n_rb;
    const int p = bid % prm.P, n = bid / prm.P;
    const int j = p / prm.S, i = p - j * prm.S;
    const int y0 = j * prm.hr + rb * prm.RB, x0 = i * prm.wr;
    const int c0 = hg * CH;
    const int tid = threadIdx.x;
    const int Lk = prm.topk * prm.w2;
    const int kpad = (Lk + kKC - 1) / kKC * kKC;

    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    __syncthreads();

    if (tid == 0) {
        for (int h = 0; h < nh; ++h) {
            tma_load_4d(base + L.q + h * L.q_half, &prm.tmQ, c0 + 64 * h, x0, y0, n, bar);
            tma_load_4d(base + L.halo + h * L.halo_half, &prm.tmH, c0 + 64 * h, x0 - 2, y0 - 2, n, bar);
        }
        griddep_wait();  // r_idx is written by the preceding routing kernel
        uint32_t bytes = nh * (prm.RB * prm.wr + (prm.RB + 4) * (prm.wr + 4)) * 128;
        int bad = 0;
        const int32_t *ri = prm.r_idx + ((size_t)n * prm.P + p) * prm.topk;
        for (int a = 0; a < prm.topk; ++a) {
            int r = ri[a];
            if (r < 0 || r >= prm.P) {
                r = -1;
                bad = 1;
            }
            sIdx[a] = r;
            if (r >= 0) {
                const int j2 = r / prm.S, i2 = r - j2 * prm.S;
                for (int h = 0; h < nh; ++h) {
                    const uint32_t off = h * L.kv_half + a * prm.slot * 128;
                    tma_load_4d(base + L.k + off, &prm.tmK, c0 + 64 * h, i2 * prm.wr, j2 * prm.hr, n, bar);
                    tma_load_4d(base + L.v + off, &prm.tmV, c0 + 64 * h, i2 * prm.wr, j2 * prm.hr, n, bar);
                }
                bytes += 2 * nh * prm.w2 * 128;
            }
        }
        sFlags[0] = bad;
        if (bad && prm.err_flag) atomicExch(prm.err_flag, 1);
        mbar_arrive_expect_tx(bar, bytes);
    }
    __syncthreads();
    const bool bad = sFlags[0] != 0;

    // key j -> shared-memory row (routed regions in r_idx order, tokens row-major);
    // keys past the end or in a bad region are flagged and point at a finite row
    for (int jj = tid; jj < kpad; jj += blockDim.x) {
        int row = kRowInvalid;
        if (jj < Lk) {
            const int a = jj / prm.w2;
            row = a * prm.slot + (jj - a * prm.w2);
            if (sIdx[a] < 0) row |= kRowInvalid;
        }
        sRow[jj] = row;
    }
    if (bad) {  // zero the K/V rows of skipped regions so masked keys read zeros
        for (int a = 0; a < prm.topk; ++a) {
            if (sIdx[a] >= 0) continue;
            for (int e = tid; e < nh * prm.w2 * 32; e += blockDim.x) {
                const int h = e / (prm.w2 * 32), r = (e / 32) % prm.w2, w = e % 32;
                const int off = h * L.kv_half + (a * prm.slot + r) * 128 + w * 4;
                *reinterpret_cast<uint32_t *>(sm + L.k + off) = 0u;
                *reinterpret_cast<uint32_t *>(sm + L.v + off) = 0u;
            }
        }
    }

    // LCE weights and bias of this thread's first channel pair, while the copies fly
    const int npairs = CH / 2;
    int w_pair = -1;
    float2 wt[25];
    float2 bias = make_float2(0.f, 0.f);
    auto load_weights = [&](int cp) {
        const int c = c0 + 2 * cp;
        const uint32_t *wp = reinterpret_cast<const uint32_t *>(prm.lce_w + (size_t)c * 25);
        uint32_t wv[25];
#pragma unroll
        for (int t = 0; t < 25; ++t) wv[t] = __ldg(wp + t);
#pragma unroll
        for (int t = 0; t < 25; ++t) {
            // element e of the 50-element run (channel c taps 0..24, then channel c+1)
            const int e0 = t, e1 = 25 + t;
            const uint32_t u0 = wv[e0 >> 1], u1 = wv[e1 >> 1];
            wt[t].x = __uint_as_float((e0 & 1) ? (u0 & 0xFFFF0000u) : (u0 << 16));
            wt[t].y = __uint_as_float((e1 & 1) ? (u1 & 0xFFFF0000u) : (u1 << 16));
        }
        bias = bf16x2_to_float2(__ldg(reinterpret_cast<const uint32_t *>(prm.lce_b + c)));
        w_pair = cp;
    };
    if (tid < npairs * prm.wr) load_weights(tid % npairs);
    __syncthreads();

    const bool ok = __syncthreads_and(mbar_wait_bounded(bar, 0, prm.wait_limit));
    if (!ok) {
        if (tid == 0) atomicExch(&g_bra_timeout_flag, 1);
        mbar_wait_bounded(bar, 0, prm.wait_limit);  // let copies in flight land before exit
        return;
    }

    // ---------------------------------------------------------------- attention
    const int warp = tid >> 5, lane = tid & 31;
    const int hl = warp / prm.QT, mt = warp - hl * prm.QT;
    const int hch = hl * D;                   // head's first channel within the CTA slice
    const int half = hch >> 6, coff = hch & 63;
    const uint32_t tQ = base + L.q + half * L.q_half;
    const uint32_t tK = base + L.k + half * L.kv_half;
    const uint32_t tV = base + L.v + half * L.kv_half;
    const int nchunks = kpad / kKC;
    const bool need_mask = bad || (Lk % kKC) != 0;

    uint32_t qa[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int row = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int col = coff + kk * 16 + ((lane >> 4) & 1) * 8;
        uint32_t a = swz(tQ, row, col);
        asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                     : "=r"(qa[kk][0]), "=r"(qa[kk][1]), "=r"(qa[kk][2]), "=r"(qa[kk][3])
                     : "r"(a));
    }
    float m_i[2] = {-INFINITY, -INFINITY}, l_i[2] = {0.f, 0.f};
    float acc[D / 8][4];
#pragma unroll
    for (int t = 0; t < D / 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

    for (int ch = 0; ch < nchunks; ++ch) {
        float s[kKC / 8][4];
#pragma unroll
        for (int t = 0; t < kKC / 8; ++t) s[t][0] = s[t][1] = s[t][2] = s[t][3] = 0.f;
#pragma unroll
        for (int np = 0; np < kKC / 16; ++np) {
            const int key = ch * kKC + np * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
            const int row = sRow[key] & (kRowInvalid - 1);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int col = coff + kk * 16 + ((lane >> 3) & 1) * 8;
                uint32_t b0, b1, b2, b3;
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                             : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3)
                             : "r"(swz(tK, row, col)));
                mma_bf16_16816(s[2 * np], qa[kk], b0, b1);
                mma_bf16_16816(s[2 * np + 1], qa[kk], b2, b3);
            }
        }
        float rmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int t = 0; t < kKC / 8; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float x = s[t][e] * prm.scale_log2;
                if (need_mask) {
                    const int key = ch * kKC + t * 8 + 2 * (lane & 3) + (e & 1);
                    if (sRow[key] & kRowInvalid) x = -INFINITY;
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
#pragma unroll
        for (int kt = 0; kt < kKC / 16; ++kt) {
            uint32_t pa[4];
            pa[0] = pack_bf16x2(s[2 * kt][0], s[2 * kt][1]);
            pa[1] = pack_bf16x2(s[2 * kt][2], s[2 * kt][3]);
            pa[2] = pack_bf16x2(s[2 * kt + 1][0], s[2 * kt + 1][1]);
            pa[3] = pack_bf16x2(s[2 * kt + 1][2], s[2 * kt + 1][3]);
            const int key = ch * kKC + kt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int row = sRow[key] & (kRowInvalid - 1);
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                const int col = coff + dp * 16 + ((lane >> 4) & 1) * 8;
                uint32_t b0, b1, b2, b3;
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                             : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3)
                             : "r"(swz(tV, row, col)));
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
    __syncthreads();  // every warp is done with K/V before O overwrites them
    {
        const int r0 = mt * 16 + (lane >> 2);
#pragma unroll
        for (int t = 0; t < D / 8; ++t) {
            const int col = hch + t * 8 + 2 * (lane & 3);
            *reinterpret_cast<float2 *>(sO + r0 * o_ld + col) = make_float2(acc[t][0] * inv0, acc[t][1] * inv0);
            *reinterpret_cast<float2 *>(sO + (r0 + 8) * o_ld + col) = make_float2(acc[t][2] * inv1, acc[t][3] * inv1);
        }
    }
    __syncthreads();

    // ---------------------------------------------------------------- LCE epilogue
    lce_epilogue_tma(base + L.halo, L.halo_half, CH, prm.wr, prm.RB, sO, o_ld,
                     prm.out + (((size_t)n * prm.H + y0) * prm.W + x0) * prm.C + c0, prm.C,
                     (size_t)prm.W * prm.C, tid, blockDim.x, w_pair, wt, bias, load_weights);
}

}  // namespace bra

namespace bra {

// Exercises the bounded-wait path: waits on an mbarrier whose phase can never
// complete (one expected arrival that never comes) and gives up after `limit`
// polls, raising g_bra_timeout_flag exactly as the attention kernel does. No copy
// is in flight, so giving up is safe.
__global__ void wait_timeout_selftest_kernel(unsigned limit) {
    __shared__ __align__(8) unsigned long long bar_storage;
    const uint32_t bar = smem_u32(&bar_storage);
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    const bool ok = __syncthreads_and(mbar_wait_bounded(bar, 0, limit));
    if (!ok && threadIdx.x == 0) atomicExch(&g_bra_timeout_flag, 1);
}

}  // namespace bra
