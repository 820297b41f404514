// attn_pipe.cuh — steps 4-5 of BRA as a persistent, warp-specialised TMA pipeline.
//
// Same computation as attn_tma_kernel (attn_tma.cuh): token-to-token attention over
// the routed regions (eqs. 6-7 of the niftyadmin walk-through, section "BRA模块")
// plus the LCE depthwise 5x5 convolution of V with bias (eq. 7).
//
// A work unit is (image n, query region p, block of RB region rows, group of HG
// heads). The grid holds a few CTAs per SM; each CTA walks the units
// blockIdx.x, blockIdx.x + gridDim.x, ... through NS shared-memory stages, with
// three warp roles:
//   - producer (last warp): waits until a stage is free ("empty"), takes the unit's
//     routing (fetched by all 32 lanes one unit ahead) and issues its tile boxes (Q
//     tile, V halo, K and V boxes of the routed regions) with cp.async.bulk.tensor
//     onto the stage's "full" barrier;
//   - QT*HG attention warps: wait on "full", run the attention of one (head,
//     16-query tile) each on mma.sync, write O (fp32) over the stage's now dead K/V
//     tiles and arrive on the stage's "O ready" barrier;
//   - nE epilogue warps: wait on "O ready", run the LCE epilogue over the unit's
//     pixels (V halo of the stage, O, weights) and release the stage ("empty").
// So while the epilogue warps finish unit k, the attention warps already work on
// unit k+1 and the copies of the following units are in flight. The grid size is a
// multiple of the number of head groups, so a CTA always works on the same channel
// slice and every epilogue thread keeps its LCE weights in registers for the whole
// kernel. Every wait is bounded; a wait that runs out raises the device timeout flag
// and the warps of a role leave their loop together.
#pragma once

#include "attn_tma.cuh"

namespace bra {

struct PipeSmem {
    int stage_bytes;                  // one stage: Q, halo, K, V tiles (1024-aligned)
    int q, halo, k, v;                // offsets inside a stage
    int q_half, halo_half, kv_half;
    int stages;                       // offset of stage 0 (from the aligned base)
    int o;                            // O tiles: -1 = inside the stage (over its dead K/V), else
    int o_stride;                     //   one per stage at o + s * o_stride
    int rowmap, idx, flags, bars;     // small arrays: shared / per stage (bars: full, oready, empty)
    int total;
};

__host__ __device__ inline PipeSmem pipe_smem_layout(int NS, int topk, int w2, int QT, int RB, int wr, int CH) {
    PipeSmem s;
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
    s.stage_bytes = s.v + nh * s.kv_half;  // multiple of 1024
    s.stages = 0;
    int end = NS * s.stage_bytes;
    const int o_bytes = QT * 16 * (CH + 4) * 4;
    s.o_stride = align16(o_bytes);
    if (o_bytes <= 2 * nh * s.kv_half) {
        s.o = -1;  // K/V of the stage are dead once every warp has finished its attention
    } else {
        // one O tile per stage: the attention warps write unit k+1's O while the
        // epilogue warps still read unit k's, and a stage is only reused after its
        // epilogue has released it
        s.o = end;
        end += NS * s.o_stride;
    }
    s.rowmap = end;
    end += align16(kpad * 4);
    s.idx = end;  // [NS][topk]: the routing of the unit in each stage
    end += align16(NS * topk * 4);
    s.flags = end;  // [NS] bad-index flags
    end += align16(NS * 4);
    s.bars = end;  // full[NS], oready[NS], empty[NS]
    end += 3 * NS * 8;
    s.total = end + 1024;
    return s;
}

struct PipeParams {
    TmaAttnParams t;  // tensor maps, pointers, shape, unit split
    int NS;           // stages
    int NE;           // epilogue warps
    int units;        // N * P * n_rb * n_hg
    int XT;           // LCE epilogue columns per item (1 or 2)
    int fast_keys;    // 1: every unit's keys fill whole 64-key chunks in consecutive rows
    FastDiv div_hg, div_rb, div_P, div_S, div_wx;  // n_hg, n_rb, P, S, wr / XT
    FastDiv div_wr, div_hw, div_nq, div_nh;         // wr, wr + 4, RB * wr, (RB + 4) * (wr + 4)
    const __nv_bfloat16 *q, *k, *v;
};

__device__ inline void bar_sync_named(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(nthreads) : "memory");
}
// Barrier over `nthreads` threads that also ANDs a predicate across them.
__device__ inline bool bar_and_named(int id, int nthreads, bool pred) {
    uint32_t out;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(out)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return out != 0;
}
__device__ inline void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}

// unit u -> (row block rb, region p, image n, region row j, region column i)
__device__ __forceinline__ void decode_unit(const PipeParams &pp, int u, int &rb, int &p, int &n, int &j, int &i) {
    uint32_t r;
    const uint32_t bid = pp.div_hg.div((uint32_t)u);
    const uint32_t b2 = pp.div_rb.divmod(bid, r);
    rb = (int)r;
    n = (int)pp.div_P.divmod(b2, r);
    p = (int)r;
    j = (int)pp.div_S.divmod((uint32_t)p, r);
    i = (int)r;
}

// Attention of one (head, 16-query tile) over the unit's keys in shared memory:
// acc = sum_j p_j v_j (unnormalised), l = sum_j p_j per query row. FAST: the keys
// occupy consecutive tile rows in whole 64-key chunks, so every ldmatrix address is a
// per-lane constant plus an immediate; otherwise rows come from the row map and keys
// past the end or in skipped regions are masked.
template <int D, bool FAST>
__device__ __forceinline__ void attend_tile(uint32_t tQ, uint32_t tK, uint32_t tV, const int *sRow, const int *sIdx,
                                            bool bad, int Lk, int w2, int nchunks, int lane, int mt, int coff,
                                            float sl2, float (&acc)[D / 8][4], float (&l_i)[2]) {
    uint32_t qa[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int row = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int col = coff + kk * 16 + ((lane >> 4) & 1) * 8;
        asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                     : "=r"(qa[kk][0]), "=r"(qa[kk][1]), "=r"(qa[kk][2]), "=r"(qa[kk][3])
                     : "r"(swz(tQ, row, col)));
    }
    // per-lane address parts of the fast path (rows k*16 + lane pattern: row & 7 == lane & 7)
    const uint32_t kbase = tK + ((lane & 7) + ((lane >> 4) & 1) * 8) * 128;
    const uint32_t vbase = tV + ((lane & 7) + ((lane >> 3) & 1) * 8) * 128;
    uint32_t kswz[D / 16], vswz[D / 16];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        kswz[kk] = (((((coff + kk * 16) >> 3) + ((lane >> 3) & 1)) ^ lane) & 7) << 4;
        vswz[kk] = (((((coff + kk * 16) >> 3) + ((lane >> 4) & 1)) ^ lane) & 7) << 4;
    }
    float m_i[2] = {-INFINITY, -INFINITY};
    l_i[0] = l_i[1] = 0.f;
#pragma unroll
    for (int t = 0; t < D / 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
    for (int ch = 0; ch < nchunks; ++ch) {
        float sc[kKC / 8][4];
#pragma unroll
        for (int t = 0; t < kKC / 8; ++t) sc[t][0] = sc[t][1] = sc[t][2] = sc[t][3] = 0.f;
#pragma unroll
        for (int np = 0; np < kKC / 16; ++np) {
            int row = 0;
            if (!FAST) row = sRow[ch * kKC + np * 16 + (lane & 7) + ((lane >> 4) & 1) * 8] & (kRowInvalid - 1);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                uint32_t addr;
                if (FAST)
                    addr = kbase + (ch * kKC + np * 16) * 128 + kswz[kk];
                else
                    addr = swz(tK, row, coff + kk * 16 + ((lane >> 3) & 1) * 8);
                uint32_t b0, b1, b2, b3;
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                             : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3)
                             : "r"(addr));
                mma_bf16_16816(sc[2 * np], qa[kk], b0, b1);
                mma_bf16_16816(sc[2 * np + 1], qa[kk], b2, b3);
            }
        }
        float rmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int t = 0; t < kKC / 8; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (!FAST) {
                    const int key = ch * kKC + t * 8 + 2 * (lane & 3) + (e & 1);
                    if ((sRow[key] & kRowInvalid) || (bad && sIdx[key / w2] < 0)) sc[t][e] = -INFINITY;
                }
                rmax[e >> 1] = fmaxf(rmax[e >> 1], sc[t][e]);
            }
        float mneg[2];  // -(running max of q.k) * scale * log2(e): the exponent offset
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
                for (int t = 0; t < D / 8; ++t) {
                    acc[t][2 * r] *= alpha;
                    acc[t][2 * r + 1] *= alpha;
                }
            }
            m_i[r] = m_new;
            mneg[r] = -mref * sl2;
        }
#pragma unroll
        for (int t = 0; t < kKC / 8; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float pe = fast_exp2(fmaf(sc[t][e], sl2, mneg[e >> 1]));
                sc[t][e] = pe;
                l_i[e >> 1] += pe;
            }
#pragma unroll
        for (int kt = 0; kt < kKC / 16; ++kt) {
            uint32_t pa[4];
            pa[0] = pack_bf16x2(sc[2 * kt][0], sc[2 * kt][1]);
            pa[1] = pack_bf16x2(sc[2 * kt][2], sc[2 * kt][3]);
            pa[2] = pack_bf16x2(sc[2 * kt + 1][0], sc[2 * kt + 1][1]);
            pa[3] = pack_bf16x2(sc[2 * kt + 1][2], sc[2 * kt + 1][3]);
            int row = 0;
            if (!FAST) row = sRow[ch * kKC + kt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8] & (kRowInvalid - 1);
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                uint32_t addr;
                if (FAST)
                    addr = vbase + (ch * kKC + kt * 16) * 128 + vswz[dp];
                else
                    addr = swz(tV, row, coff + dp * 16 + ((lane >> 4) & 1) * 8);
                uint32_t b0, b1, b2, b3;
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                             : "=r"(b0), "=r"(b1), "=r"(b2), "=r"(b3)
                             : "r"(addr));
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
}

// LCE of one (channel pair, XT pixel columns, RT rows) block: loads RT+4 halo rows of
// 4+XT pixels once and feeds every output that uses them (RT, XT fixed: no moves).
template <int RT, int XT>
__device__ __forceinline__ void lce_block(uint32_t tH, int hw, int xc, int r0, int chl, const float2 *wt, float2 bias,
                                          const float *sO, int o_ld, int wr, int cl, __nv_bfloat16 *opx,
                                          int C, size_t row_stride) {
    float2 acc[RT][XT];
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int x = 0; x < XT; ++x) acc[r][x] = bias;
#pragma unroll
    for (int hy = 0; hy < RT + 4; ++hy) {
        const uint32_t ra = tH + ((r0 + hy) * hw + xc) * 128 + chl * 2;
        float2 v[4 + XT];
#pragma unroll
        for (int b = 0; b < 4 + XT; ++b) v[b] = bf16x2_to_float2(ld_shared_u32(ra + b * 128));
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            const int a = hy - r;
            if (a >= 0 && a < 5) {
#pragma unroll
                for (int x = 0; x < XT; ++x)
#pragma unroll
                    for (int b = 0; b < 5; ++b) acc[r][x] = ffma2(wt[a * 5 + b], v[x + b], acc[r][x]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int x = 0; x < XT; ++x) {
            const float2 o = *reinterpret_cast<const float2 *>(sO + ((r0 + r) * wr + xc + x) * o_ld + cl);
            *reinterpret_cast<__nv_bfloat162 *>(opx + (size_t)(r0 + r) * row_stride + (size_t)(xc + x) * C + cl) =
                __floats2bfloat162_rn(o.x + acc[r][x].x, o.y + acc[r][x].y);
        }
}

// MAXT threads at most per CTA and MINB CTAs per SM: the register budget per thread.
template <int D, int MAXT, int MINB>
__global__ void __launch_bounds__(MAXT, MINB) attn_pipe_kernel(const __grid_constant__ PipeParams pp) {
    const TmaAttnParams &prm = pp.t;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);
    const int NS = pp.NS;
    const int CH = prm.HG * D, nh = CH / 64;
    const PipeSmem L = pipe_smem_layout(NS, prm.topk, prm.w2, prm.QT, prm.RB, prm.wr, CH);
    int *sRow = reinterpret_cast<int *>(sm + L.rowmap);
    int *sIdxAll = reinterpret_cast<int *>(sm + L.idx);
    int *sBad = reinterpret_cast<int *>(sm + L.flags);
    // full[s] at bars + 8s, oready[s] at bars + 8(NS + s), empty[s] at bars + 8(2NS + s)
    const uint32_t bars = base + L.bars;
    const int o_ld = CH + 4;
    const int nA = prm.QT * prm.HG;   // attention warps
    const int nE = pp.NE;             // epilogue warps
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Lk = prm.topk * prm.w2;
    const int kpad = (Lk + kKC - 1) / kKC * kKC;
    const int hg = blockIdx.x % prm.n_hg;  // constant: gridDim.x is a multiple of n_hg
    const int c0 = hg * CH;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(bars + 8 * s, 1);              // full: the producer's arrival + bytes
            mbar_init(bars + 8 * (NS + s), nA);      // O ready: one arrival per attention warp
            mbar_init(bars + 8 * (2 * NS + s), nE);  // empty: one arrival per epilogue warp
        }
        fence_mbar_init();
    }
    // key j -> row inside a stage's K/V tile; keys past the end are flagged
    for (int jj = tid; jj < kpad; jj += blockDim.x) {
        int row = kRowInvalid;
        if (jj < Lk) {
            const int a = jj / prm.w2;
            row = a * prm.slot + (jj - a * prm.w2);
        }
        sRow[jj] = row;
    }
    __syncthreads();

    if (warp == nA + nE) {
        // ------------------------------------------------------------ producer warp
        // Lane 0 issues the copies; all 32 lanes fetch the next unit's routing row
        // (lane a holds entries a, a+32, ...) while lane 0 waits for a free stage, so
        // no routing read sits between a stage becoming free and its copies starting.
        constexpr int kRouteRegs = 8;  // topk <= 256
        int rv[kRouteRegs];
        auto fetch_route = [&](int u) {
            int rb, p, n, j, i;
            decode_unit(pp, u, rb, p, n, j, i);
            const int32_t *ri = prm.r_idx + ((size_t)n * prm.P + p) * prm.topk;
#pragma unroll
            for (int e = 0; e < kRouteRegs; ++e) {
                const int a = lane + 32 * e;
                rv[e] = a < prm.topk ? __ldcg(ri + a) : 0;
            }
        };
        int k = 0;
        bool fetched = false;
        for (int u = blockIdx.x; u < pp.units; u += gridDim.x, ++k) {
            const int s = k % NS, use = k / NS;
            const uint32_t full = bars + 8 * s, empty = bars + 8 * (2 * NS + s);
            bool ok = true;
            if (use > 0) {
                if (lane == 0) ok = mbar_wait_bounded(empty, (use - 1) & 1, prm.wait_limit);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) {
                    if (lane == 0) atomicExch(&g_bra_timeout_flag, 1);
                    break;
                }
            }
            int rb, p, n, j, i;
            decode_unit(pp, u, rb, p, n, j, i);
            const int y0 = j * prm.hr + rb * prm.RB, x0 = i * prm.wr;
            const uint32_t st = base + L.stages + s * L.stage_bytes;
            if (lane == 0) {
                if (use > 0) fence_proxy_async();  // generic writes of the last use (O) before the new copies
                for (int h = 0; h < nh; ++h) {
                    tma_load_4d(st + L.q + h * L.q_half, &prm.tmQ, c0 + 64 * h, x0, y0, n, full);
                    tma_load_4d(st + L.halo + h * L.halo_half, &prm.tmH, c0 + 64 * h, x0 - 2, y0 - 2, n, full);
                }
            }
            if (!fetched) {
                griddep_wait();  // r_idx is written by the preceding routing kernel
                fetch_route(u);
                fetched = true;
            }
            // this unit's routing -> the stage's index list; skipped (out-of-range) regions
            int *sIdx = sIdxAll + s * prm.topk;
            bool bad_lane = false;
#pragma unroll
            for (int e = 0; e < kRouteRegs; ++e) {
                const int a = lane + 32 * e;
                if (a < prm.topk) {
                    int r = rv[e];
                    if (r < 0 || r >= prm.P) {
                        r = -1;
                        bad_lane = true;
                    }
                    sIdx[a] = r;
                }
            }
            const bool bad = __any_sync(0xffffffffu, bad_lane);
            __syncwarp();
            const int un = u + gridDim.x;
            if (un < pp.units) fetch_route(un);  // in flight while the copies go out
            if (lane == 0) {
                uint32_t bytes = nh * (prm.RB * prm.wr + (prm.RB + 4) * (prm.wr + 4)) * 128;
                for (int a = 0; a < prm.topk; ++a) {
                    const int r = sIdx[a];
                    if (r >= 0) {
                        uint32_t i2u;
                        const int j2 = (int)pp.div_S.divmod((uint32_t)r, i2u), i2 = (int)i2u;
                        for (int h = 0; h < nh; ++h) {
                            const uint32_t off = h * L.kv_half + a * prm.slot * 128;
                            tma_load_4d(st + L.k + off, &prm.tmK, c0 + 64 * h, i2 * prm.wr, j2 * prm.hr, n, full);
                            tma_load_4d(st + L.v + off, &prm.tmV, c0 + 64 * h, i2 * prm.wr, j2 * prm.hr, n, full);
                        }
                        bytes += 2 * nh * prm.w2 * 128;
                    } else {
                        // skipped region: zero its K/V rows so that masked keys read zeros
                        for (int h = 0; h < nh; ++h)
                            for (int r2 = 0; r2 < prm.w2; ++r2)
                                for (int w = 0; w < 32; ++w) {
                                    const int off =
                                        s * L.stage_bytes + h * L.kv_half + (a * prm.slot + r2) * 128 + w * 4;
                                    *reinterpret_cast<uint32_t *>(sm + L.k + off) = 0u;
                                    *reinterpret_cast<uint32_t *>(sm + L.v + off) = 0u;
                                }
                    }
                }
                sBad[s] = bad ? 1 : 0;
                if (bad && prm.err_flag) atomicExch(prm.err_flag, 1);
                mbar_arrive_expect_tx(full, bytes);
            }
            __syncwarp();
        }
        // every copy this CTA issued must land before it may exit
        if (lane == 0)
            for (int kk = (k > NS ? k - NS : 0); kk < k; ++kk)
                mbar_wait_bounded(bars + 8 * (kk % NS), (kk / NS) & 1, prm.wait_limit);
        return;
    }

    if (warp < nA) {
        // ------------------------------------------------------------ attention warps
        const int hl = warp / prm.QT, mt = warp - hl * prm.QT;
        const int hch = hl * D;
        const int half = hch >> 6, coff = hch & 63;
        const int nchunks = kpad / kKC;
        const int nAT = nA * 32;
        int k = 0;
        for (int u = blockIdx.x; u < pp.units; u += gridDim.x, ++k) {
            const int s = k % NS, use = k / NS;
            const bool ok = bar_and_named(1, nAT, mbar_wait_bounded(bars + 8 * s, use & 1, prm.wait_limit));
            if (!ok) {
                if (tid == 0) atomicExch(&g_bra_timeout_flag, 1);
                break;
            }
            const uint32_t st = base + L.stages + s * L.stage_bytes;
            const int *sIdx = sIdxAll + s * prm.topk;
            const bool bad = sBad[s] != 0;
            const uint32_t tQ = st + L.q + half * L.q_half;
            const uint32_t tK = st + L.k + half * L.kv_half;
            const uint32_t tV = st + L.v + half * L.kv_half;
            float acc[D / 8][4], l_i[2];
            if (pp.fast_keys && !bad)
                attend_tile<D, true>(tQ, tK, tV, sRow, sIdx, bad, Lk, prm.w2, nchunks, lane, mt, coff, prm.scale_log2,
                                     acc, l_i);
            else
                attend_tile<D, false>(tQ, tK, tV, sRow, sIdx, bad, Lk, prm.w2, nchunks, lane, mt, coff,
                                      prm.scale_log2, acc, l_i);
            const float inv0 = l_i[0] > 0.f ? 1.f / l_i[0] : 0.f;
            const float inv1 = l_i[1] > 0.f ? 1.f / l_i[1] : 0.f;
            bar_sync_named(2, nAT);  // every attention warp is done with this stage's K/V
            float *sO = reinterpret_cast<float *>(sm + (L.o >= 0 ? L.o + s * L.o_stride : s * L.stage_bytes + L.k));
            {
                const int r0 = mt * 16 + (lane >> 2);
#pragma unroll
                for (int t = 0; t < D / 8; ++t) {
                    const int col = hch + t * 8 + 2 * (lane & 3);
                    *reinterpret_cast<float2 *>(sO + r0 * o_ld + col) = make_float2(acc[t][0] * inv0, acc[t][1] * inv0);
                    *reinterpret_cast<float2 *>(sO + (r0 + 8) * o_ld + col) =
                        make_float2(acc[t][2] * inv1, acc[t][3] * inv1);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + 8 * (NS + s));  // O ready
        }
        return;
    }

    // ---------------------------------------------------------------- epilogue warps
    const int et = tid - nA * 32, nET = nE * 32;
    const int npairs = CH / 2, wr = prm.wr, hw = wr + 4;
    const int RT = lce_row_span(prm.RB), XT = pp.XT;
    const int pair_shift = npairs == 64 ? 6 : 5;
    const int items = npairs * (wr / XT) * (prm.RB / RT);
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
            const int e0 = t, e1 = 25 + t;
            const uint32_t u0 = wv[e0 >> 1], u1 = wv[e1 >> 1];
            wt[t].x = __uint_as_float((e0 & 1) ? (u0 & 0xFFFF0000u) : (u0 << 16));
            wt[t].y = __uint_as_float((e1 & 1) ? (u1 & 0xFFFF0000u) : (u1 << 16));
        }
        bias = bf16x2_to_float2(__ldg(reinterpret_cast<const uint32_t *>(prm.lce_b + c)));
        w_pair = cp;
    };
    load_weights(et & (npairs - 1));
    const size_t row_stride = (size_t)prm.W * prm.C;
    int k = 0;
    for (int u = blockIdx.x; u < pp.units; u += gridDim.x, ++k) {
        const int s = k % NS, use = k / NS;
        const bool ok = bar_and_named(3, nET, mbar_wait_bounded(bars + 8 * (NS + s), use & 1, prm.wait_limit));
        if (!ok) {
            if (et == 0) atomicExch(&g_bra_timeout_flag, 1);
            break;
        }
        int rb, p, n, j, i;
        decode_unit(pp, u, rb, p, n, j, i);
        const int y0 = j * prm.hr + rb * prm.RB, x0 = i * prm.wr;
        const uint32_t st = base + L.stages + s * L.stage_bytes;
        const float *sO =
            reinterpret_cast<const float *>(sm + (L.o >= 0 ? L.o + s * L.o_stride : s * L.stage_bytes + L.k));
        __nv_bfloat16 *opx = prm.out + (((size_t)n * prm.H + y0) * prm.W + x0) * prm.C + c0;
        for (int item = et; item < items; item += nET) {
            const int cp = item & (npairs - 1);
            uint32_t xg;
            const int rg = (int)pp.div_wx.divmod((uint32_t)(item >> pair_shift), xg);
            if (cp != w_pair) load_weights(cp);
            const int cl = 2 * cp;
            const uint32_t tH = st + L.halo + (cl >> 6) * L.halo_half;
            const int chl = cl & 63, xc = (int)xg * XT, r0 = rg * RT;
            if (XT == 2) {
                if (RT == 4)
                    lce_block<4, 2>(tH, hw, xc, r0, chl, wt, bias, sO, o_ld, wr, cl, opx, prm.C, row_stride);
                else if (RT == 2)
                    lce_block<2, 2>(tH, hw, xc, r0, chl, wt, bias, sO, o_ld, wr, cl, opx, prm.C, row_stride);
                else
                    lce_block<1, 2>(tH, hw, xc, r0, chl, wt, bias, sO, o_ld, wr, cl, opx, prm.C, row_stride);
            } else {
                if (RT == 4)
                    lce_block<4, 1>(tH, hw, xc, r0, chl, wt, bias, sO, o_ld, wr, cl, opx, prm.C, row_stride);
                else if (RT == 2)
                    lce_block<2, 1>(tH, hw, xc, r0, chl, wt, bias, sO, o_ld, wr, cl, opx, prm.C, row_stride);
                else
                    lce_block<1, 1>(tH, hw, xc, r0, chl, wt, bias, sO, o_ld, wr, cl, opx, prm.C, row_stride);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + 8 * (2 * NS + s));  // stage free
    }
}

}  // namespace bra
