// linear.cuh — the projections either side of the attention: the qkv projection that
// makes q, k, v from the layer input and the output projection `wo` (both nn.Linear
// with bias, y = x w^T + b). Source: "BiFormer ... 前向传播过程" (niftyadmin), section
// "BRA模块" (the qkv projection split into q and kv, the closing linear layer) and the
// module printout of section "网络结构" (qkv Linear(64 -> 192, bias=True), wo
// Linear(64 -> 64, bias=True)).
//
// Y (M x Nout) = X (M x K) W^T + b, row-major X and Y, W (Nout x K) row-major (the
// PyTorch Linear weight), i.e. both operands K-major. The output columns may be split
// into up to three row-major buffers of Ny columns each (column n goes to buffer
// n / Ny, column n % Ny): the qkv projection writes q, k and v directly.
//
// bfloat16: linear_umma_kernel, a persistent tcgen05 GEMM. One warp issues tensor
// copies of 128-row X chunks and BN-row W chunks (KC = 64 K-elements with a 128-byte
// swizzle when K allows, else 32 with a 64-byte swizzle: wider rows stream faster) into
// a ring of shared-memory stages; one thread issues the 128 x BN x 16 MMAs into a
// double-buffered float32 accumulator in tensor memory; eight warps drain it (two per
// TMEM lane quarter, alternate 32-column blocks, the next block's tensor-memory load in
// flight while the current one is processed), add the bias, round to bfloat16 and stage
// each 32 x 32 block in shared memory (64-byte swizzle), from where a tensor store
// writes it out (rows past M are clipped by the store). Every wait is bounded.
// float32: linear_f32_kernel, shared-memory tiles and FMA.
#pragma once

#include <cuda.h>

// attn_tma.cuh defines g_bra_timeout_flag, the flag every bounded wait raises
#include "attn_tma.cuh"
#include "umma.cuh"

namespace bra {

struct LinearParams {
    CUtensorMap tmX;     // X (M, K): box (KC, 128), KC-matched swizzle, zero fill past row M
    CUtensorMap tmW;     // W (Nout, K): box (KC, BN), KC-matched swizzle
    CUtensorMap tmY[3];  // Y_i (M, Ny): box (32, 32), 64-byte swizzle
    const __nv_bfloat16 *bias;
    const __nv_bfloat16 *res;  // epilogue kEpiResidual: (M, Nout) row-major, added after the bias
    int epi;                   // kEpiBias, kEpiGelu or kEpiResidual
    int M, K, Nout, Ny, BN, tiles_n, tiles_m, stages;
    int kc_elems;    // K-elements per chunk: 64 (128-byte rows) or 32 (64-byte rows)
    int w_resident;  // 1: all of W stays in shared memory, the stages carry X chunks only
    uint32_t tmem_cols;
    unsigned wait_limit;
};

// Epilogues: y = round(acc + b); y = round(GELU(acc + b)) (the BiFormer MLP's first layer,
// GELU in its exact erf form); y = round(res + round(acc + b)) (the MLP's second layer
// with the block's residual: the projection is stored in the dtype, then added).
enum { kEpiBias = 0, kEpiGelu = 1, kEpiResidual = 2 };

// erf by the rational approximation of Abramowitz and Stegun, "Handbook of Mathematical
// Functions", formula 7.1.26 (absolute error at most 1.5e-7 for x >= 0; odd extension):
//   erf(x) = 1 - (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-x^2),  t = 1 / (1 + p x),
// with the handbook's p and a1..a5. The reciprocal and the exponential (as 2^(-x^2 log2 e))
// run on the MUFU; their relative errors (about 2^-22) add well under 1e-7 here.
__device__ __forceinline__ float erf_as(float x) {
    const float ax = fabsf(x);
    float t;
    asm("rcp.approx.ftz.f32 %0, %1;\n" : "=f"(t) : "f"(fmaf(0.3275911f, ax, 1.0f)));
    const float poly =
        t * fmaf(fmaf(fmaf(fmaf(1.061405429f, t, -1.453152027f), t, 1.421413741f), t, -0.284496736f), t, 0.254829592f);
    const float e = fast_exp2(ax * (-1.4426950408889634f * ax));
    return copysignf(fmaf(-poly, e, 1.0f), x);
}
__device__ __forceinline__ float gelu_erf(float x) { return 0.5f * x * (1.0f + erf_as(x * 0.70710678118654752f)); }

constexpr int kLinEpiWarps = 8;                     // two per tensor-memory lane quarter
constexpr int kLinThreads = 64 + 32 * kLinEpiWarps;  // warp 0 copies, warp 1 MMA, then the epilogue
constexpr int kLinRows = 128;                        // rows of X per tile (the MMA's M)
constexpr int kLinOutSlots = 4;                      // 32 x 32 output blocks in flight per epilogue warp

struct LinearSmem {
    int stage_bytes, a_bytes, w, out, bias, bars, tslot, total;
};

// Two modes. W resident (Nout * K * 2 bytes of W held for the whole kernel, loaded once
// per CTA): a stage is one KC-wide K chunk of a 128-row X tile, and each X tile is used
// for all tiles_n column tiles before its stages are released. Streaming: a stage is an
// X chunk and the matching BN-row W chunk of one (row tile, column tile) unit.
__host__ __device__ inline LinearSmem linear_smem_layout(int BN, int stages, int Nout, int K, bool w_resident,
                                                        int kc_elems) {
    LinearSmem s;
    s.a_bytes = kLinRows * kc_elems * 2;  // 128 rows x one K chunk
    s.stage_bytes = w_resident ? s.a_bytes : s.a_bytes + BN * kc_elems * 2;
    int end = stages * s.stage_bytes;
    s.w = end;  // W resident: [tiles_n][K / KC][BN rows x one K chunk]
    end += w_resident ? Nout * K * 2 : 0;
    s.out = end;  // [kLinEpiWarps][kLinOutSlots][32 rows x 64 B] output staging
    end += kLinEpiWarps * kLinOutSlots * 2048;
    s.bias = end;  // float32 [Nout]
    end += ((Nout * 4 + 15) / 16) * 16;
    s.bars = end;  // full[stages], empty[stages], tfull[2], tempty[2], drain, wfull
    end += 8 * (2 * stages + 6);
    s.tslot = end;
    end += 16;
    s.total = end + 1024;  // 1024-byte alignment of the base
    return s;
}

__device__ inline void lin_tma_load_2d(uint32_t dst, const void *tmap, int c0, int c1, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];\n" ::"r"(dst),
        "l"(tmap), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}
__device__ inline void lin_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ inline void lin_tma_store_2d(const void *tmap, uint32_t src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];\n" ::"l"(tmap),
                 "r"(src), "r"(c0), "r"(c1)
                 : "memory");
}
__device__ inline void lin_bulk_commit() { asm volatile("cp.async.bulk.commit_group;\n" ::: "memory"); }
// Wait until at most N of this thread's committed store groups still read shared memory.
template <int N> __device__ inline void lin_bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;\n" ::"n"(N) : "memory");
}
// Wait until at most N of this thread's committed store groups are still incomplete.
template <int N> __device__ inline void lin_bulk_wait() {
    asm volatile("cp.async.bulk.wait_group %0;\n" ::"n"(N) : "memory");
}

// The work of a CTA is a sequence of units (row tile, column tile): W resident, its
// row tiles blockIdx.x, blockIdx.x + gridDim.x, ... each with column tiles 0 .. tiles_n-1
// in order; streaming, the units blockIdx.x, blockIdx.x + gridDim.x, ... of the
// row-major unit grid.
__device__ inline int lin_units(const LinearParams &p) {
    if (p.w_resident) {
        const int mt = (int)blockIdx.x < p.tiles_m ? (p.tiles_m - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
        return mt * p.tiles_n;
    }
    const int tiles = p.tiles_m * p.tiles_n;
    return (int)blockIdx.x < tiles ? (tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
}
__device__ inline void lin_unit(const LinearParams &p, int i, int &mt, int &nt) {
    if (p.w_resident) {
        mt = (int)blockIdx.x + (i / p.tiles_n) * (int)gridDim.x;
        nt = i % p.tiles_n;
    } else {
        const int t = (int)blockIdx.x + i * (int)gridDim.x;
        mt = t / p.tiles_n;
        nt = t % p.tiles_n;
    }
}

__global__ void __launch_bounds__(kLinThreads, 1) linear_umma_kernel(const __grid_constant__ LinearParams prm) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);
    const int BN = prm.BN, NS = prm.stages, KC = prm.kc_elems, kch = prm.K / KC;
    const bool wres = prm.w_resident != 0;
    const LinearSmem L = linear_smem_layout(BN, NS, prm.Nout, prm.K, wres, KC);
    // K-major operands: rows of KC bf16 (2 * KC bytes), 8-row groups 16 * KC bytes apart,
    // the k-th 16-element step 32 bytes into the row
    const uint32_t sbo = (uint32_t)(16 * KC);
    const uint64_t swz = KC == 64 ? kDescSwizzle128B : kDescSwizzle64B;
    const int wchunk = BN * KC * 2;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t bars = base + L.bars;
    const uint32_t full0 = bars, empty0 = bars + 8 * NS, tfull0 = bars + 16 * NS, tempty0 = tfull0 + 16,
                   drain = tfull0 + 32, wfull = tfull0 + 40;
    const uint32_t lim = prm.wait_limit;
    const int units = lin_units(prm);
    float *sBias = reinterpret_cast<float *>(sm + L.bias);

    if (warp == 1) {
        tmem_alloc(base + L.tslot, prm.tmem_cols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull0 + 8 * b, 1);
            mbar_init(tempty0 + 8 * b, 32 * kLinEpiWarps);
        }
        mbar_init(drain, 1);
        mbar_init(wfull, 1);
        fence_mbar_init();
    }
    for (int i = tid; i < prm.Nout; i += kLinThreads) sBias[i] = __bfloat162float(prm.bias[i]);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *reinterpret_cast<volatile uint32_t *>(sm + L.tslot);

    if (warp == 0) {
        // ---------------------------------------------------------------- tensor copies
        if (lane == 0) {
            if (wres && units > 0) {
                // all of W once, chunk (nt, kc) at ((nt * kch) + kc) * wchunk
                mbar_arrive_expect_tx(wfull, (uint32_t)(prm.Nout * prm.K * 2));
                for (int nt = 0; nt < prm.tiles_n; ++nt)
                    for (int kc = 0; kc < kch; ++kc)
                        lin_tma_load_2d(base + L.w + (nt * kch + kc) * wchunk, &prm.tmW, kc * KC, nt * BN, wfull);
            }
            const uint32_t bytes = (uint32_t)L.stage_bytes;
            int it = 0;
            bool ok = true;
            for (int i = 0; i < units && ok; ++i) {
                int mt, nt;
                lin_unit(prm, i, mt, nt);
                if (wres && nt > 0) continue;  // the row tile's chunks serve all its column tiles
                for (int kc = 0; kc < kch; ++kc, ++it) {
                    const int s = it % NS, use = it / NS;
                    if (use > 0 && !mbar_wait_bounded(empty0 + 8 * s, (use - 1) & 1, lim)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = base + s * L.stage_bytes;
                    mbar_arrive_expect_tx(full0 + 8 * s, bytes);
                    lin_tma_load_2d(st, &prm.tmX, kc * KC, mt * kLinRows, full0 + 8 * s);
                    if (!wres) lin_tma_load_2d(st + L.a_bytes, &prm.tmW, kc * KC, nt * BN, full0 + 8 * s);
                }
            }
            if (!ok) atomicExch(&g_bra_timeout_flag, 1);
            // every copy issued has landed before the CTA may exit (immediate when the
            // MMA thread consumed them all)
            for (int s = 0; s < NS && s < it; ++s) mbar_wait_bounded(full0 + 8 * s, ((it - 1 - s) / NS) & 1, lim);
            if (wres && units > 0) mbar_wait_bounded(wfull, 0, lim);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issue
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kLinRows, BN, 0, 0);
            bool ok = !(wres && units > 0) || mbar_wait_bounded(wfull, 0, lim);
            int it = 0;  // first stage index of the current row tile (W resident) / unit
            for (int i = 0; i < units && ok; ++i) {
                int mt, nt;
                lin_unit(prm, i, mt, nt);
                const int b = i & 1, ub = i >> 1;
                if (ub > 0 && !mbar_wait_bounded(tempty0 + 8 * b, (ub - 1) & 1, lim)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tbase + (uint32_t)(b * BN);
                for (int kc = 0; kc < kch; ++kc) {
                    const int s = (it + kc) % NS, use = (it + kc) / NS;
                    if ((!wres || nt == 0) && !mbar_wait_bounded(full0 + 8 * s, use & 1, lim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a = base + s * L.stage_bytes;
                    const uint32_t w = wres ? base + L.w + (nt * kch + kc) * wchunk : a + L.a_bytes;
                    for (int kk = 0; kk < KC / 16; ++kk)
                        umma_ss(d, smem_desc(a + 32 * kk, 16, sbo, swz), smem_desc(w + 32 * kk, 16, sbo, swz), idesc,
                                (uint32_t)((kc | kk) != 0));
                    if (!wres) umma_commit(empty0 + 8 * s);  // streaming: the stage is free once read
                }
                if (!ok) break;
                umma_commit(tfull0 + 8 * b);  // the accumulator is complete
                if (!wres) {
                    it += kch;
                } else if (nt == prm.tiles_n - 1) {
                    // the row tile's stages are free once its last column tile has read them
                    for (int kc = 0; kc < kch; ++kc) umma_commit(empty0 + 8 * ((it + kc) % NS));
                    it += kch;
                }
            }
            if (!ok) atomicExch(&g_bra_timeout_flag, 1);
            // every MMA must have completed before the tensor memory is released
            umma_commit(drain);
            mbar_wait_bounded(drain, 0, lim);
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        // warp (q, h): rows 32q .. 32q + 31 (its tensor-memory lane quarter), column
        // blocks 32h, 32h + 64, ... of each unit
        const int q = warp & 3, h = (warp - 2) >> 2;
        const uint32_t stg = base + L.out + (warp - 2) * (kLinOutSlots * 2048);
        int g = 0;
        bool ok = true;
        for (int i = 0; i < units; ++i) {
            const int b = i & 1, ub = i >> 1;
            if (!mbar_wait_bounded(tfull0 + 8 * b, ub & 1, lim)) {
                ok = false;
                break;
            }
            tc_fence_after();
            int mt, nt;
            lin_unit(prm, i, mt, nt);
            const int m0 = mt * kLinRows, n0 = nt * BN;
            const int which = n0 / prm.Ny, col0 = n0 - which * prm.Ny;
            const uint32_t taddr = tbase + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * BN);
            // bias, round, stage and store the 32 x 32 block at column c of the unit
            auto emit = [&](const uint32_t (&r)[32], int c) {
                const uint32_t sb = stg + (g % kLinOutSlots) * 2048;
                if (g >= kLinOutSlots) {
                    // the store that used this slot has finished reading it
                    if (lane == 0) lin_bulk_wait_read<kLinOutSlots - 1>();
                    __syncwarp();
                }
                // the residual's row `lane`, columns c .. c + 31 of the unit (64 bytes)
                uint4 rv[4] = {};
                if (prm.epi == kEpiResidual && m0 + 32 * q + lane < prm.M) {
                    const uint4 *rp = reinterpret_cast<const uint4 *>(prm.res + (size_t)(m0 + 32 * q + lane) * prm.Nout +
                                                                      n0 + c);
#pragma unroll
                    for (int j = 0; j < 4; ++j) rv[j] = __ldg(rp + j);
                }
                // row `lane` of the block: four 16-byte chunks, 64-byte swizzle
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t pk[4];
                    const uint32_t *rw = reinterpret_cast<const uint32_t *>(&rv[j]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int col = 8 * j + 2 * e;
                        const float2 bb = *reinterpret_cast<const float2 *>(sBias + n0 + c + col);
                        float v0 = __uint_as_float(r[col]) + bb.x, v1 = __uint_as_float(r[col + 1]) + bb.y;
                        if (prm.epi == kEpiGelu) {
                            v0 = gelu_erf(v0);
                            v1 = gelu_erf(v1);
                        } else if (prm.epi == kEpiResidual) {
                            v0 = __bfloat162float(__float2bfloat16_rn(v0)) + __uint_as_float(rw[e] << 16);
                            v1 = __bfloat162float(__float2bfloat16_rn(v1)) + __uint_as_float(rw[e] & 0xFFFF0000u);
                        }
                        const __nv_bfloat162 hv = __floats2bfloat162_rn(v0, v1);
                        pk[e] = *reinterpret_cast<const uint32_t *>(&hv);
                    }
                    const uint32_t dst = sb + lane * 64 + (((j ^ (lane >> 1)) & 3) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(dst), "r"(pk[0]), "r"(pk[1]),
                                 "r"(pk[2]), "r"(pk[3])
                                 : "memory");
                }
                fence_proxy_async();  // the tensor store reads what the generic stores wrote
                __syncwarp();
                if (lane == 0) {
                    // a block wholly past row M is not stored (its group is empty), so that
                    // every block still commits one group for the slot bookkeeping
                    if (m0 + 32 * q < prm.M) lin_tma_store_2d(&prm.tmY[which], sb, col0 + c, m0 + 32 * q);
                    lin_bulk_commit();
                }
                ++g;
            };
            uint32_t ra[32], rb[32];
            int c = 32 * h;
            if (c < BN) tmem_ld32_nowait(taddr + (uint32_t)c, ra);
            while (c < BN) {
                tmem_wait_ld(ra);
                const int c1 = c + 64;
                if (c1 < BN) tmem_ld32_nowait(taddr + (uint32_t)c1, rb);
                emit(ra, c);
                if (c1 >= BN) break;
                tmem_wait_ld(rb);
                const int c2 = c1 + 64;
                if (c2 < BN) tmem_ld32_nowait(taddr + (uint32_t)c2, ra);
                emit(rb, c1);
                c = c2;
            }
            tc_fence_before();
            lin_arrive(tempty0 + 8 * b);  // this thread's share of the accumulator is read
        }
        if (lane == 0) lin_bulk_wait<0>();  // the stores are complete before the CTA exits
        if (!ok && lane == 0) atomicExch(&g_bra_timeout_flag, 1);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, prm.tmem_cols);
    }
}

// ----------------------------------------------------------------------------- float32

struct LinearF32Params {
    const float *x, *w, *b;
    const float *res;  // kEpiResidual: (M, Nout) row-major
    float *y[3];
    int M, K, Nout, Ny, epi;
};

// 64 x 64 output tiles, one column block per blockIdx.x, row blocks blockIdx.y,
// blockIdx.y + gridDim.y, ...; 256 threads (4 x 4 outputs each), K in steps of 16 staged
// in shared memory (both tiles stored K-outer, so each is read along its output index).
__global__ void __launch_bounds__(256) linear_f32_kernel(const LinearF32Params prm) {
    __shared__ float sX[16][64 + 4];
    __shared__ float sW[16][64 + 4];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int n0 = blockIdx.x * 64;
    for (int m0 = blockIdx.y * 64; m0 < prm.M; m0 += gridDim.y * 64) {
    float acc[4][4] = {};
    for (int k0 = 0; k0 < prm.K; k0 += 16) {
        for (int e = tid; e < 64 * 16; e += 256) {
            const int r = e >> 4, kk = e & 15;
            const int m = m0 + r, n = n0 + r, kx = k0 + kk;
            sX[kk][r] = (m < prm.M && kx < prm.K) ? prm.x[(size_t)m * prm.K + kx] : 0.f;
            sW[kk][r] = (n < prm.Nout && kx < prm.K) ? prm.w[(size_t)n * prm.K + kx] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float a[4], bw[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = sX[kk][ty + 16 * i];
                bw[i] = sW[kk][tx + 16 * i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bw[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty + 16 * i;
        if (m >= prm.M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx + 16 * j;
            if (n >= prm.Nout) continue;
            const int which = n / prm.Ny;
            float v = acc[i][j] + prm.b[n];
            if (prm.epi == kEpiGelu) v = gelu_erf(v);
            else if (prm.epi == kEpiResidual) v += prm.res[(size_t)m * prm.Nout + n];
            prm.y[which][(size_t)m * prm.Ny + (n - which * prm.Ny)] = v;
        }
    }
    }
}

}  // namespace bra
