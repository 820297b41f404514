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
// copies of 128-row X chunks and BN-row W chunks (32 K-elements, 64-byte swizzle) into
// a ring of shared-memory stages; one thread issues the 128 x BN x 16 MMAs into a
// double-buffered float32 accumulator in tensor memory; four warps drain it (one TMEM
// lane quarter each), add the bias, round to bfloat16 and store. Every wait is bounded.
// float32: linear_f32_kernel, shared-memory tiles and FMA.
#pragma once

#include <cuda.h>

// attn_tma.cuh defines g_bra_timeout_flag, the flag every bounded wait raises
#include "attn_tma.cuh"
#include "umma.cuh"

namespace bra {

struct LinearParams {
    CUtensorMap tmX;  // X (M, K): box (32, 128), 64-byte swizzle, zero fill past row M
    CUtensorMap tmW;  // W (Nout, K): box (32, BN), 64-byte swizzle
    const __nv_bfloat16 *bias;
    __nv_bfloat16 *y[3];
    int M, K, Nout, Ny, BN, tiles_n, tiles, stages;
    uint32_t tmem_cols;
    unsigned wait_limit;
};

constexpr int kLinThreads = 192;  // warp 0 copies, warp 1 MMA, warps 2-5 epilogue
constexpr int kLinRows = 128;     // rows of X per tile (the MMA's M)

struct LinearSmem {
    int stage_bytes, a_bytes, bias, bars, tslot, total;
};

__host__ __device__ inline LinearSmem linear_smem_layout(int BN, int stages, int Nout) {
    LinearSmem s;
    s.a_bytes = kLinRows * 64;  // 128 rows x 32 bf16
    s.stage_bytes = s.a_bytes + BN * 64;
    int end = stages * s.stage_bytes;
    s.bias = end;  // float32 [Nout]
    end += ((Nout * 4 + 15) / 16) * 16;
    s.bars = end;  // full[stages], empty[stages], tfull[2], tempty[2], drain
    end += 8 * (2 * stages + 5);
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

__global__ void __launch_bounds__(kLinThreads, 1) linear_umma_kernel(const __grid_constant__ LinearParams prm) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);
    const int BN = prm.BN, NS = prm.stages, kch = prm.K >> 5;
    const LinearSmem L = linear_smem_layout(BN, NS, prm.Nout);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t bars = base + L.bars;
    const uint32_t full0 = bars, empty0 = bars + 8 * NS, tfull0 = bars + 16 * NS, tempty0 = tfull0 + 16,
                   drain = tfull0 + 32;
    const uint32_t lim = prm.wait_limit;
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
            mbar_init(tempty0 + 8 * b, 128);
        }
        mbar_init(drain, 1);
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
            const uint32_t bytes = (uint32_t)L.stage_bytes;
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < prm.tiles && ok; t += gridDim.x) {
                const int m0 = (t / prm.tiles_n) * kLinRows, n0 = (t % prm.tiles_n) * BN;
                for (int kc = 0; kc < kch; ++kc, ++it) {
                    const int s = it % NS, use = it / NS;
                    if (use > 0 && !mbar_wait_bounded(empty0 + 8 * s, (use - 1) & 1, lim)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = base + s * L.stage_bytes;
                    mbar_arrive_expect_tx(full0 + 8 * s, bytes);
                    lin_tma_load_2d(st, &prm.tmX, kc * 32, m0, full0 + 8 * s);
                    lin_tma_load_2d(st + L.a_bytes, &prm.tmW, kc * 32, n0, full0 + 8 * s);
                }
            }
            if (!ok) atomicExch(&g_bra_timeout_flag, 1);
            // every copy issued has landed before the CTA may exit (immediate when the
            // MMA thread consumed them all)
            for (int s = 0; s < NS && s < it; ++s) mbar_wait_bounded(full0 + 8 * s, ((it - 1 - s) / NS) & 1, lim);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issue
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kLinRows, BN, 0, 0);
            int it = 0, k = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < prm.tiles && ok; t += gridDim.x, ++k) {
                const int b = k & 1, ub = k >> 1;
                if (ub > 0 && !mbar_wait_bounded(tempty0 + 8 * b, (ub - 1) & 1, lim)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tbase + (uint32_t)(b * BN);
                for (int kc = 0; kc < kch; ++kc, ++it) {
                    const int s = it % NS, use = it / NS;
                    if (!mbar_wait_bounded(full0 + 8 * s, use & 1, lim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = base + s * L.stage_bytes;
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        umma_ss(d, smem_desc(st + 32 * kk, 16, 512, kDescSwizzle64B),
                                smem_desc(st + L.a_bytes + 32 * kk, 16, 512, kDescSwizzle64B), idesc,
                                (uint32_t)((kc | kk) != 0));
                    umma_commit(empty0 + 8 * s);  // the stage is free once these MMAs have read it
                }
                if (!ok) break;
                umma_commit(tfull0 + 8 * b);  // the accumulator is complete
            }
            if (!ok) atomicExch(&g_bra_timeout_flag, 1);
            // every MMA must have completed before the tensor memory is released
            umma_commit(drain);
            mbar_wait_bounded(drain, 0, lim);
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int q = warp & 3;  // tensor-memory lane quarter of this warp
        int k = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < prm.tiles; t += gridDim.x, ++k) {
            const int b = k & 1, ub = k >> 1;
            if (!mbar_wait_bounded(tfull0 + 8 * b, ub & 1, lim)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int m0 = (t / prm.tiles_n) * kLinRows, n0 = (t % prm.tiles_n) * BN;
            const int row = m0 + 32 * q + lane;
            const int which = n0 / prm.Ny, col0 = n0 - which * prm.Ny;
            __nv_bfloat16 *dst = prm.y[which] + (size_t)row * prm.Ny + col0;
            const uint32_t taddr = tbase + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * BN);
            for (int c = 0; c < BN; c += 32) {
                uint32_t r[32];
                tmem_ld32(taddr + (uint32_t)c, r);
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float2 bb = *reinterpret_cast<const float2 *>(sBias + n0 + c + 2 * j);
                    const __nv_bfloat162 h =
                        __floats2bfloat162_rn(__uint_as_float(r[2 * j]) + bb.x, __uint_as_float(r[2 * j + 1]) + bb.y);
                    pk[j] = *reinterpret_cast<const uint32_t *>(&h);
                }
                if (row < prm.M) {
                    uint4 *o = reinterpret_cast<uint4 *>(dst + c);
#pragma unroll
                    for (int j = 0; j < 4; ++j) o[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                }
            }
            tc_fence_before();
            lin_arrive(tempty0 + 8 * b);  // this thread's lane of the accumulator is read
        }
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
    float *y[3];
    int M, K, Nout, Ny;
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
            prm.y[which][(size_t)m * prm.Ny + (n - which * prm.Ny)] = acc[i][j] + prm.b[n];
        }
    }
    }
}

}  // namespace bra
