// attn_umma.cuh — steps 4-5 of BRA for large regions on the 5th-generation tensor
// cores (tcgen05), with scores and probabilities held in tensor memory.
//
// Same computation as the other attention kernels: token-to-token softmax attention
// of every query of a region over the keys of its topk routed regions (eq. 6 of the
// niftyadmin BiFormer walk-through, section "BRA模块"; BiFormer paper, section 3.2,
// "Token-to-token attention") plus the LCE term, a depthwise 5x5 convolution of V with
// bias (same section, eq. 7).
//
// Shapes: bf16, head dim 32, regions of 128 or 256 tokens (hr a multiple of 8, wr
// even), topk * w2 <= 256 keys per query. Work unit = (image n, query region p, head
// h); a CTA (one per SM) keeps one head and walks its units through two shared-memory
// stages. Each 128-query tile t owns 256 TMEM columns, used as two halves of 128: the
// scores of keys 0..127 of unit k go to half F(k) = k mod 2, those of keys 128..255 to the
// other half G(k). O(k) accumulates in the first 32 columns of F(k) and every P is
// written over scores already read, so the next unit's first-half scores (into G(k)) can
// be computed as soon as O(k) is complete, while O(k) itself is still being read.
// Warp roles:
//   - warp 0, lane 0: TMA producer. Per unit: the Q tile (w2 rows of 32 channels,
//     64-byte swizzle), the K and V tiles of the routed regions (same layout) and the
//     V halo of the query region ((hr+4) x (wr+4) pixels, no swizzle, zero outside the
//     image) onto the stage's "full" barrier.
//   - warps 1 and 2, lane 0: MMA issuers, one per tile t: S_F = Q_t K_{0..127}^T, then
//     (once the epilogue has read the previous O) S_G = Q_t K_{128..255}^T, then
//     O_t = P_t V with P_t read from TMEM (the A operand) and V from shared memory
//     (MN-major), four 16-key steps per 64-key chunk pair as soon as that pair's P is
//     stored.
//   - warps 3..10: softmax, two warpgroups; warpgroup t owns tile t, each thread one
//     query row, and does nothing but the passes: two 32-key chunks at a time,
//     p = 2^((s - m) * scale * log2 e) on the MUFU with m the max of the first valid
//     chunk, row sum in fp32, P packed to bf16 over scores already read; the row sum
//     goes to shared memory before the last pair is signalled.
//   - warps 11..: LCE and epilogue, kUmmaLceWarps / 4 warpgroups. The depthwise 5x5 convolution
//     plus bias of the unit's pixels in fp32 (one channel pair per thread, weights in
//     registers, 8 rows x 2 columns per item) into an fp32 staging tile; then warpgroup
//     g finishes tiles g, g + groups, ..., one query row per thread (the warp's TMEM lane quarter): O read
//     from TMEM, O / l + LCE rounded once to bf16 into a 64B-swizzled smem tile that
//     one thread stores with the TMA.
//     A row whose p, sum or O is not finite (a later key far above m) is recomputed
//     exactly from the stage's Q, K, V.
// Every wait is bounded; a wait that runs out raises the device timeout flag and the
// role leaves its loop. Tensor memory is released on every path.
#pragma once

#include "attn_pipe.cuh"
#include "umma.cuh"

namespace bra {

constexpr int kUmmaLceWarps = 4;  // one or two warpgroups
constexpr int kUmmaSoftWarp0 = 3;                      // first softmax warp
constexpr int kUmmaLceWarp0 = kUmmaSoftWarp0 + 8;      // first LCE warp
constexpr int kUmmaThreads = (kUmmaLceWarp0 + kUmmaLceWarps) * 32;
constexpr int kUmmaStagePitch = 36;  // floats per staging row (conflict-free float4 rows)
constexpr int kUmmaRows = 8;         // LCE output rows per item (two pixel columns per item)

// barrier slots
enum {
    kUbFull = 0,      // [2] stage loaded (TMA bytes)
    kUbEmpty = 2,     // [2] stage free: MMA commits + every LCE/epilogue thread
    kUbSFullF = 4,    // [2] first-half scores of tile t in TMEM
    kUbSFullG = 6,    // [2] second-half scores of tile t in TMEM
    kUbOFull = 8,     // [2] O_t complete in TMEM
    kUbOEmpty = 10,   // [2] O_t read by the epilogue
    kUbDrain = 12,    // [2] MMA drain before the TMEM is released
    kUbOTFree = 14,   // [2] output tile t free (the previous unit's store has read it)
    kUbOTReady = 16,  // [2] output tile t written by all 128 rows
    kUbGRead = 18,    // [2] second-half scores of tile t read by the pass
    kUbPFree = 20,    // [2] P of pair 0 of tile t consumed by the MMA
    kUbLFull = 22,    // LCE staging written
    kUbLEmpty = 23,   // LCE staging consumed
    kUbP = 24,        // [2][4] P of chunk pair j of tile t stored
    kUbCount = 32
};

struct UmmaSmem {
    int q, k, v, halo, stage_bytes;  // offsets inside a stage; stage size (1024-aligned)
    int staging;                     // fp32 [w2][kUmmaStagePitch]: LCE + bias
    int otile;                       // bf16 output tiles [2 tiles][128 rows][32] (64B swizzle)
    int rsum;                        // fp32 [2 tiles][128]: row sums of the current pass
    int idx;                         // int [2][topk]: routing of the unit in each stage
    int bars, tslot, total;
};

__host__ __device__ inline UmmaSmem umma_smem_layout(int topk, int w2, int hr, int wr) {
    UmmaSmem L;
    L.q = 0;
    L.k = w2 * 64;
    L.v = L.k + topk * w2 * 64;
    L.halo = L.v + topk * w2 * 64;
    L.stage_bytes = L.halo + (((hr + 4) * (wr + 4) * 64 + 1023) & ~1023);
    L.staging = 2 * L.stage_bytes;
    L.otile = L.staging + ((w2 * kUmmaStagePitch * 4 + 1023) & ~1023);
    L.rsum = L.otile + 2 * 128 * 64;
    L.idx = L.rsum + 2 * 128 * 4;
    L.bars = L.idx + ((2 * topk * 4 + 7) & ~7);
    L.tslot = L.bars + kUbCount * 8;
    L.total = L.tslot + 16 + 1024;  // + alignment of the dynamic base to 1024
    return L;
}

struct UmmaParams {
    CUtensorMap tmQ, tmK, tmV, tmH;  // Q/K/V: 32 x wr x hr boxes, 64B swizzle; H: 32 x (wr+4) x (hr+4)
    CUtensorMap tmO;                 // out: 32 x wr x (128 / wr) boxes, 64B swizzle (stores)
    const __nv_bfloat16 *lce_w, *lce_b;
    __nv_bfloat16 *out;
    const int32_t *r_idx;
    int *err_flag;
    int H, W, C, heads, S, topk, hr, wr, w2, P;
    int regions;  // N * P
    float scale_log2;
    unsigned wait_limit;
    FastDiv div_P, div_S, div_wr, div_wx;  // div_wx: wr / 2
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;\n" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ void umma_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}

// Bounded wait whose outcome is the same for every lane of the warp.
__device__ __forceinline__ bool umma_wait_warp(uint32_t bar, uint32_t parity, uint32_t limit) {
    return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity, limit));
}

// Row max of 32 scores, two independent chains.
__device__ __forceinline__ float max32(const uint32_t (&r)[32], float m) {
    float a = m, b = m;
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
        a = fmax3(a, __uint_as_float(r[e]), __uint_as_float(r[e + 1]));
        b = fmax3(b, __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
    }
    return fmaxf(a, b);
}

// p = 2^(s * sl2 + mneg) for 32 scores: row sums into two accumulators, P packed to bf16.
__device__ __forceinline__ void exp32(const uint32_t (&r)[32], float2 sl2v, float2 mnv, float2 &la, float2 &lb,
                                      uint32_t (&pk)[16]) {
    const float2 one = make_float2(1.f, 1.f);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const float2 x = ffma2(make_float2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])), sl2v, mnv);
        const float p0 = fast_exp2(x.x), p1 = fast_exp2(x.y);
        if (e & 1)
            lb = ffma2(make_float2(p0, p1), one, lb);
        else
            la = ffma2(make_float2(p0, p1), one, la);
        pk[e] = pack_bf16x2(p0, p1);
    }
}

// 4-D tiled tensor store from shared memory (bulk-group completion).
__device__ __forceinline__ void tma_store_4d(const void *tmap, uint32_t src, int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];\n" ::"l"(tmap), "r"(src),
        "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;\n" ::: "memory"); }
// Wait until at most N committed bulk groups of this thread still read shared memory.
template <int N> __device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;\n" ::"n"(N) : "memory");
}
template <int N> __device__ __forceinline__ void bulk_wait() {
    asm volatile("cp.async.bulk.wait_group %0;\n" ::"n"(N) : "memory");
}

// 16-byte chunk j of row r of a 64-byte-swizzled tile (rows of 32 bf16).
__device__ __forceinline__ uint4 umma_tile_chunk(const unsigned char *tile, int r, int j) {
    return *reinterpret_cast<const uint4 *>(tile + r * 64 + ((j ^ ((r >> 1) & 3)) << 4));
}

// Exact attention of query row qi from the Q, K and V tiles of a stage, in fp32 on the
// CUDA cores with the true row max: the fallback for a row whose single-pass
// probabilities overflowed. Returns the normalised O row and the row sum l (then 1).
__device__ __noinline__ void umma_exact_row(const unsigned char *stage, const UmmaSmem &L, int qi, int w2, int topk,
                                            uint32_t vmask, float sl2, float (&o)[32], float &l) {
    float q[32];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint4 u = umma_tile_chunk(stage + L.q, qi, j);
        unpack16(u, q + 8 * j, (const __nv_bfloat16 *)nullptr);
    }
    const int Lk = topk * w2;
    auto score = [&](int key) {
        float kk[32], acc = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) unpack16(umma_tile_chunk(stage + L.k, key, j), kk + 8 * j, (const __nv_bfloat16 *)nullptr);
#pragma unroll
        for (int c = 0; c < 32; ++c) acc = fmaf(q[c], kk[c], acc);
        return acc;
    };
    float m = -INFINITY;
    for (int key = 0; key < Lk; ++key)
        if ((vmask >> (key / w2)) & 1u) m = fmaxf(m, score(key));
#pragma unroll
    for (int c = 0; c < 32; ++c) o[c] = 0.f;
    l = 0.f;
    for (int key = 0; key < Lk; ++key) {
        if (!((vmask >> (key / w2)) & 1u)) continue;
        const float p = exp2f((score(key) - m) * sl2);
        l += p;
        float vv[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) unpack16(umma_tile_chunk(stage + L.v, key, j), vv + 8 * j, (const __nv_bfloat16 *)nullptr);
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = fmaf(p, vv[c], o[c]);
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int c = 0; c < 32; ++c) o[c] *= inv;
    l = l > 0.f ? 1.f : 0.f;
}

__global__ void __launch_bounds__(kUmmaThreads, 1) attn_umma_kernel(const __grid_constant__ UmmaParams prm) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sm = smem_raw + (base - raw);
    const UmmaSmem L = umma_smem_layout(prm.topk, prm.w2, prm.hr, prm.wr);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t bars = base + L.bars;
    const int Lk = prm.topk * prm.w2;
    // 128-query tiles per unit; a 64-token region fills the first 64 rows of one tile (the
    // other rows are independent of them in every product and are never stored)
    const int nT = prm.w2 >= 128 ? prm.w2 >> 7 : 1;
    const int tile_rows = prm.w2 < 128 ? prm.w2 : 128;
    const int np = Lk >> 6;       // 64-key chunk pairs per row
    const int cpr = prm.w2 >> 5;  // 32-key chunks per routed region
    const int heads = prm.heads;
    const int h = blockIdx.x % heads;
    const int stride_ru = gridDim.x / heads;  // gridDim.x is a multiple of heads
    const int ru0 = blockIdx.x / heads;
    const int c0 = h * 32;
    const uint32_t lim = prm.wait_limit;
    int *sIdx = reinterpret_cast<int *>(sm + L.idx);
    float *sStage = reinterpret_cast<float *>(sm + L.staging);

    if (warp == 1) {
        tmem_alloc(base + L.tslot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(bars + 8 * (kUbFull + s), 1);
            mbar_init(bars + 8 * (kUbEmpty + s), nT + 32 * kUmmaLceWarps);
            mbar_init(bars + 8 * (kUbSFullF + s), 1);
            mbar_init(bars + 8 * (kUbSFullG + s), 1);
            mbar_init(bars + 8 * (kUbOFull + s), 1);
            mbar_init(bars + 8 * (kUbOEmpty + s), 128);
            mbar_init(bars + 8 * (kUbDrain + s), 1);
            mbar_init(bars + 8 * (kUbOTFree + s), 1);
            mbar_init(bars + 8 * (kUbOTReady + s), 128);
            mbar_init(bars + 8 * (kUbGRead + s), 128);
            mbar_init(bars + 8 * (kUbPFree + s), 1);
            for (int j = 0; j < 4; ++j) mbar_init(bars + 8 * (kUbP + 4 * s + j), 128);
        }
        mbar_init(bars + 8 * kUbLFull, 32 * kUmmaLceWarps);
        mbar_init(bars + 8 * kUbLEmpty, 32 * kUmmaLceWarps);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *reinterpret_cast<volatile uint32_t *>(sm + L.tslot);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            griddep_wait();  // r_idx comes from the preceding routing kernel
            const int kv_bytes = prm.w2 * 64;
            int k = 0;
            for (int ru = ru0; ru < prm.regions; ru += stride_ru, ++k) {
                const int s = k & 1, use = k >> 1;
                if (use > 0 && !mbar_wait_bounded(bars + 8 * (kUbEmpty + s), (use - 1) & 1, lim)) {
                    atomicExch(&g_bra_timeout_flag, 1);
                    break;
                }
                uint32_t pr, ir;
                const int n = (int)prm.div_P.divmod((uint32_t)ru, pr);
                const int j = (int)prm.div_S.divmod(pr, ir), i = (int)ir;
                const int y0 = j * prm.hr, x0 = i * prm.wr;
                const uint32_t st = base + s * L.stage_bytes;
                const uint32_t full = bars + 8 * (kUbFull + s);
                uint32_t bytes = (uint32_t)(kv_bytes + (prm.hr + 4) * (prm.wr + 4) * 64);
                tma_load_4d(st + L.q, &prm.tmQ, c0, x0, y0, n, full);
                tma_load_4d(st + L.halo, &prm.tmH, c0, x0 - 2, y0 - 2, n, full);
                bool bad = false;
                for (int a = 0; a < prm.topk; ++a) {
                    int r = __ldcg(prm.r_idx + (size_t)ru * prm.topk + a);
                    if (r < 0 || r >= prm.P) {
                        // skipped region: zero its K/V rows so that the masked keys read zeros
                        r = -1;
                        bad = true;
                        uint4 *zk = reinterpret_cast<uint4 *>(sm + s * L.stage_bytes + L.k + a * kv_bytes);
                        uint4 *zv = reinterpret_cast<uint4 *>(sm + s * L.stage_bytes + L.v + a * kv_bytes);
                        for (int e = 0; e < kv_bytes / 16; ++e) zk[e] = zv[e] = make_uint4(0u, 0u, 0u, 0u);
                    } else {
                        uint32_t i2u;
                        const int j2 = (int)prm.div_S.divmod((uint32_t)r, i2u);
                        tma_load_4d(st + L.k + a * kv_bytes, &prm.tmK, c0, (int)i2u * prm.wr, j2 * prm.hr, n, full);
                        tma_load_4d(st + L.v + a * kv_bytes, &prm.tmV, c0, (int)i2u * prm.wr, j2 * prm.hr, n, full);
                        bytes += 2 * kv_bytes;
                    }
                    sIdx[s * prm.topk + a] = r;
                }
                if (bad) {
                    fence_proxy_async();  // the zeroed rows are read by the tensor cores
                    if (prm.err_flag) atomicExch(prm.err_flag, 1);
                }
                mbar_arrive_expect_tx(full, bytes);
            }
            // every copy this CTA issued must land before it may exit
            for (int kk = (k > 2 ? k - 2 : 0); kk < k; ++kk)
                mbar_wait_bounded(bars + 8 * (kUbFull + (kk & 1)), (kk >> 1) & 1, lim);
        }
    } else if (warp < kUmmaSoftWarp0) {
        // ------------------------------------------------------------ MMA issuers (one per tile)
        // Unit k of tile t: half F = k mod 2 of the tile's 256 columns takes the scores of
        // keys 0..127 and O (its columns 0..31), half G the scores of keys 128..255. P of
        // pair j goes to F + 32 (j + 1) for j < 3 and, once pair 0's MMAs are done, over
        // P_0 for j = 3, so G holds nothing but scores: the next unit's first-half scores
        // (into G) are issued as soon as the pass has read them, before the last PV steps.
        // Writing G(k) = F(k-1) needs unit k-1's MMAs complete and O(k-1) read. With 128
        // keys (no second half) the next unit's scores wait for that read as well.
        const int t = warp - 1;
        if (lane == 0 && t < nT) {
            const uint32_t idS = idesc_bf16_f32(128, 128, 0, 0);
            const uint32_t idV = idesc_bf16_f32(128, 32, 0, 1);
            const uint32_t d = tbase + 256 * t;
            bool ok = true;
            int k = 0;
            auto issue_s = [&](uint32_t dst, uint32_t stage, int key0) {
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
                    umma_ss(dst, smem_desc(stage + L.q + t * 8192 + 32 * kk, 16, 512, kDescSwizzle64B),
                            smem_desc(stage + L.k + key0 * 64 + 32 * kk, 16, 512, kDescSwizzle64B), idS, (uint32_t)kk);
            };
            for (int ru = ru0; ru < prm.regions && ok; ru += stride_ru, ++k) {
                const int s = k & 1, use = k >> 1;
                const uint32_t st = base + s * L.stage_bytes;
                const uint32_t F = d + 128 * (k & 1), G = d + 128 * ((k & 1) ^ 1);
                const bool next = ru + stride_ru < prm.regions;
                if (!mbar_wait_bounded(bars + 8 * (kUbFull + s), use & 1, lim) ||
                    (k > 0 && !mbar_wait_bounded(bars + 8 * (kUbOFull + t), (k - 1) & 1, lim)) ||
                    (k > 0 && !mbar_wait_bounded(bars + 8 * (kUbOEmpty + t), (k - 1) & 1, lim))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (np < 4 || k == 0) {  // otherwise issued during the previous unit
                    issue_s(F, st, 0);
                    umma_commit(bars + 8 * (kUbSFullF + t));
                }
                if (np == 4) {
                    issue_s(G, st, 128);
                    umma_commit(bars + 8 * (kUbSFullG + t));
                }
                // O_t = P_t V, one chunk pair (four 16-key steps) as soon as its P is stored
                for (int j = 0; j < np; ++j) {
                    if (j == 3 && next) {  // the next unit's first half, into G
                        if (!mbar_wait_bounded(bars + 8 * (kUbGRead + t), k & 1, lim) ||
                            !mbar_wait_bounded(bars + 8 * (kUbFull + (s ^ 1)), ((k + 1) >> 1) & 1, lim)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_s(G, base + (s ^ 1) * L.stage_bytes, 0);
                        umma_commit(bars + 8 * (kUbSFullF + t));
                    }
                    if (!mbar_wait_bounded(bars + 8 * (kUbP + 4 * t + j), k & 1, lim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t pcol = F + 32 * (j < 3 ? j + 1 : 1);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int kk = 4 * j + i;
                        umma_ts(F, pcol + 8 * i, smem_desc(st + L.v + 1024 * kk, 0, 512, kDescSwizzle64B), idV,
                                (uint32_t)(kk > 0));
                    }
                    if (j == 0 && np == 4) umma_commit(bars + 8 * (kUbPFree + t));
                }
                if (!ok) break;
                umma_commit(bars + 8 * (kUbOFull + t));
                umma_commit(bars + 8 * (kUbEmpty + s));  // this tile's reads of Q, K, V are done
            }
            if (!ok) atomicExch(&g_bra_timeout_flag, 1);
            // every MMA must have completed before the tensor memory is released
            umma_commit(bars + 8 * (kUbDrain + t));
            mbar_wait_bounded(bars + 8 * (kUbDrain + t), 0, lim);
        }
    } else if (warp < kUmmaLceWarp0) {
        // ------------------------------------------------------------ softmax warpgroups
        const int t = (warp - kUmmaSoftWarp0) >> 2, sub = warp & 3;
        if (t < nT) {
            const int row = 32 * sub + lane;
            const uint32_t trow = tbase + ((uint32_t)(32 * sub) << 16) + 256 * t;
            const float sl2 = prm.scale_log2;
            float *rsum = reinterpret_cast<float *>(sm + L.rsum) + t * 128 + row;
            int k = 0;
            for (int ru = ru0; ru < prm.regions; ru += stride_ru, ++k) {
                const int s = k & 1, use = k >> 1;
                if (!umma_wait_warp(bars + 8 * (kUbFull + s), use & 1, lim)) break;
                uint32_t cmask = 0;  // the 32-key chunks of the routed regions present in the stage
                for (int a = 0; a < prm.topk; ++a)
                    if (sIdx[s * prm.topk + a] >= 0) cmask |= ((1u << cpr) - 1u) << (a * cpr);
                const uint32_t F = trow + 128 * (k & 1), G = trow + 128 * ((k & 1) ^ 1);
                if (32 * sub >= tile_rows) {
                    // a warp with no live row: no scores to read or P to store, only the
                    // arrivals the barriers count; then it waits until the unit's O is complete
                    // (every P barrier of the unit has finished its phase) before the next unit
                    for (int j = 0; j < np; ++j) umma_arrive(bars + 8 * (kUbP + 4 * t + j));
                    if (np == 4) umma_arrive(bars + 8 * (kUbGRead + t));
                    if (!umma_wait_warp(bars + 8 * (kUbOFull + t), k & 1, lim)) break;
                    continue;
                }
                if (!umma_wait_warp(bars + 8 * (kUbSFullF + t), k & 1, lim)) break;
                tc_fence_after();
                bool gready = np < 4, fail = false;
                auto wait_g = [&]() {
                    if (!gready) {
                        if (!umma_wait_warp(bars + 8 * (kUbSFullG + t), k & 1, lim)) return false;
                        tc_fence_after();
                        gready = true;
                    }
                    return true;
                };
                // reference: the exact max of the first valid 32-key chunk. Every p is
                // taken relative to it; a row whose later keys exceed it by so much that p,
                // the row sum or O overflows is recomputed exactly in the epilogue.
                // Chunk c (32 keys) sits at F + 32 c for c < 4, at G + 32 (c - 4) after; even
                // chunks go through buffer ra, odd ones through rb, so that the next chunk's
                // scores load while the current chunk's exponentials are computed.
                const int nch = 2 * np;
                auto chunk_col = [&](int c) { return c < 4 ? F + 32 * c : G + 32 * (c - 4); };
                auto chunk_valid = [&](int c) { return ((cmask >> c) & 1u) != 0u; };
                uint32_t ra[32], rb[32];
                float m = -INFINITY;
                int cref = 0;  // the first valid chunk
                while (cref < nch && !chunk_valid(cref)) ++cref;
                if (cref == 0) {
                    tmem_ld32(F, ra);  // chunk 0, kept for its exponentials
                    m = max32(ra, -INFINITY);
                } else if (cref < nch) {  // read for its max only; the pass loads it again
                    if (cref >= 4 && !wait_g()) break;
                    tmem_ld32(chunk_col(cref), rb);
                    m = max32(rb, -INFINITY);
                }
                const float mneg = m == -INFINITY ? 0.f : -m * sl2;
                const float2 sl2v = make_float2(sl2, sl2), mnv = make_float2(mneg, mneg);
                float2 la = make_float2(0.f, 0.f), lb = make_float2(0.f, 0.f);
                float2 lc = make_float2(0.f, 0.f), ld = make_float2(0.f, 0.f);
                uint32_t pk[16];  // P of one chunk (bf16 pairs)
                for (int c = 0; c < nch && !fail; c += 2) {
                    const int j = c >> 1;  // the pair
                    // ---- even chunk c (in ra); the odd chunk c + 1 loads into rb meanwhile
                    const bool ve = chunk_valid(c), vo = chunk_valid(c + 1);
                    if (vo) {
                        if (c + 1 >= 4 && !wait_g()) {
                            fail = true;
                            break;
                        }
                        tmem_ld32_nowait(chunk_col(c + 1), rb);
                    }
                    if (ve)
                        exp32(ra, sl2v, mnv, la, lb, pk);
                    else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) pk[e] = 0u;
                    }
                    if (j > 0) {  // pair j - 1's P was stored a chunk ago: hand it to the MMA
                        tmem_wait_st();
                        tc_fence_before();
                        umma_arrive(bars + 8 * (kUbP + 4 * t + j - 1));
                    }
                    if (vo) tmem_wait_ld(rb);
                    if (j == 3) {  // P_3 goes over P_0: wait for pair 0's MMAs
                        if (!umma_wait_warp(bars + 8 * (kUbPFree + t), k & 1, lim)) {
                            fail = true;
                            break;
                        }
                        tc_fence_after();
                    }
                    // P of pair j over scores already read (both chunks of the pair are in
                    // registers now): F + 32 (j + 1) for j < 3, over P_0 for j = 3
                    const uint32_t pcol = F + 32 * (j < 3 ? j + 1 : 1);
                    tmem_st16_nowait(pcol, pk);
                    // every score of G is in registers once the last chunk is: the next unit
                    // may take G
                    if (np == 4 && c + 1 == nch - 1) {
                        if (!wait_g()) {
                            fail = true;
                            break;
                        }
                        tc_fence_before();
                        umma_arrive(bars + 8 * (kUbGRead + t));
                    }
                    // ---- odd chunk c + 1 (in rb); the next pair's first chunk loads into ra
                    const bool vn = c + 2 < nch && chunk_valid(c + 2);
                    if (vn) {
                        if (c + 2 >= 4 && !wait_g()) {
                            fail = true;
                            break;
                        }
                        tmem_ld32_nowait(chunk_col(c + 2), ra);
                    }
                    if (vo)
                        exp32(rb, sl2v, mnv, lc, ld, pk);
                    else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) pk[e] = 0u;
                    }
                    tmem_st16_nowait(pcol + 16, pk);
                    if (j == np - 1) {  // the last pair: no later chunk to wait behind
                        tmem_wait_st();
                        *rsum = ((la.x + la.y) + (lb.x + lb.y)) + ((lc.x + lc.y) + (ld.x + ld.y));
                        tc_fence_before();
                        umma_arrive(bars + 8 * (kUbP + 4 * t + j));
                    }
                    if (vn) tmem_wait_ld(ra);
                }
                if (fail) break;
            }
            if (lane == 0 && ru0 + k * stride_ru < prm.regions) atomicExch(&g_bra_timeout_flag, 1);
        }
    } else {
        // ------------------------------------------------------------ LCE + epilogue warps
        // LCE item = (channel pair, two adjacent pixel columns, 8 rows): the 12 x 6 halo
        // values it reads feed all 16 of its outputs, split over both warpgroups.
        // Epilogue: warpgroup t finishes tile t, one query row per thread (the warp's TMEM
        // lane quarter).
        const int lt = tid - kUmmaLceWarp0 * 32;
        const int pair = lt & 15;
        const int erow = 32 * (warp & 3) + lane;
        const int tw = lt >> 7;  // the warpgroup: the epilogue's first tile
        const uint32_t etm = tbase + ((uint32_t)(32 * (warp & 3)) << 16);
        const float *sRsum = reinterpret_cast<const float *>(sm + L.rsum);
        const int c = c0 + 2 * pair;
        float2 wt[25];
        {
            const uint32_t *wp = reinterpret_cast<const uint32_t *>(prm.lce_w + (size_t)c * 25);
            uint32_t wv[25];
#pragma unroll
            for (int e = 0; e < 25; ++e) wv[e] = __ldg(wp + e);
#pragma unroll
            for (int e = 0; e < 25; ++e) {
                const int e0 = e, e1 = 25 + e;
                const uint32_t u0 = wv[e0 >> 1], u1 = wv[e1 >> 1];
                wt[e].x = __uint_as_float((e0 & 1) ? (u0 & 0xFFFF0000u) : (u0 << 16));
                wt[e].y = __uint_as_float((e1 & 1) ? (u1 & 0xFFFF0000u) : (u1 << 16));
            }
        }
        const float2 bias = bf16x2_to_float2(__ldg(reinterpret_cast<const uint32_t *>(prm.lce_b + c)));
        const int wr = prm.wr, hw = wr + 4;
        const int items = 16 * (wr >> 1) * (prm.hr / kUmmaRows);
        int k = 0;
        for (int ru = ru0; ru < prm.regions; ru += stride_ru, ++k) {
            const int s = k & 1, use = k >> 1;
            if (!umma_wait_warp(bars + 8 * (kUbFull + s), use & 1, lim)) break;
            if (k > 0 && !umma_wait_warp(bars + 8 * kUbLEmpty, (k - 1) & 1, lim)) break;
            const uint32_t tH = base + s * L.stage_bytes + L.halo + pair * 4;
            for (int it = lt; it < items; it += 32 * kUmmaLceWarps) {
                const int col = it >> 4;  // rb * (wr / 2) + xp
                uint32_t xp;
                const int rb = (int)prm.div_wx.divmod((uint32_t)col, xp);
                const int r0 = rb * kUmmaRows, x0 = 2 * (int)xp;
                float2 acc[kUmmaRows][2];
#pragma unroll
                for (int r = 0; r < kUmmaRows; ++r) acc[r][0] = acc[r][1] = bias;
#pragma unroll
                for (int hy = 0; hy < kUmmaRows + 4; ++hy) {
                    const uint32_t ra = tH + ((r0 + hy) * hw + x0) * 64;
                    float2 v[6];
#pragma unroll
                    for (int b = 0; b < 6; ++b) v[b] = bf16x2_to_float2(ld_shared_u32(ra + b * 64));
#pragma unroll
                    for (int r = 0; r < kUmmaRows; ++r) {
                        const int a = hy - r;
                        if (a >= 0 && a < 5) {
#pragma unroll
                            for (int b = 0; b < 5; ++b) {
                                acc[r][0] = ffma2(wt[a * 5 + b], v[b], acc[r][0]);
                                acc[r][1] = ffma2(wt[a * 5 + b], v[b + 1], acc[r][1]);
                            }
                        }
                    }
                }
#pragma unroll
                for (int r = 0; r < kUmmaRows; ++r) {
                    float *dst = sStage + ((r0 + r) * wr + x0) * kUmmaStagePitch + 2 * pair;
                    *reinterpret_cast<float2 *>(dst) = acc[r][0];
                    *reinterpret_cast<float2 *>(dst + kUmmaStagePitch) = acc[r][1];
                }
            }
            umma_arrive(bars + 8 * kUbLFull);
            if (!umma_wait_warp(bars + 8 * kUbLFull, k & 1, lim)) break;  // every staging row written
            // ---- epilogue, tiles t = warpgroup, warpgroup + warpgroups, ...: O / l + LCE + bias -> out
            bool fail = false;
            for (int t = tw; t < nT; t += kUmmaLceWarps / 4) {
                const bool leader = lt == 128 * tw;  // stores the warpgroup's tiles
                if (leader) {
                    // the previous unit's store of this tile has read it (a warpgroup that
                    // owns both tiles has just issued this unit's store of tile 0)
                    if (t > tw)
                        bulk_wait_read<1>();
                    else
                        bulk_wait_read<0>();
                    umma_arrive(bars + 8 * (kUbOTFree + t));
                }
                const int qi = t * 128 + erow;
                if (!umma_wait_warp(bars + 8 * (kUbOFull + t), k & 1, lim) ||
                    !umma_wait_warp(bars + 8 * (kUbP + 4 * t + np - 1), k & 1, lim)) {  // row sums stored
                    fail = true;
                    break;
                }
                tc_fence_after();
                const bool live = 32 * (warp & 3) < tile_rows;  // the warp's 32 rows hold queries
                if (!live) {  // only the arrivals the barriers count (the storing warp still stores)
                    umma_arrive(bars + 8 * (kUbOEmpty + t));
                    if (!umma_wait_warp(bars + 8 * (kUbOTFree + t), k & 1, lim)) {
                        fail = true;
                        break;
                    }
                    umma_arrive(bars + 8 * (kUbOTReady + t));
                } else {
                    uint32_t o[32];
                    tmem_ld32(etm + 256 * t + 128 * (k & 1), o);
                    float l = sRsum[t * 128 + erow];
                    tc_fence_before();
                    umma_arrive(bars + 8 * (kUbOEmpty + t));  // the half may take the next scores
                    float ck[4] = {l, 0.f, 0.f, 0.f};  // NaN unless l and every O value are finite
#pragma unroll
                    for (int e = 0; e < 32; ++e) ck[e & 3] = fmaf(__uint_as_float(o[e]), 0.f, ck[e & 3]);
                    if (!(fabsf((ck[0] + ck[1]) + (ck[2] + ck[3])) <= 3.0e38f)) {
                        uint32_t vmask = 0;
                        for (int a = 0; a < prm.topk; ++a) vmask |= (sIdx[s * prm.topk + a] >= 0 ? 1u : 0u) << a;
                        float of[32];
                        umma_exact_row(sm + s * L.stage_bytes, L, qi, prm.w2, prm.topk, vmask, prm.scale_log2, of, l);
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(of[e]);
                    }
                    const float inv = l > 0.f ? 1.f / l : 0.f;
                    const float4 *srow = reinterpret_cast<const float4 *>(sStage + qi * kUmmaStagePitch);
                    uint4 ov[4];
                    uint32_t *ow = reinterpret_cast<uint32_t *>(ov);
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        const float4 a = srow[q4];
                        ow[2 * q4] = pack_bf16x2(fmaf(__uint_as_float(o[4 * q4]), inv, a.x),
                                                 fmaf(__uint_as_float(o[4 * q4 + 1]), inv, a.y));
                        ow[2 * q4 + 1] = pack_bf16x2(fmaf(__uint_as_float(o[4 * q4 + 2]), inv, a.z),
                                                     fmaf(__uint_as_float(o[4 * q4 + 3]), inv, a.w));
                    }
                    // the row goes to the tile's smem image; one thread stores the whole tile
                    if (!umma_wait_warp(bars + 8 * (kUbOTFree + t), k & 1, lim)) {
                        fail = true;
                        break;
                    }
                    unsigned char *otile = sm + L.otile + t * 8192;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        *reinterpret_cast<uint4 *>(otile + erow * 64 + ((q4 ^ ((erow >> 1) & 3)) << 4)) = ov[q4];
                    fence_proxy_async();  // the rows are read by the tensor store
                    umma_arrive(bars + 8 * (kUbOTReady + t));
                }
                if (warp == kUmmaLceWarp0 + 4 * tw) {  // the storing thread's warp: keep its control flow uniform
                    bool stored = true;
                    if (lane == 0) {
                        stored = mbar_wait_bounded(bars + 8 * (kUbOTReady + t), k & 1, lim);
                        if (stored) {
                            uint32_t pr, ir;
                            const int n = (int)prm.div_P.divmod((uint32_t)ru, pr);
                            const int j = (int)prm.div_S.divmod(pr, ir);
                            tma_store_4d(&prm.tmO, base + L.otile + t * 8192, c0, (int)ir * prm.wr,
                                         j * prm.hr + t * (128 / prm.wr), n);
                            bulk_commit();
                        }
                    }
                    if (!__shfl_sync(0xffffffffu, stored, 0)) {
                        fail = true;
                        break;
                    }
                }
            }
            if (fail) break;
            umma_arrive(bars + 8 * kUbLEmpty);       // staging rows consumed
            umma_arrive(bars + 8 * (kUbEmpty + s));  // halo, Q, K, V of the stage no longer needed
        }
        if (lane == 0 && ru0 + k * stride_ru < prm.regions) atomicExch(&g_bra_timeout_flag, 1);
        if (lt == 128 * tw) bulk_wait<0>();  // the output tiles are written before the CTA exits
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

}  // namespace bra
