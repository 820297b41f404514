/*
 * bra.h — C ABI of the B200 (sm_100a) Bi-Level Routing Attention forward.
 *
 * Bi-Level Routing Attention (BRA) is the attention of BiFormer. The operation is
 * the one the official code computes, as walked through on the page
 * "BiFormer ... 前向传播过程" (TRANSFORMER.niftyadmin.cn/n/347023.html), section
 * "BRA模块", eqs. 3-7, and Algorithm 1 as described on bernice.tw
 * ("Bi-Level Routing Attention", parts one to three):
 *
 *   1. patchify: the (N,H,W,C) map is cut into S x S regions of
 *      hr x wr = (H/S) x (W/S) tokens (padded grid below when S does not
 *      divide H or W); region p = j*S + i is region row j,
 *      region column i; tokens inside a region are row-major;
 *   2. region query/key = mean of the region's tokens over all C channels;
 *      affinity A[p][p'] = (scale * q_r[p]) . k_r[p']                     (eq. 4)
 *   3. r_idx = the topk largest affinities of each row, in descending order
 *      (ties: lower region index first); r_weight = softmax of those topk
 *      affinities                                                          (eq. 5)
 *   4. every query token attends, per head, jointly over the tokens of its
 *      region's topk routed regions: softmax((scale*q) . k) v              (eqs. 6-7)
 *   5. plus LCE(V): depthwise 5x5 cross-correlation of the whole V image,
 *      zero padding 2, plus a per-channel bias                             (eq. 7)
 *
 * scale = d^-0.5 with d = C/heads, for both the routing and the attention.
 * r_weight is an output only: it does not weight K or V.
 *
 * Conventions for every entry point:
 *   - q, k, v, out: (N,H,W,C) contiguous channels-last, element type `dtype`;
 *     channel m*d + c is component c of head m.
 *   - lce_w: (C,5,5) contiguous (a PyTorch (C,1,5,5) depthwise weight), element
 *     type `dtype`; lce_b: (C), element type `dtype`.
 *   - r_idx: int32 (N,S*S,topk); r_weight: float32 (N,S*S,topk).
 *   - All pointers are DEVICE pointers of the current device (except in
 *     bra_forward_host), owned by the caller; the library never frees them.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Every call only
 *     enqueues work on `stream`: it never synchronises it and never blocks the
 *     host, except bra_forward_host, which returns after its results are on the
 *     host.
 *   - Scratch memory (the pooled region queries and keys, 2*N*S*S*C floats) is
 *     taken stream-ordered from the device's default memory pool
 *     (cudaMallocAsync on `stream`) and released stream-ordered after its last
 *     use.
 *   - Errors: arguments are checked before any CUDA call; on a bad argument
 *     nothing is launched and a BRA_ERR_* code is returned. BRA_ERR_CUDA reports
 *     a failed allocation or launch (the CUDA error is left for the caller to
 *     inspect with cudaGetLastError()). No C++ exception crosses this boundary.
 *   - Supported shapes: 1 <= S*S <= 256, 1 <= topk <= S*S, C % heads == 0,
 *     d in {32, 64}, C <= 1024, ceil(W/S) <= 128. N may be 0 (nothing is
 *     launched; pointers may be NULL).
 *   - H or W not a multiple of S (the padded grid; the bernice.tw notes, section
 *     "消融實驗", name padding's cost as the reason S is chosen per task and define
 *     it no further): q, k and v are zero-padded at the bottom and the right to
 *     Hp = S*ceil(H/S), Wp = S*ceil(W/S); regions are ceil(H/S) x ceil(W/S)
 *     tokens; region means are taken over whole padded regions; padded tokens
 *     take part as keys (k = v = 0); out holds the H x W real pixels only. The
 *     library makes the padded copies in scratch taken like the pooled means
 *     (3*N*Hp*Wp*C elements for q, k, v plus N*Hp*Wp*C for the padded output)
 *     and crops the result into `out`. With H and W multiples of S nothing of
 *     this happens.
 *   - Alignment: q, k, v, out 16-byte aligned; r_idx, r_weight 4-byte aligned.
 */
#ifndef BRA_H
#define BRA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *bra_stream_t;

typedef enum { BRA_F32 = 0, BRA_BF16 = 1 } bra_dtype_t;

enum {
    BRA_OK = 0,
    BRA_ERR_NULL = 1,        /* a required pointer is NULL                      */
    BRA_ERR_SHAPE = 2,       /* shape outside the supported set listed above     */
    BRA_ERR_ALIGN = 3,       /* a pointer is not aligned as required             */
    BRA_ERR_DTYPE = 4,       /* dtype is not BRA_F32 or BRA_BF16                 */
    BRA_ERR_CUDA = 5,        /* a CUDA allocation, copy or launch failed         */
    BRA_ERR_INDEX = 6,       /* bra_attend: a region index outside [0, S*S)      */
    BRA_ERR_SCRATCH = 7,     /* bra_forward_noalloc: problem needs more scratch
                                than the library's static array holds          */
    BRA_ERR_TIMEOUT = 8      /* bra_device_status: a kernel's bounded wait for its
                                tile copies ran out (its outputs are invalid)  */
};

/* Steps 1-5: the whole BRA forward.
 * In:  q, k, v, lce_w, lce_b (device).  Out: out (N,H,W,C) in `dtype`, r_idx,
 * r_weight (device). Routing (steps 1-3) is computed in float32 from the
 * stored values; the attention accumulates in float32 (bf16 tensor-core
 * products for BRA_BF16, float32 FMA for BRA_F32); the output is rounded once
 * to `dtype` (round to nearest even). */
int bra_forward(const void *q, const void *k, const void *v, const void *lce_w, const void *lce_b,
                int N, int H, int W, int C, int heads, int S, int topk, int dtype, void *out,
                int32_t *r_idx, float *r_weight, bra_stream_t stream);

/* Steps 1-3 only (region pooling, affinity, top-k routing): writes r_idx and
 * r_weight. Same conventions as bra_forward. */
int bra_route(const void *q, const void *k, int N, int H, int W, int C, int heads, int S, int topk,
              int dtype, int32_t *r_idx, float *r_weight, bra_stream_t stream);

/* Steps 4-5 only, for a routing given by the caller: r_idx (N,S*S,topk) int32
 * device array of region indices (any order; duplicates allowed and counted
 * twice). Every index must lie in [0, S*S); the kernel treats an index outside
 * that range as a zero key/value tile that takes no part in the softmax and
 * flags it, and the call then returns BRA_ERR_INDEX — this check reads one word
 * back, so unlike the other entry points bra_attend synchronises `stream`. */
int bra_attend(const void *q, const void *k, const void *v, const void *lce_w, const void *lce_b,
               int N, int H, int W, int C, int heads, int S, int topk, int dtype,
               const int32_t *r_idx, void *out, bra_stream_t stream);

/* bra_forward on HOST buffers: copies the inputs from host memory to the
 * device (pinned host memory gives asynchronous copies), runs the forward on
 * `stream`, copies out, r_idx and r_weight back to the host buffers and
 * synchronises `stream` before returning. Device buffers are taken from and
 * returned to a stream-ordered memory pool that the library creates once per
 * device and that keeps its memory between calls (so repeated calls do not map
 * device memory again); that memory stays reserved until the process exits.
 * Same shapes, dtypes and error codes as bra_forward; host pointers need no
 * alignment. */
int bra_forward_host(const void *q, const void *k, const void *v, const void *lce_w,
                     const void *lce_b, int N, int H, int W, int C, int heads, int S, int topk,
                     int dtype, void *out, int32_t *r_idx, float *r_weight, bra_stream_t stream);

/* bra_forward without any device allocation. (No counterpart on the pages: this
 * is a deployment variant of bra_forward, not a step of the method.)
 *
 * Some callers cannot allocate device memory at the moment they call in: a
 * framework whose caching allocator has already reserved the device's memory, a
 * real-time loop that forbids allocation after start-up, or a process whose
 * default memory pool is disabled or capped. bra_forward takes its scratch (the
 * pooled region means, 2*N*S*S*C floats) from the memory pool on every call;
 * this entry point instead uses one fixed scratch array compiled into the
 * library: BRA_STATIC_SCRATCH_FLOATS floats (16 MiB), present on every GPU that
 * loads the library and held until the process exits. It calls no allocator.
 *
 *   - Same arguments, layouts and error codes as bra_forward, and the same
 *     kernels: the results are bit for bit those of bra_forward on the same
 *     inputs. The caller still passes (and owns) every input and output buffer.
 *   - Limit: 2*N*S*S*C must not exceed BRA_STATIC_SCRATCH_FLOATS, even for shapes
 *     whose one-kernel form needs no scratch; a larger problem returns
 *     BRA_ERR_SCRATCH before anything is launched. So does a shape whose H or W
 *     is not a multiple of S: its padded copies would need more scratch than the
 *     array holds.
 *   - Every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress, no allocation). The first call on a device may load
 *     the library's kernels onto it, so make that first call before any CUDA
 *     graph capture starts on the device.
 *   - All calls share the one array, which keeps the last call's contents. No
 *     part of it needs to start at zero: a call writes every element it reads.
 *     Two calls whose kernels overlap on the GPU (different streams, or
 *     different host threads without ordering) race on the array and give wrong
 *     results: order them on one stream or with events. */
#define BRA_STATIC_SCRATCH_FLOATS (4u * 1024u * 1024u)
int bra_forward_noalloc(const void *q, const void *k, const void *v, const void *lce_w,
                        const void *lce_b, int N, int H, int W, int C, int heads, int S,
                        int topk, int dtype, void *out, int32_t *r_idx, float *r_weight,
                        bra_stream_t stream);

/* ---------------------------------------------------------------------------
 * The attention layer around BRA: the qkv projection before it and the output
 * projection `wo` after it, both nn.Linear modules with bias (y = x w^T + b), as
 * printed in the walk-through's module listing ("BiFormer ... 前向传播过程",
 * section "网络结构": qkv Linear(64 -> 192, bias=True), wo Linear(64 -> 64,
 * bias=True)) and used in its section "BRA模块" (q, k, v are consecutive C-wide
 * chunks of the qkv output; a linear layer closes the block).
 *
 * Conventions (besides those above): x, y, q, k, v, out are row-major with one row
 * per token ((N,H,W,C) maps are (N*H*W) x C matrices); a weight w is (Nout, K)
 * row-major (the PyTorch Linear weight) and a bias b is (Nout); all in `dtype`.
 * The products accumulate in float32 (bfloat16 tensor-core products for BRA_BF16,
 * float32 FMA for BRA_F32); the bias is added in float32 and every stored value is
 * rounded once to `dtype` (round to nearest even). Supported: 1 <= K, Nout <= 4096;
 * for BRA_BF16 also K % 32 == 0 and Nout (each third of it for bra_qkv) a multiple
 * of 32. x, w and the outputs 16-byte aligned; biases aligned to their element. */

/* y (M x Nout) = x (M x K) w^T + b. M may be 0 (nothing is launched). */
int bra_linear(const void *x, const void *w, const void *b, int M, int K, int Nout, int dtype, void *y,
               bra_stream_t stream);

/* The qkv projection: [q | k | v] = x w_qkv^T + b_qkv with x (M x C), w_qkv (3C, C),
 * b_qkv (3C); q, k, v (M x C) each get their C-wide chunk, in that order. */
int bra_qkv(const void *x, const void *w_qkv, const void *b_qkv, int M, int C, int dtype, void *q, void *k,
            void *v, bra_stream_t stream);

/* The whole layer: out = wo(BRA(qkv(x))) with x, out (N,H,W,C); q, k, v and the
 * attention output are stored in `dtype` between the steps. Scratch (4*N*H*W*C
 * elements plus the routing's 2*N*S*S*C floats) is taken stream-ordered: outside a
 * stream capture from the library's per-device pool that keeps its memory between
 * calls (the pool of bra_forward_host), inside a capture from the device's default
 * pool (a memory node of the graph). r_idx and r_weight as in bra_forward. BRA's
 * shape rules apply, plus those of the projections with K = C. */
int bra_attention_layer(const void *x, const void *w_qkv, const void *b_qkv, const void *w_o, const void *b_o,
                        const void *lce_w, const void *lce_b, int N, int H, int W, int C, int heads, int S,
                        int topk, int dtype, void *out, int32_t *r_idx, float *r_weight, bra_stream_t stream);

/* ---------------------------------------------------------------------------
 * The BiFormer block around the attention layer, as the walk-through prints and runs it
 * ("BiFormer ... 前向传播过程", section "2、BiFormer Block": x = x + pos_embed(x), then
 * x = x + drop_path(attn(norm1(x))); the module printout of section "网络结构":
 * pos_embed = Conv2d(C, C, 3, padding 1, groups C), norm1 / norm2 = LayerNorm(C,
 * eps 1e-6), mlp = Linear(C, 3C) -> GELU -> Linear(3C, C), drop_path = Identity). The
 * walk-through says nothing of the MLP line; it is read as the same pre-norm residual
 * form, x = x + mlp(norm2(x)), with PyTorch's default (exact erf) GELU. */

/* The MLP's linear layers: y (M x Nout) = act(x w^T + b) with x (M x K), w (Nout, K),
 * b (Nout), all in `dtype`, float32 accumulation:
 *   BRA_ACT_NONE:     y = round(x w^T + b)                   (as bra_linear)
 *   BRA_ACT_GELU:     y = round(GELU(x w^T + b)), GELU(t) = t/2 (1 + erf(t / sqrt 2))
 *   BRA_ACT_RESIDUAL: y = round(res + round(x w^T + b)), res (M x Nout) in `dtype`
 * round = the dtype's rounding (nearest even for bf16; none for float32). Shape and
 * alignment rules of bra_linear; res (when used) 16-byte aligned. */
enum { BRA_ACT_NONE = 0, BRA_ACT_GELU = 1, BRA_ACT_RESIDUAL = 2 };
int bra_linear_act(const void *x, const void *w, const void *b, const void *res, int M, int K, int Nout, int act,
                   int dtype, void *y, bra_stream_t stream);

/* One block: x, out (N,H,W,C) in `dtype`;
 *   x1 = x + pos_embed(x)        pos_w (C,3,3), pos_b (C): depthwise 3x3 cross-correlation,
 *                                zero padding 1, plus bias
 *   h  = norm1(x1)               ln1_g, ln1_b (C): (t - mean) / sqrt(var + 1e-6) * g + b over
 *                                the C channels of a pixel, var the mean squared deviation
 *   x2 = x1 + attn(h)            the attention layer (bra_attention_layer's weights)
 *   out = x2 + mlp(norm2(x2))    ln2_g, ln2_b (C); mlp_w1 (3C, C), mlp_b1 (3C), GELU,
 *                                mlp_w2 (C, 3C), mlp_b2 (C)
 * Every stored intermediate (x1, h, the layer's own, x2, norm2's output, the MLP hidden
 * layer after GELU, the MLP output before the residual) is rounded once to `dtype`.
 * r_idx, r_weight: the attention's routing, as in bra_forward. Shapes: BRA's rules (the
 * padded grid included) and the projections', with C <= 256. x, out, w_qkv, w_o, mlp_w1,
 * mlp_w2 16-byte aligned; the other parameters aligned to their element. Scratch
 * (7*N*H*W*C elements plus the attention layer's) is taken like bra_attention_layer's. */
int bra_block(const void *x, const void *pos_w, const void *pos_b, const void *ln1_g, const void *ln1_b,
              const void *w_qkv, const void *b_qkv, const void *w_o, const void *b_o, const void *lce_w,
              const void *lce_b, const void *ln2_g, const void *ln2_b, const void *mlp_w1, const void *mlp_b1,
              const void *mlp_w2, const void *mlp_b2, int N, int H, int W, int C, int heads, int S, int topk,
              int dtype, void *out, int32_t *r_idx, float *r_weight, bra_stream_t stream);

/* ---------------------------------------------------------------------------
 * The backward pass of steps 4-5 with the routing detached: the walk-through's router
 * ("BiFormer ... 前向传播过程", section "BRA模块", TopkRouting) detaches the region
 * query and key when diff_routing is off (its default); the top-k index is discrete and
 * r_weight does not scale K or V, so gradients flow through the token attention and the
 * LCE only. Given dout = dL/dout (N,H,W,C) in `dtype` and the forward's r_idx, writes
 *   dq, dk, dv: (N,H,W,C) float32;  dlce_w: (C,5,5) float32;  dlce_b: (C) float32.
 * The attention softmax is recomputed from q and k.
 *   - BRA_BF16 with 32 channels per head, q, k, v, dout and dv 16-byte aligned and dq,
 *     dk 8-byte aligned: tensor-core kernels (bf16 products, float32 accumulation; the
 *     probabilities and dS enter their products as bf16 high + low parts).
 *     Deterministic: every output element has one writer and every sum a fixed order,
 *     so repeated calls give identical bits. Scratch (the transposed routing, per-query
 *     statistics, LCE partial sums) is taken like bra_attention_layer's.
 *   - otherwise (float32, 64 channels per head, or less aligned buffers): float32 SIMT
 *     kernels; dk and dv are accumulated with atomics (the summation order, and so the
 *     last bits, can differ between calls).
 * Every r_idx entry must lie in [0, S*S): an entry outside is skipped and the call
 * returns BRA_ERR_INDEX; like bra_attend, this call synchronises `stream` to read that
 * flag. Shapes as bra_forward, with H and W multiples of S (no padded grid:
 * BRA_ERR_SHAPE otherwise); q, k, v, dout, lce_w aligned to their element,
 * the float32 outputs and r_idx to 4 bytes. N = 0 zeroes dlce_w and dlce_b only. */
int bra_backward(const void *q, const void *k, const void *v, const void *lce_w, const int32_t *r_idx,
                 const void *dout, int N, int H, int W, int C, int heads, int S, int topk, int dtype, float *dq,
                 float *dk, float *dv, float *dlce_w, float *dlce_b, bra_stream_t stream);

/* bra_backward without the host synchronisation, so that it can be enqueued back to back
 * or captured in a CUDA graph: same arguments, kernels and results. An r_idx entry outside
 * [0, S*S) is skipped as in bra_backward and raises the library's device flag, which the
 * next bra_device_status call reports as BRA_ERR_INDEX (and clears); the return value
 * covers argument checks and launches only. */
int bra_backward_async(const void *q, const void *k, const void *v, const void *lce_w, const int32_t *r_idx,
                       const void *dout, int N, int H, int W, int C, int heads, int S, int topk, int dtype,
                       float *dq, float *dk, float *dv, float *dlce_w, float *dlce_b, bra_stream_t stream);

/* ---------------------------------------------------------------------------
 * Tracing (measurement support; no part of the computation).
 *
 * Kernel classes the library launches, for bra_trace_end and bra_kernel_name. */
enum {
    BRA_KERNEL_REGION_MEAN = 0, /* step 2 prelude: region means of q and k        */
    BRA_KERNEL_ROUTE = 1,       /* steps 2-3: affinity row, top-k, softmax        */
    BRA_KERNEL_ATTN_BF16 = 2,   /* steps 4-5, bfloat16 tensor-core kernel         */
    BRA_KERNEL_ATTN_F32 = 3,    /* steps 4-5, float32 SIMT kernel                 */
    BRA_KERNEL_FUSED_IMAGE = 4, /* steps 1-5 in one kernel (small images)         */
    BRA_KERNEL_ATTN_UMMA = 5,   /* steps 4-5, tcgen05 kernel (large regions)       */
    BRA_KERNEL_LINEAR_BF16 = 6, /* qkv / output projection, tcgen05 GEMM          */
    BRA_KERNEL_LINEAR_F32 = 7,  /* qkv / output projection, float32 SIMT          */
    BRA_KERNEL_BACKWARD = 8,    /* bra_backward's kernels, timed together          */
    BRA_KERNEL_PAD = 9,         /* padded grid: zero-padded copies and the crop   */
    BRA_KERNEL_BLOCK = 10,      /* BiFormer block: pos-embed + LN1, residual + LN2 */
    BRA_KERNEL_CLASSES = 11
};

/* Number of kernels this library has launched since it was loaded (all threads,
 * all devices). */
long long bra_launch_count(void);

/* Start tracing: until bra_trace_end, every kernel launch is bracketed by two
 * CUDA events recorded on its own stream; inside a CUDA graph capture the events
 * become event-record nodes of the graph (see bra_trace_read). Returns BRA_OK. */
int bra_trace_begin(void);

/* Without stopping the trace: wait for the recorded events and write, per kernel
 * class, the device time between each recorded pair summed over all pairs, and the
 * number of pairs. A pair recorded inside a CUDA graph capture is re-recorded by
 * every replay of that graph, so reading after a replay gives that replay's times.
 * Returns BRA_OK or BRA_ERR_CUDA. */
int bra_trace_read(double *ms, long long *launches);

/* Stop tracing, wait for the recorded events and write, per kernel class
 * (BRA_KERNEL_CLASSES entries each), the summed device time in milliseconds and
 * the number of traced launches. Either array may be NULL. Returns BRA_OK or
 * BRA_ERR_CUDA. */
int bra_trace_end(double *ms, long long *launches);

/* Name of a kernel class, or "unknown". */
const char *bra_kernel_name(int kernel_class);

/* ---------------------------------------------------------------------------
 * Kernel selection and device status.
 *
 * By default (BRA_VARIANT_AUTO) a bfloat16 forward whose images are small runs its
 * attention and LCE in one fused kernel that holds one head's Q, K and V slices of a
 * whole image in shared memory: this needs d = 32, regions of 4x4 or 2x2 tokens,
 * S*S <= 64, topk <= 64, heads <= 8 and those slices within one CTA's shared memory.
 * With topk <= 8 the fused kernel also pools and routes (one thread-block cluster of
 * `heads` CTAs per image, ONE launch in all); with topk > 8 the routing kernels run
 * first and the fused kernel follows them. Otherwise the forward runs as three kernels
 * (region means, routing, attention). The bfloat16 attention then runs, in this order of preference:
 *  - on the 5th-generation tensor cores (tcgen05: scores and probabilities in tensor
 *    memory, one CTA per SM) when d = 32, a region holds 128 or 256 tokens (H/S a
 *    multiple of 8, W/S even) and topk * (H/S) * (W/S) <= 256; under BRA_VARIANT_SPLIT
 *    also for regions of 64 tokens (8 x 8) with topk 2 or 4, which fill half of each
 *    128-row tensor-core tile;
 *  - in the persistent pipeline kernel (tile boxes fetched by the tensor memory
 *    accelerator into multi-stage shared memory by a producer warp, consumed by
 *    mma.sync attention warps and LCE warps) where the shape allows it (64 or 128
 *    channels per CTA, every stage within the shared-memory budget);
 *  - else in the generic kernel (16-byte cp.async pieces, one CTA per work unit).
 * The first two need 4-byte aligned lce_w and lce_b. BRA_VARIANT_SPLIT keeps the
 * three-kernel path with the automatic attention kernel; BRA_VARIANT_PIPE skips the
 * tcgen05 kernel (pipeline, else generic); BRA_VARIANT_TMA selects the
 * one-unit-per-CTA TMA attention kernel (same shape rules as the pipeline),
 * BRA_VARIANT_GENERIC the generic kernel. All variants compute the same function. */
enum {
    BRA_VARIANT_AUTO = 0,
    BRA_VARIANT_GENERIC = 1,
    BRA_VARIANT_TMA = 2,
    BRA_VARIANT_SPLIT = 3,
    BRA_VARIANT_PIPE = 4
};

/* Select the attention kernel for all later calls in this process (for testing and
 * comparison): one of the BRA_VARIANT_* values above.
 * Returns the previous setting, or -1 for an unknown variant. */
int bra_set_kernel_variant(int variant);

/* Synchronise `stream`, then report whether any kernel of this library gave up a
 * bounded wait since the last call (BRA_ERR_TIMEOUT), else whether a bra_backward_async
 * call met an r_idx entry outside [0, S*S) (BRA_ERR_INDEX), else BRA_OK; the flags are
 * cleared. BRA_ERR_CUDA if the synchronisation or the read fails. Kernels never
 * spin without a limit: a wait that runs out raises this flag and the kernel
 * returns. */
int bra_device_status(bra_stream_t stream);

/* Launch a one-CTA kernel that waits, `polls` times at most, on a barrier that
 * never completes, so that its bounded wait runs out and raises the flag that
 * bra_device_status reports. It moves no data. For testing the timeout path. */
int bra_selftest_wait_timeout(unsigned polls, bra_stream_t stream);

/* A static, human-readable description of a status code. */
const char *bra_status_string(int status);

/* Library ABI version: (major << 16) | minor. */
int bra_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BRA_H */
