// bra.cu — the C ABI of the BRA forward (declared in include/bra.h): argument
// checking, launch-shape selection and the kernel launches.
//
// Call path of bra_forward on one stream, no host synchronisation:
//   region_mean_kernel  (q, k -> pooled region means, float32 scratch)
//   route_kernel        (pooled means -> affinity row, bitonic top-k, r_idx, r_weight)
//   attn_tma_kernel     (bf16: TMA tiles of q, routed k/v and the v halo -> attention
//                        + LCE epilogue -> out), or attn_bf16_kernel / attn_f32_kernel
//                        (cp.async tiles) for shapes the TMA kernel does not cover
// The route and attention kernels are launched with programmatic dependent launch,
// so each may start (and the attention kernel may fetch its q tile and v halo)
// while the previous kernel drains.
#include <algorithm>
#include <atomic>
#include <climits>
#include <cstdio>
#include <cstdlib>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <set>
#include <tuple>
#include <type_traits>
#include <utility>
#include <vector>

#include <cudaTypedefs.h>

#include "../../include/bra.h"
#include "attn.cuh"
#include "attn_pipe.cuh"
#include "attn_tma.cuh"
#include "attn_umma.cuh"
#include "backward.cuh"
#include "backward_tc.cuh"
#include "block.cuh"
#include "fused_image.cuh"
#include "linear.cuh"
#include "pad.cuh"
#include "route.cuh"

namespace bra {

constexpr int kMaxSmem = 227 * 1024;

// ----------------------------------------------------------------------------- tracing

static std::atomic<long long> g_launches{0};
static std::mutex g_trace_mu;
static bool g_tracing = false;
struct TraceRec {
    int kid;
    cudaEvent_t a, b;
};
static std::vector<TraceRec> g_trace;

// Brackets one kernel launch: counts it and, while tracing (and not capturing),
// records an event pair on its stream.
class LaunchScope {
  public:
    LaunchScope(int kid, cudaStream_t st) : kid_(kid), st_(st) {
        g_launches.fetch_add(1, std::memory_order_relaxed);
        std::lock_guard<std::mutex> g(g_trace_mu);
        if (!g_tracing) return;
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return;
        // inside a stream capture the pair becomes event-record nodes of the graph
        flags_ = cs == cudaStreamCaptureStatusNone ? cudaEventRecordDefault : cudaEventRecordExternal;
        if (cudaEventCreate(&a_) != cudaSuccess) return;
        if (cudaEventCreate(&b_) != cudaSuccess) {
            cudaEventDestroy(a_);
            return;
        }
        if (cudaEventRecordWithFlags(a_, st, flags_) != cudaSuccess) {
            cudaEventDestroy(a_);
            cudaEventDestroy(b_);
            return;
        }
        on_ = true;
    }
    ~LaunchScope() {
        if (!on_) return;
        cudaEventRecordWithFlags(b_, st_, flags_);
        std::lock_guard<std::mutex> g(g_trace_mu);
        g_trace.push_back({kid_, a_, b_});
    }

  private:
    int kid_;
    cudaStream_t st_;
    cudaEvent_t a_{}, b_{};
    unsigned flags_ = cudaEventRecordDefault;
    bool on_ = false;
};

struct Shape {
    int N, H, W, C, heads, S, topk, dtype;
    int P, hr, wr, w2, d;
    int Hp, Wp;  // the padded grid: S * hr, S * wr (== H, W when S divides them)
    bool padded() const { return Hp != H || Wp != W; }
};

static bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shape rules of include/bra.h; nothing here touches CUDA.
static int check_shape(const Shape &s) {
    if (s.dtype != BRA_F32 && s.dtype != BRA_BF16) return BRA_ERR_DTYPE;
    if (s.N < 0 || s.H <= 0 || s.W <= 0 || s.C <= 0 || s.heads <= 0 || s.S <= 0) return BRA_ERR_SHAPE;
    if (s.S > 16) return BRA_ERR_SHAPE;
    if (s.topk < 1 || s.topk > s.S * s.S) return BRA_ERR_SHAPE;
    if (s.C % s.heads != 0 || s.C > 1024) return BRA_ERR_SHAPE;
    const int d = s.C / s.heads;
    if (d != 32 && d != 64) return BRA_ERR_SHAPE;
    if (s.wr > 128) return BRA_ERR_SHAPE;
    // element offsets are formed in 64-bit; grid sizes (the padded copies: one CTA per
    // row of three maps) must fit in int
    if ((long long)s.N * s.S * s.S * s.Hp > INT_MAX / 3) return BRA_ERR_SHAPE;
    if ((long long)s.Hp * s.Wp > INT_MAX / 4) return BRA_ERR_SHAPE;
    return BRA_OK;
}

static Shape make_shape(int N, int H, int W, int C, int heads, int S, int topk, int dtype) {
    Shape s{N, H, W, C, heads, S, topk, dtype, 0, 0, 0, 0, 0, H, W};
    if (S > 0 && heads > 0 && H > 0 && W > 0) {
        s.P = S * S;
        s.hr = (H + S - 1) / S;  // ceil: the padded grid when S does not divide H
        s.wr = (W + S - 1) / S;
        s.w2 = s.hr * s.wr;
        s.d = C / heads;
        s.Hp = S * s.hr;
        s.Wp = S * s.wr;
    }
    return s;
}

// The same problem on the zero-padded maps (Hp x Wp), which S divides.
static Shape padded_shape(const Shape &s) {
    Shape p = s;
    p.H = s.Hp;
    p.W = s.Wp;
    return p;
}

static int largest_divisor_at_most(int n, int cap) {
    for (int x = cap < n ? cap : n; x >= 1; --x)
        if (n % x == 0) return x;
    return 1;
}

// ----------------------------------------------------------------------------- routing

// PDL launch: the kernel may begin before the preceding kernel on the stream has
// finished; it calls griddepcontrol.wait before reading that kernel's results.
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ----------------------------------------------------------------------------- launch facts
// Attribute and occupancy queries cost far more than a launch (a cluster-occupancy query
// takes milliseconds), and their answers depend only on (device, kernel, block, shared
// memory): each is made once per key and kept.

static std::mutex g_facts_mu;
static std::map<int, int> g_sms;                                          // device -> SMs
static std::map<std::pair<int, const void *>, int> g_smem_set;            // (device, kernel) -> bytes allowed
static std::map<std::tuple<int, const void *, int, int, int>, int> g_occ;  // (device, kernel, threads, smem, cluster)

static int sm_count(int *sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BRA_ERR_CUDA;
    std::lock_guard<std::mutex> g(g_facts_mu);
    auto it = g_sms.find(dev);
    if (it == g_sms.end()) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return BRA_ERR_CUDA;
        it = g_sms.emplace(dev, n).first;
    }
    *sms = it->second;
    return BRA_OK;
}

// Allow `bytes` of dynamic shared memory for `kern` on the current device.
template <typename K> static cudaError_t allow_smem(K kern, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const auto key = std::make_pair(dev, reinterpret_cast<const void *>(kern));
    std::lock_guard<std::mutex> g(g_facts_mu);
    auto it = g_smem_set.find(key);
    if (it != g_smem_set.end() && it->second >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    // every kernel with dynamic shared memory asks for the same (largest) carveout, so that
    // consecutive kernels of a forward do not make the SMs change their L1 / shared split
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess) g_smem_set[key] = bytes;
    return e;
}

// Ask for the largest shared-memory carveout for `kern` on the current device, so that
// the occupancy reported (and reached) counts every CTA the shared memory can hold.
static std::set<std::pair<int, const void *>> g_carveout;
template <typename K> static cudaError_t prefer_shared(K kern) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const auto key = std::make_pair(dev, reinterpret_cast<const void *>(kern));
    std::lock_guard<std::mutex> g(g_facts_mu);
    if (g_carveout.count(key)) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess) g_carveout.insert(key);
    return e;
}

// Resident CTAs per SM (cluster = 0) or resident clusters on the device (cluster > 0,
// for the launch configuration cfg).
template <typename K>
static cudaError_t occupancy(int *out, K kern, int threads, int smem, int cluster, const cudaLaunchConfig_t *cfg) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const auto key = std::make_tuple(dev, reinterpret_cast<const void *>(kern), threads, smem, cluster);
    {
        std::lock_guard<std::mutex> g(g_facts_mu);
        auto it = g_occ.find(key);
        if (it != g_occ.end()) {
            *out = it->second;
            return cudaSuccess;
        }
    }
    int v = 0;
    e = cluster > 0 ? cudaOccupancyMaxActiveClusters(&v, kern, cfg)
                    : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kern, threads, smem);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> g(g_facts_mu);
    g_occ[key] = v;
    *out = v;
    return cudaSuccess;
}

// Device buffers of bra_forward_host come from a library-owned stream-ordered pool per
// device whose memory is kept between calls (release threshold = unlimited): the
// default pool returns its memory at every synchronisation, and mapping tens of MB
// again on the next call costs milliseconds.
struct HostCallRes {
    cudaMemPool_t pool;
    cudaStream_t up, back;  // non-blocking streams for the host-to-device and device-to-host copies
};
static std::map<int, HostCallRes> g_host_pools;

// The pool and the two copy streams, per device.
static int host_call_pool(cudaMemPool_t *pool, cudaStream_t *up, cudaStream_t *back) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BRA_ERR_CUDA;
    std::lock_guard<std::mutex> g(g_facts_mu);
    auto it = g_host_pools.find(dev);
    if (it == g_host_pools.end()) {
        cudaMemPoolProps props;
        memset(&props, 0, sizeof(props));
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t p = nullptr;
        if (cudaMemPoolCreate(&p, &props) != cudaSuccess) return BRA_ERR_CUDA;
        uint64_t keep = UINT64_MAX;
        if (cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess) return BRA_ERR_CUDA;
        cudaStream_t u = nullptr, b = nullptr;
        if (cudaStreamCreateWithFlags(&u, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&b, cudaStreamNonBlocking) != cudaSuccess)
            return BRA_ERR_CUDA;
        it = g_host_pools.emplace(dev, HostCallRes{p, u, b}).first;
    }
    *pool = it->second.pool;
    *up = it->second.up;
    *back = it->second.back;
    return BRA_OK;
}

// Token slots per (region, channel group) for the region-mean kernel: ns divides wr,
// G*ns divides 32, and each thread keeps at least 4 tokens.
static int pool_ns_log2(const Shape &s) {
    const int V = s.dtype == BRA_BF16 ? 8 : 4;
    const int G = s.C / V;
    int l = 0;
    if (32 % G != 0) return 0;
    while ((G << (l + 1)) <= 32 && s.wr % (1 << (l + 1)) == 0 && s.w2 / (1 << (l + 1)) >= 4) ++l;
    return l;
}

// Steps 1-3 into scratch ws (2*N*S*S*C floats): region means, then the routing.
static int launch_route_into(const Shape &s, const void *q, const void *k, int32_t *r_idx, float *r_weight,
                             float *ws, cudaStream_t st) {
    const size_t pooled = (size_t)s.N * s.P * s.C;
    {
        const int V = s.dtype == BRA_BF16 ? 8 : 4;
        const int l = pool_ns_log2(s);
        const long long total = (long long)s.N * s.P * (s.C / V) << l;
        if (total >= INT_MAX - kPoolThreads) return BRA_ERR_SHAPE;
        const unsigned blocks = (unsigned)((total + kPoolThreads - 1) / kPoolThreads);
        LaunchScope ls(BRA_KERNEL_REGION_MEAN, st);
        const bool big = s.w2 >= 64 && s.C / V <= kPoolThreads;  // one CTA per region
        if (s.dtype == BRA_BF16) {
            if (big)
                region_mean_big_kernel<__nv_bfloat16><<<s.N * s.P, kPoolThreads, 0, st>>>(
                    static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k), ws, ws + pooled,
                    s.H, s.W, s.C, s.S, FastDiv((uint32_t)s.wr));
            else
                region_mean_kernel<__nv_bfloat16><<<blocks, kPoolThreads, 0, st>>>(
                    static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k), ws, ws + pooled,
                    s.N, s.H, s.W, s.C, s.S, l, (int)total);
        } else {
            if (big)
                region_mean_big_kernel<float><<<s.N * s.P, kPoolThreads, 0, st>>>(
                    static_cast<const float *>(q), static_cast<const float *>(k), ws, ws + pooled, s.H, s.W, s.C, s.S,
                    FastDiv((uint32_t)s.wr));
            else
                region_mean_kernel<float><<<blocks, kPoolThreads, 0, st>>>(static_cast<const float *>(q),
                                                                          static_cast<const float *>(k), ws,
                                                                          ws + pooled, s.N, s.H, s.W, s.C, s.S, l,
                                                                          (int)total);
        }
        if (cudaGetLastError() != cudaSuccess) return BRA_ERR_CUDA;
    }
    const float scale = 1.0f / sqrtf((float)s.d);
    const int E = s.P <= 32 ? 1 : s.P <= 64 ? 2 : s.P <= 128 ? 4 : 8;
    // rows per CTA: as many as still leave about one CTA per SM
    int sms = 148;
    if (sm_count(&sms) != BRA_OK) return BRA_ERR_CUDA;
    int rpw = 4;
    while (rpw > 1 && (long long)s.N * ((s.P + kRouteWarps * rpw - 1) / (kRouteWarps * rpw)) < sms) rpw >>= 1;
    // more than 128 regions: the column-per-lane kernel with 4 or 8 rows per CTA
    const int cols_rows = (long long)s.N * ((s.P + 7) / 8) >= sms ? 8 : 4;
    const int rows = E == 8 ? cols_rows : kRouteWarps * rpw;
    // route_kernel stages key means in passes of cc channels; route_cols_kernel reads them
    // straight into registers
    int cc = route_chunk(32 * E, rows, s.C);
    while (s.C % cc) cc -= 32;  // equal passes: one divisor for the staging index
    const int smem = E == 8 ? route_cols_smem_bytes(rows, s.C) : route_smem_bytes(32 * E, rows, cc);
    const FastDiv div_q4((uint32_t)(cc / 4));
    int rc = BRA_OK;
    auto go = [&](auto kern) {
        if (allow_smem(kern, smem) != cudaSuccess) {
            rc = BRA_ERR_CUDA;
            return;
        }
        for (int n0 = 0; n0 < s.N && rc == BRA_OK; n0 += 65535) {
            const int nb = s.N - n0 < 65535 ? s.N - n0 : 65535;
            const dim3 g((s.P + rows - 1) / rows, nb, 1);
            LaunchScope ls(BRA_KERNEL_ROUTE, st);
            if (launch_pdl(kern, g, dim3(kRouteWarps * 32), smem, st, (const float *)(ws + (size_t)n0 * s.P * s.C),
                           (const float *)(ws + pooled + (size_t)n0 * s.P * s.C), s.C, s.P, s.topk, scale,
                           r_idx + (size_t)n0 * s.P * s.topk, r_weight + (size_t)n0 * s.P * s.topk) != cudaSuccess)
                rc = BRA_ERR_CUDA;
        }
    };
    auto go_staged = [&](auto kern) {
        if (allow_smem(kern, smem) != cudaSuccess) {
            rc = BRA_ERR_CUDA;
            return;
        }
        for (int n0 = 0; n0 < s.N && rc == BRA_OK; n0 += 65535) {
            const int nb = s.N - n0 < 65535 ? s.N - n0 : 65535;
            const dim3 g((s.P + rows - 1) / rows, nb, 1);
            LaunchScope ls(BRA_KERNEL_ROUTE, st);
            if (launch_pdl(kern, g, dim3(kRouteWarps * 32), smem, st, (const float *)(ws + (size_t)n0 * s.P * s.C),
                           (const float *)(ws + pooled + (size_t)n0 * s.P * s.C), s.C, s.P, s.topk, cc, scale,
                           r_idx + (size_t)n0 * s.P * s.topk, r_weight + (size_t)n0 * s.P * s.topk, div_q4) !=
                cudaSuccess)
                rc = BRA_ERR_CUDA;
        }
    };
    auto by_rpw = [&](auto e_tag) {
        constexpr int EE = decltype(e_tag)::value;
        if (rpw == 4)
            go_staged(route_kernel<EE, 4>);
        else if (rpw == 2)
            go_staged(route_kernel<EE, 2>);
        else
            go_staged(route_kernel<EE, 1>);
    };
    if (E == 1)
        by_rpw(std::integral_constant<int, 1>{});
    else if (E == 2)
        by_rpw(std::integral_constant<int, 2>{});
    else if (E == 4)
        by_rpw(std::integral_constant<int, 4>{});
    else if (cols_rows == 8)
        go(route_cols_kernel<8>);
    else
        go(route_cols_kernel<4>);
    return rc;
}

// ----------------------------------------------------------------------------- attention

static AttnParams base_params(const Shape &s, const void *q, const void *k, const void *v, const void *w,
                              const void *b, void *out, const int32_t *r_idx, int *err) {
    AttnParams p{};
    p.q = q;
    p.k = k;
    p.v = v;
    p.lce_w = w;
    p.lce_b = b;
    p.out = out;
    p.r_idx = r_idx;
    p.err_flag = err;
    p.N = s.N;
    p.H = s.H;
    p.W = s.W;
    p.C = s.C;
    p.heads = s.heads;
    p.S = s.S;
    p.topk = s.topk;
    p.hr = s.hr;
    p.wr = s.wr;
    p.w2 = s.w2;
    p.P = s.P;
    p.scale_log2 = (float)(1.0 / std::sqrt((double)s.d) * 1.4426950408889634);
    return p;
}

// Tensor-core kernel shape: HG heads (HG*d <= 128 channels) and RB region rows per
// CTA, with at most 8 warps of (head, 16-query tile) and 128 queries per CTA.
static bool plan_bf16(const Shape &s, AttnParams &p, int &threads, int &smem) {
    const int Lk = s.topk * s.w2;
    p.stages = Lk > kKC ? 2 : 1;
    for (int hg = largest_divisor_at_most(s.heads, 128 / s.d); hg >= 1; --hg) {
        if (s.heads % hg) continue;
        for (int rb = s.hr; rb >= 1; --rb) {
            if (s.hr % rb) continue;
            const int nq = rb * s.wr;
            const int qt = (nq + 15) / 16;
            if (nq > 128 || qt * hg > 8) continue;
            const Bf16Smem L = bf16_smem_layout(s.topk, qt, rb, s.wr, hg * s.d, p.stages);
            if (L.total > kMaxSmem) continue;
            p.HG = hg;
            p.RB = rb;
            p.QT = qt;
            p.n_hg = s.heads / hg;
            p.n_rb = s.hr / rb;
            threads = qt * hg * 32;
            smem = L.total;
            return true;
        }
    }
    return false;
}

// SIMT float32 kernel shape: F32Lanes<d>::n threads per (query, head), at most
// F32Lanes<d>::max_threads per CTA.
static bool plan_f32(const Shape &s, AttnParams &p, int &threads, int &smem) {
    const int lanes = s.d == 32 ? F32Lanes<32>::n : F32Lanes<64>::n;
    const int max_threads = s.d == 32 ? F32Lanes<32>::max_threads : F32Lanes<64>::max_threads;
    for (int hg = largest_divisor_at_most(s.heads, 128 / s.d); hg >= 1; --hg) {
        if (s.heads % hg) continue;
        for (int rb = s.hr; rb >= 1; --rb) {
            if (s.hr % rb) continue;
            const int nq = rb * s.wr;
            if (nq * hg * lanes > max_threads) continue;
            const F32Smem L = f32_smem_layout(s.topk, nq, rb, s.wr, hg * s.d);
            if (L.total > kMaxSmem) continue;
            p.HG = hg;
            p.RB = rb;
            p.QT = 0;
            p.stages = 1;
            p.n_hg = s.heads / hg;
            p.n_rb = s.hr / rb;
            threads = ((nq * hg * lanes + 31) / 32) * 32;
            smem = L.total;
            return true;
        }
    }
    return false;
}

template <typename K>
static int launch_kernel(K kern, int kid, int blocks, int threads, int smem, cudaStream_t st,
                         const AttnParams &p) {
    if (allow_smem(kern, smem) != cudaSuccess) return BRA_ERR_CUDA;
    LaunchScope ls(kid, st);
    kern<<<blocks, threads, smem, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

// ----------------------------------------------------------------------------- TMA attention

static std::atomic<int> g_variant{BRA_VARIANT_AUTO};
constexpr unsigned kWaitLimit = 1u << 22;  // mbarrier polls before a kernel gives up

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// (N,H,W,C) bf16 map, boxes of (64 channels, bw columns, bh rows, 1 image), 128-byte
// swizzle, zero fill outside the map.
static bool encode_map_box(CUtensorMap *m, const void *base, const Shape &s, int inner, int bw, int bh,
                           CUtensorMapSwizzle swizzle) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)s.C, (cuuint64_t)s.W, (cuuint64_t)s.H, (cuuint64_t)s.N};
    cuuint64_t strides[3] = {(cuuint64_t)s.C * 2, (cuuint64_t)s.W * s.C * 2, (cuuint64_t)s.H * s.W * s.C * 2};
    cuuint32_t box[4] = {(cuuint32_t)inner, (cuuint32_t)bw, (cuuint32_t)bh, 1u};
    cuuint32_t es[4] = {1u, 1u, 1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
static bool encode_map(CUtensorMap *m, const void *base, const Shape &s, int bw, int bh, bool swizzle = true) {
    return encode_map_box(m, base, s, 64, bw, bh, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

// TMA kernel shape: 64 or 128 channels (HG heads) and RB region rows per CTA, at most
// 8 warps of (head, 16-query tile) and 128 queries; prefer two CTAs per SM.
static bool plan_tma(const Shape &s, TmaAttnParams &p, int &threads, int &smem) {
    if (s.dtype != BRA_BF16 || s.hr > 256 || s.wr + 4 > 256) return false;
    for (int limit : {112 * 1024, kMaxSmem}) {
        for (int hg = s.heads; hg >= 1; --hg) {
            if (s.heads % hg) continue;
            const int CH = hg * s.d;
            if (CH != 64 && CH != 128) continue;
            for (int rb = s.hr; rb >= 1; --rb) {
                if (s.hr % rb) continue;
                const int nq = rb * s.wr, qt = (nq + 15) / 16;
                if (nq > 128 || qt * hg > 8) continue;
                const TmaSmem L = tma_smem_layout(s.topk, s.w2, qt, rb, s.wr, CH);
                if (L.total > limit) continue;
                p.HG = hg;
                p.RB = rb;
                p.QT = qt;
                p.n_hg = s.heads / hg;
                p.n_rb = s.hr / rb;
                p.slot = (s.w2 + 7) & ~7;
                threads = qt * hg * 32;
                smem = L.total;
                return true;
            }
        }
    }
    return false;
}

static int launch_attend_tma(const Shape &s, const void *q, const void *k, const void *v, const void *w,
                             const void *b, void *out, const int32_t *r_idx, int *err, cudaStream_t st,
                             bool *used) {
    *used = false;
    if (g_variant.load() != BRA_VARIANT_TMA) return BRA_OK;
    if (!aligned(w, 4) || !aligned(b, 4)) return BRA_OK;
    TmaAttnParams p;
    memset(&p, 0, sizeof(p));
    int threads = 0, smem = 0;
    if (!plan_tma(s, p, threads, smem)) return BRA_OK;
    if (!encode_map(&p.tmQ, q, s, s.wr, p.RB) || !encode_map(&p.tmK, k, s, s.wr, s.hr) ||
        !encode_map(&p.tmV, v, s, s.wr, s.hr) || !encode_map(&p.tmH, v, s, s.wr + 4, p.RB + 4, false))
        return BRA_OK;  // no tensor-map support: the generic kernel runs instead
    p.lce_w = static_cast<const __nv_bfloat16 *>(w);
    p.lce_b = static_cast<const __nv_bfloat16 *>(b);
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.r_idx = r_idx;
    p.err_flag = err;
    p.N = s.N;
    p.H = s.H;
    p.W = s.W;
    p.C = s.C;
    p.heads = s.heads;
    p.S = s.S;
    p.topk = s.topk;
    p.hr = s.hr;
    p.wr = s.wr;
    p.w2 = s.w2;
    p.P = s.P;
    p.scale_log2 = (float)(1.0 / std::sqrt((double)s.d) * 1.4426950408889634);
    p.wait_limit = kWaitLimit;
    const int blocks = s.N * s.P * p.n_rb * p.n_hg;
    auto kern = s.d == 32 ? attn_tma_kernel<32> : attn_tma_kernel<64>;
    if (allow_smem(kern, smem) != cudaSuccess) return BRA_ERR_CUDA;
    *used = true;
    LaunchScope ls(BRA_KERNEL_ATTN_BF16, st);
    return launch_pdl(kern, dim3(blocks), dim3(threads), smem, st, p) == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

// ----------------------------------------------------------------------------- persistent pipeline

struct PipePlan {
    int HG, RB, QT, NS, NE, threads, smem, ctas_per_sm;
};

// Choose (head group, row block, stages, epilogue warps): whole regions per unit where
// possible (a region's routed K/V is then fetched once), then the most resident
// attention warps per SM, then the most CTAs per SM, then the most stages. The
// epilogue gets about one warp per 64 LCE items (an item is one channel pair, pixel
// column and group of up to four rows). BRA_PIPE_PLAN="HG,RB,NS[,NE]" in the
// environment forces a plan (for tuning sweeps) when that plan is valid.
static bool plan_pipe(const Shape &s, PipePlan &best) {
    if (s.dtype != BRA_BF16 || s.hr > 256 || s.wr + 4 > 256) return false;
    // register cap per thread: 96 for CTAs of up to 160 threads (4 per SM), else 128
    int force_hg = 0, force_rb = 0, force_ns = 0, force_ne = 0;
    if (const char *env = getenv("BRA_PIPE_PLAN"))
        sscanf(env, "%d,%d,%d,%d", &force_hg, &force_rb, &force_ns, &force_ne);
    bool found = false;
    long best_score = -1;
    for (int hg = s.heads; hg >= 1; --hg) {
        if (s.heads % hg) continue;
        const int CH = hg * s.d;
        if (CH != 64 && CH != 128) continue;
        for (int rb = s.hr; rb >= 1; --rb) {
            if (s.hr % rb) continue;
            const int nq = rb * s.wr, qt = (nq + 15) / 16;
            if (nq > 128 || qt * hg > 8) continue;
            const int items = (CH / 2) * (s.wr / (s.wr % 2 == 0 ? 2 : 1)) * (rb / lce_row_span(rb));
            int ne = std::max(1, std::min(7, (items + 31) / 32));
            if (force_ne > 0) ne = std::min(7, force_ne);
            for (int ns = 3; ns >= 2; --ns) {
                if (force_hg && (hg != force_hg || rb != force_rb || ns != force_ns)) continue;
                const PipeSmem L = pipe_smem_layout(ns, s.topk, s.w2, qt, rb, s.wr, CH);
                if (L.total > kMaxSmem) continue;
                const int threads = (qt * hg + ne + 1) * 32;
                const int regs = threads <= 160 ? 96 : 128;
                int occ = (228 * 1024) / (L.total + 1024);
                occ = std::min(occ, 65536 / (threads * regs));
                occ = std::min(occ, 2048 / threads);
                if (occ < 1) continue;
                const long score = (rb == s.hr ? 1L << 40 : 0) + ((long)occ * qt * hg << 16) + (occ << 4) + ns;
                if (score > best_score) {
                    best_score = score;
                    best = {hg, rb, qt, ns, ne, threads, L.total, occ};
                    found = true;
                }
            }
        }
    }
    return found;
}

static int fill_tma_params(const Shape &s, TmaAttnParams &p, int HG, int RB, int QT, const void *q, const void *k,
                           const void *v, const void *w, const void *b, void *out, const int32_t *r_idx, int *err,
                           bool maps = true) {
    p.HG = HG;
    p.RB = RB;
    p.QT = QT;
    p.n_hg = s.heads / HG;
    p.n_rb = s.hr / RB;
    p.slot = (s.w2 + 7) & ~7;
    if (maps && (!encode_map(&p.tmQ, q, s, s.wr, RB) || !encode_map(&p.tmK, k, s, s.wr, s.hr) ||
        !encode_map(&p.tmV, v, s, s.wr, s.hr) || !encode_map(&p.tmH, v, s, s.wr + 4, RB + 4, false)))
        return 0;
    p.lce_w = static_cast<const __nv_bfloat16 *>(w);
    p.lce_b = static_cast<const __nv_bfloat16 *>(b);
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.r_idx = r_idx;
    p.err_flag = err;
    p.N = s.N;
    p.H = s.H;
    p.W = s.W;
    p.C = s.C;
    p.heads = s.heads;
    p.S = s.S;
    p.topk = s.topk;
    p.hr = s.hr;
    p.wr = s.wr;
    p.w2 = s.w2;
    p.P = s.P;
    p.scale_log2 = (float)(1.0 / std::sqrt((double)s.d) * 1.4426950408889634);
    p.wait_limit = kWaitLimit;
    return 1;
}

static int launch_attend_pipe(const Shape &s, const void *q, const void *k, const void *v, const void *w,
                              const void *b, void *out, const int32_t *r_idx, int *err, cudaStream_t st,
                              bool *used) {
    *used = false;
    const int var = g_variant.load();
    if (var != BRA_VARIANT_AUTO && var != BRA_VARIANT_SPLIT && var != BRA_VARIANT_PIPE) return BRA_OK;
    if (!aligned(w, 4) || !aligned(b, 4)) return BRA_OK;
    PipePlan pl;
    if (!plan_pipe(s, pl)) return BRA_OK;
    PipeParams pp;
    memset(&pp, 0, sizeof(pp));
    if (!fill_tma_params(s, pp.t, pl.HG, pl.RB, pl.QT, q, k, v, w, b, out, r_idx, err)) return BRA_OK;
    pp.q = static_cast<const __nv_bfloat16 *>(q);
    pp.k = static_cast<const __nv_bfloat16 *>(k);
    pp.v = static_cast<const __nv_bfloat16 *>(v);
    pp.div_wr = FastDiv((uint32_t)s.wr);
    pp.div_hw = FastDiv((uint32_t)(s.wr + 4));
    pp.div_nq = FastDiv((uint32_t)(pl.RB * s.wr));
    pp.div_nh = FastDiv((uint32_t)((pl.RB + 4) * (s.wr + 4)));
    pp.NS = pl.NS;
    pp.NE = pl.NE;
    pp.units = s.N * s.P * pp.t.n_rb * pp.t.n_hg;
    pp.XT = s.wr % 2 == 0 ? 2 : 1;
    pp.fast_keys = (s.w2 % 8 == 0 && (s.topk * s.w2) % kKC == 0) ? 1 : 0;
    pp.div_hg = FastDiv((uint32_t)pp.t.n_hg);
    pp.div_rb = FastDiv((uint32_t)pp.t.n_rb);
    pp.div_P = FastDiv((uint32_t)s.P);
    pp.div_S = FastDiv((uint32_t)s.S);
    pp.div_wx = FastDiv((uint32_t)(s.wr / pp.XT));
    auto kern = pl.threads <= 160 ? (s.d == 32 ? attn_pipe_kernel<32, 160, 4> : attn_pipe_kernel<64, 160, 4>)
                                  : (s.d == 32 ? attn_pipe_kernel<32, 512, 1> : attn_pipe_kernel<64, 512, 1>);
    if (allow_smem(kern, pl.smem) != cudaSuccess) return BRA_ERR_CUDA;
    int sms = 0, occ = 0;
    if (sm_count(&sms) != BRA_OK || occupancy(&occ, kern, pl.threads, pl.smem, 0, nullptr) != cudaSuccess)
        return BRA_ERR_CUDA;
    if (occ < 1) return BRA_OK;
    int ctas = std::min(pp.units, sms * occ);
    ctas -= ctas % pp.t.n_hg;  // a CTA keeps one head group (and its LCE weights)
    if (ctas < pp.t.n_hg) ctas = pp.t.n_hg;
    *used = true;
    LaunchScope ls(BRA_KERNEL_ATTN_BF16, st);
    return launch_pdl(kern, dim3(ctas), dim3(pl.threads), pl.smem, st, pp) == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

// ----------------------------------------------------------------------------- tcgen05 attention

// The tcgen05 kernel takes bf16 heads of 32 channels, regions of 64, 128 or 256 tokens
// (hr a multiple of 8, wr even), whole 128-key score halves and at most 256 keys per
// query. Regions of 128 or 256 tokens fill whole 128-query tiles; 64-token regions fill
// the first half of one.
static bool umma_shape_ok(const Shape &s) {
    return s.dtype == BRA_BF16 && s.d == 32 && (s.w2 % 128 == 0 || s.w2 == 64) && (s.topk * s.w2) % 128 == 0 &&
           s.topk * s.w2 <= 256 &&
           s.hr % kUmmaRows == 0 && s.wr % 2 == 0 && 128 % s.wr == 0 && s.hr + 4 <= 256 && s.wr + 4 <= 256;
}

static int launch_attend_umma(const Shape &s, const void *q, const void *k, const void *v, const void *w,
                              const void *b, void *out, const int32_t *r_idx, int *err, cudaStream_t st,
                              bool *used) {
    *used = false;
    const int var = g_variant.load();
    if (var != BRA_VARIANT_AUTO && var != BRA_VARIANT_SPLIT) return BRA_OK;
    if (!umma_shape_ok(s) || !aligned(w, 4) || !aligned(b, 4)) return BRA_OK;
    // 64-token regions: the half-filled tile only when asked for (BRA_VARIANT_SPLIT)
    if (s.w2 < 128 && var != BRA_VARIANT_SPLIT) return BRA_OK;
    const UmmaSmem L = umma_smem_layout(s.topk, s.w2, s.hr, s.wr);
    if (L.total > kMaxSmem) return BRA_OK;
    UmmaParams p;
    memset(&p, 0, sizeof(p));
    if (!encode_map_box(&p.tmQ, q, s, 32, s.wr, s.hr, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !encode_map_box(&p.tmK, k, s, 32, s.wr, s.hr, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !encode_map_box(&p.tmV, v, s, 32, s.wr, s.hr, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !encode_map_box(&p.tmH, v, s, 32, s.wr + 4, s.hr + 4, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_map_box(&p.tmO, out, s, 32, s.wr, std::min(128, s.w2) / s.wr, CU_TENSOR_MAP_SWIZZLE_64B))
        return BRA_OK;
    p.lce_w = static_cast<const __nv_bfloat16 *>(w);
    p.lce_b = static_cast<const __nv_bfloat16 *>(b);
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.r_idx = r_idx;
    p.err_flag = err;
    p.H = s.H;
    p.W = s.W;
    p.C = s.C;
    p.heads = s.heads;
    p.S = s.S;
    p.topk = s.topk;
    p.hr = s.hr;
    p.wr = s.wr;
    p.w2 = s.w2;
    p.P = s.P;
    p.regions = s.N * s.P;
    p.scale_log2 = (float)(1.0 / std::sqrt((double)s.d) * 1.4426950408889634);
    p.wait_limit = kWaitLimit;
    p.div_P = FastDiv((uint32_t)s.P);
    p.div_S = FastDiv((uint32_t)s.S);
    p.div_wr = FastDiv((uint32_t)s.wr);
    p.div_wx = FastDiv((uint32_t)(s.wr / 2));
    auto kern = attn_umma_kernel;
    if (allow_smem(kern, L.total) != cudaSuccess) return BRA_ERR_CUDA;
    int sms = 0;
    if (sm_count(&sms) != BRA_OK) return BRA_ERR_CUDA;
    // one CTA per SM (the whole tensor memory); a CTA keeps one head
    int ctas = std::min(sms, s.heads * p.regions);
    ctas -= ctas % s.heads;
    if (ctas < s.heads) ctas = s.heads;
    *used = true;
    LaunchScope ls(BRA_KERNEL_ATTN_UMMA, st);
    return launch_pdl(kern, dim3(ctas), dim3(kUmmaThreads), L.total, st, p) == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

static int launch_attend(const Shape &s, const void *q, const void *k, const void *v, const void *w,
                         const void *b, void *out, const int32_t *r_idx, int *err, cudaStream_t st) {
    bool used = false;
    int rc = launch_attend_umma(s, q, k, v, w, b, out, r_idx, err, st, &used);
    if (rc || used) return rc;
    rc = launch_attend_pipe(s, q, k, v, w, b, out, r_idx, err, st, &used);
    if (rc || used) return rc;
    rc = launch_attend_tma(s, q, k, v, w, b, out, r_idx, err, st, &used);
    if (rc || used) return rc;
    AttnParams p = base_params(s, q, k, v, w, b, out, r_idx, err);
    int threads = 0, smem = 0;
    if (s.dtype == BRA_BF16) {
        if (!plan_bf16(s, p, threads, smem)) return BRA_ERR_SHAPE;
        const int blocks = s.N * s.P * p.n_rb * p.n_hg;
        return s.d == 32 ? launch_kernel(attn_bf16_kernel<32>, BRA_KERNEL_ATTN_BF16, blocks, threads, smem, st, p)
                         : launch_kernel(attn_bf16_kernel<64>, BRA_KERNEL_ATTN_BF16, blocks, threads, smem, st, p);
    }
    if (!plan_f32(s, p, threads, smem)) return BRA_ERR_SHAPE;
    const int blocks = s.N * s.P * p.n_rb * p.n_hg;
    return s.d == 32 ? launch_kernel(attn_f32_kernel<32>, BRA_KERNEL_ATTN_F32, blocks, threads, smem, st, p)
                     : launch_kernel(attn_f32_kernel<64>, BRA_KERNEL_ATTN_F32, blocks, threads, smem, st, p);
}

// ----------------------------------------------------------------------------- fused small-image path

constexpr int kImageWarps = 16;

// Small images: attention and LCE of one (image, head) from shared memory (see
// include/bra.h), in one of two forms. Cluster form: everything in one launch, each
// cluster pooling, scoring and selecting its own image's routing. Routed form: the
// routing kernels first, then this kernel (programmatic dependent launch; its tile
// copies overlap the routing). The cluster form repeats its top-k rounds (one warp
// argmax per selected region) in every CTA, so past 8 routed regions the routed form
// is faster (measured: 14x14 maps, topk 16: 122 vs 150 us; 28x28, topk 4: 61 vs 59 us).
static bool fused_routed(const Shape &s) { return s.topk > 8; }

static bool fused_image_shape_ok(const Shape &s, const void *w, const void *b) {
    if (g_variant.load() != BRA_VARIANT_AUTO) return false;
    if (s.dtype != BRA_BF16 || s.d != 32 || s.P > 64 || s.topk > 64 || s.heads > 8) return false;
    if (!((s.hr == 4 && s.wr == 4) || (s.hr == 2 && s.wr == 2))) return false;
    return s.H + 4 <= 256 && s.W + 4 <= 256 && aligned(w, 4) && aligned(b, 4);
}

// 16 warps when one CTA fills an SM's shared memory; 8 when two fit (the kernel's 128
// registers per thread then allow two CTAs per SM).
static ImageSmem fused_image_layout(const Shape &s, bool routed, int *nwarps) {
    *nwarps = kImageWarps;
    if (image_smem_layout(s.H, s.W, s.P, s.topk, s.w2, kImageWarps / 2, routed).total <= kMaxSmem / 2)
        *nwarps = kImageWarps / 2;
    return image_smem_layout(s.H, s.W, s.P, s.topk, s.w2, *nwarps, routed);
}

// routed: r_idx already holds (or, on the stream, will hold) the routing; the kernel
// reads it and writes neither r_idx nor r_weight.
static int launch_fused_image(const Shape &s, bool routed, const void *q, const void *k, const void *v,
                              const void *w, const void *b, void *out, int32_t *r_idx, float *r_weight,
                              cudaStream_t st, bool *used) {
    *used = false;
    if (!fused_image_shape_ok(s, w, b)) return BRA_OK;
    int nwarps = 0;
    const ImageSmem L = fused_image_layout(s, routed, &nwarps);
    if (L.total > kMaxSmem) return BRA_OK;
    ImageParams p;
    memset(&p, 0, sizeof(p));
    if (!encode_map_box(&p.tmQ, q, s, 32, s.W, s.H, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !encode_map_box(&p.tmK, k, s, 32, s.W, s.H, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !encode_map_box(&p.tmV, v, s, 32, s.W + 4, s.H + 4, CU_TENSOR_MAP_SWIZZLE_NONE))
        return BRA_OK;
    p.lce_w = static_cast<const __nv_bfloat16 *>(w);
    p.lce_b = static_cast<const __nv_bfloat16 *>(b);
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.r_idx = r_idx;
    p.r_weight = r_weight;
    p.N = s.N;
    p.H = s.H;
    p.W = s.W;
    p.C = s.C;
    p.heads = s.heads;
    p.S = s.S;
    p.topk = s.topk;
    p.P = s.P;
    p.scale = (float)(1.0 / std::sqrt((double)s.d));
    p.scale_log2 = (float)(1.0 / std::sqrt((double)s.d) * 1.4426950408889634);
    p.wait_limit = kWaitLimit;
    p.div_S = FastDiv((uint32_t)s.S);
    p.div_W = FastDiv((uint32_t)s.W);
    if (routed) {
        auto kern = s.hr == 4 ? bra_image_kernel<4, 4, true> : bra_image_kernel<2, 2, true>;
        int per_sm = 0;
        if (allow_smem(kern, L.total) != cudaSuccess ||
            occupancy(&per_sm, kern, nwarps * 32, L.total, 0, nullptr) != cudaSuccess || per_sm < 1) {
            cudaGetLastError();
            return BRA_OK;
        }
        *used = true;
        LaunchScope ls(BRA_KERNEL_FUSED_IMAGE, st);
        return launch_pdl(kern, dim3(s.N * s.heads), dim3(nwarps * 32), L.total, st, p) == cudaSuccess ? BRA_OK
                                                                                                      : BRA_ERR_CUDA;
    }
    auto kern = s.hr == 4 ? bra_image_kernel<4, 4, false> : bra_image_kernel<2, 2, false>;
    if (allow_smem(kern, L.total) != cudaSuccess) return BRA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(s.N * s.heads);
    cfg.blockDim = dim3(nwarps * 32);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = s.heads;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (occupancy(&clusters, kern, nwarps * 32, L.total, s.heads, &cfg) != cudaSuccess || clusters < 1) {
        cudaGetLastError();  // not schedulable here: the three-kernel path runs instead
        return BRA_OK;
    }
    *used = true;
    LaunchScope ls(BRA_KERNEL_FUSED_IMAGE, st);
    return cudaLaunchKernelEx(&cfg, kern, p) == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

// ----------------------------------------------------------------------------- projections

// 2-D bfloat16 map of a row-major (rows x cols) matrix: boxes of box_cols (32 or 64)
// columns x box_rows rows with the matching 64- or 128-byte swizzle (the MMA operand and
// output staging layouts); loads fill zeros past the last row, stores clip there.
static bool encode_map_rows(CUtensorMap *m, const void *base, int rows, int cols, int box_rows, int box_cols = 32) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output columns per tile: the largest power of two in [32, 256] dividing ny (so that a
// tile never straddles two output buffers), 0 if none.
static int linear_tile_n(int ny) {
    for (int b = 256; b >= 32; b >>= 1)
        if (ny % b == 0) return b;
    return 0;
}

// Shapes the projections take (checked before any CUDA call): y (M x Nout) = x (M x K)
// w^T + b, output split into nsplit buffers of Nout / nsplit columns.
static int check_linear(int M, int K, int Nout, int nsplit, int dtype) {
    if (dtype != BRA_F32 && dtype != BRA_BF16) return BRA_ERR_DTYPE;
    if (M < 0 || K <= 0 || Nout <= 0 || nsplit < 1 || nsplit > 3 || Nout % nsplit) return BRA_ERR_SHAPE;
    if (K > 4096 || Nout > 4096) return BRA_ERR_SHAPE;
    if (dtype == BRA_BF16 && (K % 32 || linear_tile_n(Nout / nsplit) == 0)) return BRA_ERR_SHAPE;
    return BRA_OK;
}

// y[i] (M x Nout/nsplit, row-major) = column block i of x w^T + b.
static int launch_linear(const void *x, const void *w, const void *b, int M, int K, int Nout, int nsplit,
                         void *const *y, int dtype, cudaStream_t st, int epi = kEpiBias, const void *res = nullptr) {
    if (M == 0) return BRA_OK;
    const int ny = Nout / nsplit;
    if (dtype == BRA_F32) {
        LinearF32Params p;
        p.x = static_cast<const float *>(x);
        p.w = static_cast<const float *>(w);
        p.b = static_cast<const float *>(b);
        p.res = static_cast<const float *>(res);
        p.epi = epi;
        for (int i = 0; i < 3; ++i) p.y[i] = static_cast<float *>(y[i < nsplit ? i : 0]);
        p.M = M;
        p.K = K;
        p.Nout = Nout;
        p.Ny = ny;
        const dim3 grid((Nout + 63) / 64, (unsigned)std::min((M + 63) / 64, 65535));
        LaunchScope ls(BRA_KERNEL_LINEAR_F32, st);
        linear_f32_kernel<<<grid, 256, 0, st>>>(p);
        return cudaGetLastError() == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
    }
    LinearParams p;
    memset(&p, 0, sizeof(p));
    p.BN = linear_tile_n(ny);
    p.kc_elems = K % 64 == 0 ? 64 : 32;
    if (!encode_map_rows(&p.tmX, x, M, K, kLinRows, p.kc_elems) || !encode_map_rows(&p.tmW, w, Nout, K, p.BN, p.kc_elems))
        return BRA_ERR_CUDA;
    for (int i = 0; i < nsplit; ++i)
        if (!encode_map_rows(&p.tmY[i], y[i], M, ny, 32)) return BRA_ERR_CUDA;
    p.bias = static_cast<const __nv_bfloat16 *>(b);
    p.res = static_cast<const __nv_bfloat16 *>(res);
    p.epi = epi;
    p.M = M;
    p.K = K;
    p.Nout = Nout;
    p.Ny = ny;
    p.tiles_n = Nout / p.BN;
    p.tiles_m = (M + kLinRows - 1) / kLinRows;
    p.tmem_cols = 32;
    while (p.tmem_cols < (uint32_t)(2 * p.BN)) p.tmem_cols <<= 1;
    p.wait_limit = kWaitLimit;
    const int kch = K / p.kc_elems, a_bytes = kLinRows * p.kc_elems * 2;
    int sms = 0;
    int rc = sm_count(&sms);
    if (rc) return rc;
    constexpr int kSmPerSmBytes = 228 * 1024, kCtaReserve = 1024;
    // One CTA per SM (its 320 threads take most of the register file). W resident when
    // W and two row tiles' worth of X chunks fit: X is then read once and W once per
    // CTA. Otherwise streaming, with 2 to 8 stages. Each CTA asks for enough shared
    // memory that a second one would not fit: the tensor memory would not hold it (an
    // allocation beyond its 512 columns would wait for a resident CTA to finish).
    int smem = 0;
    const int res_fixed = linear_smem_layout(p.BN, 0, Nout, K, true, p.kc_elems).total;
    if (res_fixed + 2 * kch * (a_bytes + 16) <= kMaxSmem) {
        p.w_resident = 1;
        p.stages = std::min(4 * kch, (kMaxSmem - res_fixed) / (a_bytes + 16));
        smem = linear_smem_layout(p.BN, p.stages, Nout, K, true, p.kc_elems).total;
        smem = std::max(smem, kSmPerSmBytes / 2 - kCtaReserve + 16);  // one CTA per SM
    } else {
        p.stages = 2;
        while (p.stages < 8 && linear_smem_layout(p.BN, p.stages + 1, Nout, K, false, p.kc_elems).total <= kMaxSmem)
            ++p.stages;
        smem = linear_smem_layout(p.BN, p.stages, Nout, K, false, p.kc_elems).total;
        smem = std::max(smem, kSmPerSmBytes / 2 - kCtaReserve + 16);
    }
    if (smem > kMaxSmem) return BRA_ERR_SHAPE;
    if (allow_smem(linear_umma_kernel, smem) != cudaSuccess || prefer_shared(linear_umma_kernel) != cudaSuccess)
        return BRA_ERR_CUDA;
    const int work = p.w_resident ? p.tiles_m : p.tiles_m * p.tiles_n;
    const int grid = std::min(work, sms);
    LaunchScope ls(BRA_KERNEL_LINEAR_BF16, st);
    linear_umma_kernel<<<grid, kLinThreads, smem, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

// Everything a shape must pass before any CUDA call is made.
static int check_plan(const Shape &s) {
    int rc = check_shape(s);
    if (rc) return rc;
    const Shape sp = padded_shape(s);  // the kernels run on the padded grid
    AttnParams p{};
    int t, m;
    if (sp.dtype == BRA_BF16 ? !plan_bf16(sp, p, t, m) : !plan_f32(sp, p, t, m)) return BRA_ERR_SHAPE;
    return BRA_OK;
}

// ----------------------------------------------------------------------------- padded grid

// Zero-padded copies of up to three (N,H,W,C) maps into (N,Hp,Wp,C) buffers.
static int launch_pad(const Shape &s, int nmaps, const void *const *src, void *const *dst, cudaStream_t st) {
    PadParams p{};
    for (int i = 0; i < nmaps; ++i) {
        p.src[i] = static_cast<const uint4 *>(src[i]);
        p.dst[i] = static_cast<uint4 *>(dst[i]);
    }
    p.N = s.N;
    p.H = s.H;
    p.W = s.W;
    p.Hp = s.Hp;
    p.Wp = s.Wp;
    p.cv = s.C * (s.dtype == BRA_BF16 ? 2 : 4) / 16;
    LaunchScope ls(BRA_KERNEL_PAD, st);
    pad_maps_kernel<<<(unsigned)(nmaps * s.N * s.Hp), kPadThreads, 0, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

// The H x W real pixels of a padded (N,Hp,Wp,C) map into out (N,H,W,C).
static int launch_crop(const Shape &s, const void *src, void *out, cudaStream_t st) {
    LaunchScope ls(BRA_KERNEL_PAD, st);
    crop_map_kernel<<<(unsigned)(s.N * s.H), kPadThreads, 0, st>>>(
        static_cast<const uint4 *>(src), static_cast<uint4 *>(out), s.H, s.W, s.Hp, s.Wp,
        s.C * (s.dtype == BRA_BF16 ? 2 : 4) / 16);
    return cudaGetLastError() == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

// ----------------------------------------------------------------------------- BiFormer block

// The block's per-pixel kernels (pos-embed + LN1, residual + LN2), C <= 256.
template <typename T>
static int launch_block_pixels(bool pos, const BlockParams &p, cudaStream_t st) {
    int sms = 0;
    int rc = sm_count(&sms);
    if (rc) return rc;
    const long long want = (p.pixels + kBlockThreads / 32 - 1) / (kBlockThreads / 32);
    const unsigned grid = (unsigned)std::max<long long>(1, std::min<long long>(want, (long long)sms * 8));
    const int np = (p.C + 63) / 64;
    // the positional embedding: tiles of kPosTH x kPosTW pixels staged in shared memory
    const int tiles_x = (p.W + kPosTW - 1) / kPosTW, tiles_y = (p.H + kPosTH - 1) / kPosTH;
    const long long tiles = p.pixels / ((long long)p.H * p.W) * tiles_x * tiles_y;
    const int tsmem = pos_tile_smem_bytes(p.C, (int)sizeof(T));
    if (pos && tiles > INT_MAX) return BRA_ERR_SHAPE;
    // add_ln with 16-byte accesses when a pixel is a power-of-two number (<= 32) of 16-byte chunks
    const int lpp = p.C * (int)sizeof(T) / 16;
    if (!pos && p.C * (int)sizeof(T) % 16 == 0 && lpp >= 1 && lpp <= 32 && (lpp & (lpp - 1)) == 0) {
        const long long groups = (p.pixels + 32 / lpp * kAddUnroll - 1) / (32 / lpp * kAddUnroll);
        const unsigned g2 = (unsigned)std::max<long long>(
            1, std::min<long long>((groups + kBlockThreads / 32 - 1) / (kBlockThreads / 32), (long long)sms * 8));
        LaunchScope ls(BRA_KERNEL_BLOCK, st);
        switch (lpp) {
            case 1: add_ln_vec_kernel<T, 1><<<g2, kBlockThreads, 0, st>>>(p); break;
            case 2: add_ln_vec_kernel<T, 2><<<g2, kBlockThreads, 0, st>>>(p); break;
            case 4: add_ln_vec_kernel<T, 4><<<g2, kBlockThreads, 0, st>>>(p); break;
            case 8: add_ln_vec_kernel<T, 8><<<g2, kBlockThreads, 0, st>>>(p); break;
            case 16: add_ln_vec_kernel<T, 16><<<g2, kBlockThreads, 0, st>>>(p); break;
            default: add_ln_vec_kernel<T, 32><<<g2, kBlockThreads, 0, st>>>(p); break;
        }
        return cudaGetLastError() == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
    }
    LaunchScope ls(BRA_KERNEL_BLOCK, st);
    switch (np) {
#define BRA_BLOCK_CASE(NP)                                                                                    \
    case NP:                                                                                                  \
        if (pos) {                                                                                            \
            if (allow_smem(pos_ln_tile_kernel<T, NP>, tsmem) != cudaSuccess) return BRA_ERR_CUDA;             \
            pos_ln_tile_kernel<T, NP><<<(unsigned)tiles, kBlockThreads, tsmem, st>>>(p, tiles_x, tiles_y);    \
        } else                                                                                                \
            add_ln_kernel<T, NP><<<grid, kBlockThreads, 0, st>>>(p);                                          \
        break;
        BRA_BLOCK_CASE(1)
        BRA_BLOCK_CASE(2)
        BRA_BLOCK_CASE(3)
        BRA_BLOCK_CASE(4)
#undef BRA_BLOCK_CASE
        default: return BRA_ERR_SHAPE;
    }
    return cudaGetLastError() == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

static int launch_block(bool pos, int dtype, const BlockParams &p, cudaStream_t st) {
    return dtype == BRA_BF16 ? launch_block_pixels<__nv_bfloat16>(pos, p, st) : launch_block_pixels<float>(pos, p, st);
}

// Bytes of one padded (N,Hp,Wp,C) map, rounded up to 256.
static size_t padded_map_bytes(const Shape &s) {
    return ((size_t)s.N * s.Hp * s.Wp * s.C * (s.dtype == BRA_BF16 ? 2 : 4) + 255) / 256 * 256;
}

}  // namespace bra

using namespace bra;

extern "C" {

int bra_version(void) { return (1 << 16) | 1; }

int bra_set_kernel_variant(int variant) {
    if (variant < BRA_VARIANT_AUTO || variant > BRA_VARIANT_PIPE) return -1;
    return g_variant.exchange(variant);
}

int bra_device_status(bra_stream_t stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return BRA_ERR_CUDA;
    int flag = 0, index = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&flag, g_bra_timeout_flag, sizeof(int)) != cudaSuccess ||
        cudaMemcpyFromSymbol(&index, g_bra_index_flag, sizeof(int)) != cudaSuccess)
        return BRA_ERR_CUDA;
    if (flag && cudaMemcpyToSymbol(g_bra_timeout_flag, &zero, sizeof(int)) != cudaSuccess) return BRA_ERR_CUDA;
    if (index && cudaMemcpyToSymbol(g_bra_index_flag, &zero, sizeof(int)) != cudaSuccess) return BRA_ERR_CUDA;
    return flag ? BRA_ERR_TIMEOUT : index ? BRA_ERR_INDEX : BRA_OK;
}

int bra_selftest_wait_timeout(unsigned polls, bra_stream_t stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(polls);
    return cudaGetLastError() == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

long long bra_launch_count(void) { return g_launches.load(); }

int bra_trace_begin(void) {
    std::lock_guard<std::mutex> g(g_trace_mu);
    g_tracing = true;
    return BRA_OK;
}

int bra_trace_read(double *ms, long long *launches) {
    std::lock_guard<std::mutex> g(g_trace_mu);
    double tot[BRA_KERNEL_CLASSES] = {0};
    long long cnt[BRA_KERNEL_CLASSES] = {0};
    int rc = BRA_OK;
    for (auto &r : g_trace) {
        float t = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
            rc = BRA_ERR_CUDA;
        tot[r.kid] += t;
        cnt[r.kid] += 1;
    }
    for (int i = 0; i < BRA_KERNEL_CLASSES; ++i) {
        if (ms) ms[i] = tot[i];
        if (launches) launches[i] = cnt[i];
    }
    return rc;
}

int bra_trace_end(double *ms, long long *launches) {
    std::vector<TraceRec> recs;
    {
        std::lock_guard<std::mutex> g(g_trace_mu);
        g_tracing = false;
        recs.swap(g_trace);
    }
    double tot[BRA_KERNEL_CLASSES] = {0};
    long long cnt[BRA_KERNEL_CLASSES] = {0};
    int rc = BRA_OK;
    for (auto &r : recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
            rc = BRA_ERR_CUDA;
        tot[r.kid] += t;
        cnt[r.kid] += 1;
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
    }
    for (int i = 0; i < BRA_KERNEL_CLASSES; ++i) {
        if (ms) ms[i] = tot[i];
        if (launches) launches[i] = cnt[i];
    }
    return rc;
}

const char *bra_kernel_name(int kernel_class) {
    switch (kernel_class) {
        case BRA_KERNEL_REGION_MEAN: return "region_mean_kernel";
        case BRA_KERNEL_ROUTE: return "route_kernel";
        case BRA_KERNEL_ATTN_BF16: return "attn_bf16_kernel";
        case BRA_KERNEL_ATTN_F32: return "attn_f32_kernel";
        case BRA_KERNEL_FUSED_IMAGE: return "bra_image_kernel";
        case BRA_KERNEL_ATTN_UMMA: return "attn_umma_kernel";
        case BRA_KERNEL_LINEAR_BF16: return "linear_umma_kernel";
        case BRA_KERNEL_LINEAR_F32: return "linear_f32_kernel";
        case BRA_KERNEL_BACKWARD: return "bwd_kernels";
        case BRA_KERNEL_PAD: return "pad_crop_kernels";
        case BRA_KERNEL_BLOCK: return "block_pixel_kernels";
        default: return "unknown";
    }
}

const char *bra_status_string(int status) {
    switch (status) {
        case BRA_OK: return "ok";
        case BRA_ERR_NULL: return "a required pointer is NULL";
        case BRA_ERR_SHAPE: return "unsupported shape (C%heads, topk, S*S<=256, d in {32,64}, C<=1024, ceil(W/S)<=128; bra_backward: H%S, W%S)";
        case BRA_ERR_ALIGN: return "pointer misaligned (q, k, v, out need 16 bytes; r_idx, r_weight 4)";
        case BRA_ERR_DTYPE: return "dtype must be BRA_F32 or BRA_BF16";
        case BRA_ERR_CUDA: return "a CUDA allocation, copy or kernel launch failed";
        case BRA_ERR_INDEX: return "a region index in r_idx lies outside [0, S*S)";
        case BRA_ERR_SCRATCH: return "problem needs more scratch than the static array holds (2*N*S*S*C > BRA_STATIC_SCRATCH_FLOATS)";
        case BRA_ERR_TIMEOUT: return "a kernel's bounded wait for its tile copies ran out";
        default: return "unknown status";
    }
}

int bra_route(const void *q, const void *k, int N, int H, int W, int C, int heads, int S, int topk,
              int dtype, int32_t *r_idx, float *r_weight, bra_stream_t stream) {
    const Shape s = make_shape(N, H, W, C, heads, S, topk, dtype);
    int rc = check_plan(s);
    if (rc) return rc;
    if (N == 0) return BRA_OK;
    if (!q || !k || !r_idx || !r_weight) return BRA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(r_idx, 4) || !aligned(r_weight, 4)) return BRA_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t pooled = 2 * (size_t)N * s.P * C * sizeof(float);
    const size_t map = s.padded() ? padded_map_bytes(s) : 0;  // padded grid: copies of q, k
    unsigned char *buf = nullptr;
    if (cudaMallocAsync(reinterpret_cast<void **>(&buf), pooled + 2 * map, st) != cudaSuccess) return BRA_ERR_CUDA;
    float *ws = reinterpret_cast<float *>(buf + 2 * map);
    if (s.padded()) {
        const void *src[2] = {q, k};
        void *dst[2] = {buf, buf + map};
        rc = launch_pad(s, 2, src, dst, st);
        if (rc == BRA_OK) rc = launch_route_into(padded_shape(s), dst[0], dst[1], r_idx, r_weight, ws, st);
    } else {
        rc = launch_route_into(s, q, k, r_idx, r_weight, ws, st);
    }
    if (cudaFreeAsync(buf, st) != cudaSuccess && rc == BRA_OK) rc = BRA_ERR_CUDA;
    return rc;
}

// The forward with its scratch taken from (and returned to) the stream-ordered pool;
// the scratch is released after the attention launch so that nothing separates the
// route and attention kernels on the stream.
// ws_given: scratch of 2*N*S*S*C floats owned by the caller, or NULL to take it from the
// stream-ordered default pool for the duration of the call.
static int forward_device(const Shape &s, const void *q, const void *k, const void *v, const void *lce_w,
                          const void *lce_b, void *out, int32_t *r_idx, float *r_weight, cudaStream_t st,
                          float *ws_given = nullptr) {
    if (s.padded()) {
        // the padded grid: zero-padded copies of q, k, v, the forward on them, the crop
        const size_t map = padded_map_bytes(s);
        unsigned char *buf = nullptr;
        if (cudaMallocAsync(reinterpret_cast<void **>(&buf), 4 * map, st) != cudaSuccess) return BRA_ERR_CUDA;
        const void *src[3] = {q, k, v};
        void *dst[3] = {buf, buf + map, buf + 2 * map};
        int rc = launch_pad(s, 3, src, dst, st);
        if (rc == BRA_OK)
            rc = forward_device(padded_shape(s), dst[0], dst[1], dst[2], lce_w, lce_b, buf + 3 * map, r_idx, r_weight,
                                st, ws_given);
        if (rc == BRA_OK) rc = launch_crop(s, buf + 3 * map, out, st);
        if (cudaFreeAsync(buf, st) != cudaSuccess && rc == BRA_OK) rc = BRA_ERR_CUDA;
        return rc;
    }
    bool fused = false;
    const bool routed = fused_routed(s) && fused_image_shape_ok(s, lce_w, lce_b);
    if (!routed) {
        const int frc = launch_fused_image(s, false, q, k, v, lce_w, lce_b, out, r_idx, r_weight, st, &fused);
        if (frc || fused) return frc;
    }
    float *ws = ws_given;
    if (!ws && cudaMallocAsync(reinterpret_cast<void **>(&ws), 2 * (size_t)s.N * s.P * s.C * sizeof(float), st) !=
                   cudaSuccess)
        return BRA_ERR_CUDA;
    int rc = launch_route_into(s, q, k, r_idx, r_weight, ws, st);
    if (rc == BRA_OK && routed) rc = launch_fused_image(s, true, q, k, v, lce_w, lce_b, out, r_idx, r_weight, st, &fused);
    if (rc == BRA_OK && !fused) rc = launch_attend(s, q, k, v, lce_w, lce_b, out, r_idx, nullptr, st);
    if (!ws_given && cudaFreeAsync(ws, st) != cudaSuccess && rc == BRA_OK) rc = BRA_ERR_CUDA;
    return rc;
}

int bra_forward(const void *q, const void *k, const void *v, const void *lce_w, const void *lce_b, int N,
                int H, int W, int C, int heads, int S, int topk, int dtype, void *out, int32_t *r_idx,
                float *r_weight, bra_stream_t stream) {
    const Shape s = make_shape(N, H, W, C, heads, S, topk, dtype);
    int rc = check_plan(s);
    if (rc) return rc;
    if (N == 0) return BRA_OK;
    if (!q || !k || !v || !lce_w || !lce_b || !out || !r_idx || !r_weight) return BRA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(r_idx, 4) ||
        !aligned(r_weight, 4))
        return BRA_ERR_ALIGN;
    const size_t es = dtype == BRA_BF16 ? 2 : 4;
    if (!aligned(lce_w, es) || !aligned(lce_b, es)) return BRA_ERR_ALIGN;
    return forward_device(s, q, k, v, lce_w, lce_b, out, r_idx, r_weight, reinterpret_cast<cudaStream_t>(stream));
}

int bra_linear(const void *x, const void *w, const void *b, int M, int K, int Nout, int dtype, void *y,
               bra_stream_t stream) {
    int rc = check_linear(M, K, Nout, 1, dtype);
    if (rc) return rc;
    if (M == 0) return BRA_OK;
    if (!x || !w || !b || !y) return BRA_ERR_NULL;
    const size_t es = dtype == BRA_BF16 ? 2 : 4;
    if (!aligned(x, 16) || !aligned(w, 16) || !aligned(y, 16) || !aligned(b, es)) return BRA_ERR_ALIGN;
    void *ys[1] = {y};
    return launch_linear(x, w, b, M, K, Nout, 1, ys, dtype, reinterpret_cast<cudaStream_t>(stream));
}

int bra_qkv(const void *x, const void *w_qkv, const void *b_qkv, int M, int C, int dtype, void *q, void *k,
            void *v, bra_stream_t stream) {
    if (C <= 0 || C > 4096 / 3) return dtype == BRA_F32 || dtype == BRA_BF16 ? BRA_ERR_SHAPE : BRA_ERR_DTYPE;
    int rc = check_linear(M, C, 3 * C, 3, dtype);
    if (rc) return rc;
    if (M == 0) return BRA_OK;
    if (!x || !w_qkv || !b_qkv || !q || !k || !v) return BRA_ERR_NULL;
    const size_t es = dtype == BRA_BF16 ? 2 : 4;
    if (!aligned(x, 16) || !aligned(w_qkv, 16) || !aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) ||
        !aligned(b_qkv, es))
        return BRA_ERR_ALIGN;
    void *ys[3] = {q, k, v};
    return launch_linear(x, w_qkv, b_qkv, M, C, 3 * C, 3, ys, dtype, reinterpret_cast<cudaStream_t>(stream));
}

// Layer scratch: q, k, v and the attention output (one map each), then the pooled means.
static size_t map_bytes(const Shape &s) {
    return ((size_t)s.N * s.H * s.W * s.C * (s.dtype == BRA_BF16 ? 2 : 4) + 255) / 256 * 256;
}
static size_t layer_scratch_bytes(const Shape &s) { return 4 * map_bytes(s) + 2 * (size_t)s.N * s.P * s.C * 4; }

// qkv projection -> BRA forward -> output projection, on caller scratch of
// layer_scratch_bytes(s).
static int layer_device(const Shape &s, const void *x, const void *w_qkv, const void *b_qkv, const void *w_o,
                        const void *b_o, const void *lce_w, const void *lce_b, void *out, int32_t *r_idx,
                        float *r_weight, cudaStream_t st, unsigned char *buf) {
    const int T = s.N * s.H * s.W;
    const size_t plane = map_bytes(s);
    void *qkv[3] = {buf, buf + plane, buf + 2 * plane};
    void *o = buf + 3 * plane;
    float *ws = reinterpret_cast<float *>(buf + 4 * plane);
    int rc = launch_linear(x, w_qkv, b_qkv, T, s.C, 3 * s.C, 3, qkv, s.dtype, st);
    if (rc == BRA_OK) rc = forward_device(s, qkv[0], qkv[1], qkv[2], lce_w, lce_b, o, r_idx, r_weight, st, ws);
    if (rc == BRA_OK) rc = launch_linear(o, w_o, b_o, T, s.C, s.C, 1, &out, s.dtype, st);
    return rc;
}

// Scratch of `bytes` taken stream-ordered: outside a stream capture from the library's
// per-device pool that keeps its memory between calls (mapping tens of MB again on every
// call costs milliseconds); inside one, from the default pool (a memory node of the graph).
static int scratch_alloc(unsigned char **buf, size_t bytes, cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return BRA_ERR_CUDA;
    if (cs == cudaStreamCaptureStatusNone) {
        cudaMemPool_t pool = nullptr;
        cudaStream_t up = nullptr, back = nullptr;
        int rc = host_call_pool(&pool, &up, &back);
        if (rc) return rc;
        return cudaMallocFromPoolAsync(reinterpret_cast<void **>(buf), bytes, pool, st) == cudaSuccess ? BRA_OK
                                                                                                      : BRA_ERR_CUDA;
    }
    return cudaMallocAsync(reinterpret_cast<void **>(buf), bytes, st) == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

int bra_attention_layer(const void *x, const void *w_qkv, const void *b_qkv, const void *w_o, const void *b_o,
                        const void *lce_w, const void *lce_b, int N, int H, int W, int C, int heads, int S,
                        int topk, int dtype, void *out, int32_t *r_idx, float *r_weight, bra_stream_t stream) {
    const Shape s = make_shape(N, H, W, C, heads, S, topk, dtype);
    int rc = check_plan(s);
    if (rc) return rc;
    const long long T = (long long)N * H * W;
    if (T > INT_MAX) return BRA_ERR_SHAPE;
    if ((rc = check_linear((int)T, C, 3 * C, 3, dtype)) || (rc = check_linear((int)T, C, C, 1, dtype))) return rc;
    if (N == 0) return BRA_OK;
    if (!x || !w_qkv || !b_qkv || !w_o || !b_o || !lce_w || !lce_b || !out || !r_idx || !r_weight)
        return BRA_ERR_NULL;
    const size_t es = dtype == BRA_BF16 ? 2 : 4;
    if (!aligned(x, 16) || !aligned(w_qkv, 16) || !aligned(w_o, 16) || !aligned(out, 16) || !aligned(b_qkv, es) ||
        !aligned(b_o, es) || !aligned(lce_w, es) || !aligned(lce_b, es) || !aligned(r_idx, 4) ||
        !aligned(r_weight, 4))
        return BRA_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    unsigned char *buf = nullptr;
    if ((rc = scratch_alloc(&buf, layer_scratch_bytes(s), st))) return rc;
    rc = layer_device(s, x, w_qkv, b_qkv, w_o, b_o, lce_w, lce_b, out, r_idx, r_weight, st, buf);
    if (cudaFreeAsync(buf, st) != cudaSuccess && rc == BRA_OK) rc = BRA_ERR_CUDA;
    return rc;
}

int bra_linear_act(const void *x, const void *w, const void *b, const void *res, int M, int K, int Nout, int act,
                   int dtype, void *y, bra_stream_t stream) {
    int rc = check_linear(M, K, Nout, 1, dtype);
    if (rc) return rc;
    if (act != BRA_ACT_NONE && act != BRA_ACT_GELU && act != BRA_ACT_RESIDUAL) return BRA_ERR_SHAPE;
    if (M == 0) return BRA_OK;
    if (!x || !w || !b || !y || (act == BRA_ACT_RESIDUAL && !res)) return BRA_ERR_NULL;
    const size_t es = dtype == BRA_BF16 ? 2 : 4;
    if (!aligned(x, 16) || !aligned(w, 16) || !aligned(y, 16) || !aligned(b, es) ||
        (act == BRA_ACT_RESIDUAL && !aligned(res, 16)))
        return BRA_ERR_ALIGN;
    void *ys[1] = {y};
    return launch_linear(x, w, b, M, K, Nout, 1, ys, dtype, reinterpret_cast<cudaStream_t>(stream), act, res);
}

int bra_block(const void *x, const void *pos_w, const void *pos_b, const void *ln1_g, const void *ln1_b,
              const void *w_qkv, const void *b_qkv, const void *w_o, const void *b_o, const void *lce_w,
              const void *lce_b, const void *ln2_g, const void *ln2_b, const void *mlp_w1, const void *mlp_b1,
              const void *mlp_w2, const void *mlp_b2, int N, int H, int W, int C, int heads, int S, int topk,
              int dtype, void *out, int32_t *r_idx, float *r_weight, bra_stream_t stream) {
    const Shape s = make_shape(N, H, W, C, heads, S, topk, dtype);
    int rc = check_plan(s);
    if (rc) return rc;
    if (C > 256) return BRA_ERR_SHAPE;
    const long long T = (long long)N * H * W;
    if (T > INT_MAX) return BRA_ERR_SHAPE;
    if ((rc = check_linear((int)T, C, 3 * C, 3, dtype)) || (rc = check_linear((int)T, C, C, 1, dtype)) ||
        (rc = check_linear((int)T, C, 3 * C, 1, dtype)) || (rc = check_linear((int)T, 3 * C, C, 1, dtype)))
        return rc;
    if (N == 0) return BRA_OK;
    const void *params[] = {pos_w, pos_b, ln1_g, ln1_b, b_qkv, b_o, lce_w, lce_b, ln2_g, ln2_b, mlp_b1, mlp_b2};
    for (const void *q : params)
        if (!q) return BRA_ERR_NULL;
    if (!x || !w_qkv || !w_o || !mlp_w1 || !mlp_w2 || !out || !r_idx || !r_weight) return BRA_ERR_NULL;
    const size_t es = dtype == BRA_BF16 ? 2 : 4;
    for (const void *q : params)
        if (!aligned(q, es)) return BRA_ERR_ALIGN;
    if (!aligned(x, 16) || !aligned(w_qkv, 16) || !aligned(w_o, 16) || !aligned(mlp_w1, 16) ||
        !aligned(mlp_w2, 16) || !aligned(out, 16) || !aligned(r_idx, 4) || !aligned(r_weight, 4))
        return BRA_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t plane = map_bytes(s);
    // x1, h (reused for h2), a, x2, the MLP hidden layer (three planes), the layer's scratch
    unsigned char *buf = nullptr;
    if ((rc = scratch_alloc(&buf, 7 * plane + layer_scratch_bytes(s), st))) return rc;
    unsigned char *x1 = buf, *h = buf + plane, *a = buf + 2 * plane, *x2 = buf + 3 * plane, *m = buf + 4 * plane;
    unsigned char *lbuf = buf + 7 * plane;
    BlockParams bp{};
    bp.pixels = T;
    bp.H = H;
    bp.W = W;
    bp.C = C;
    // x1 = x + pos_embed(x), h = norm1(x1)
    bp.x = x;
    bp.pos_w = pos_w;
    bp.pos_b = pos_b;
    bp.ln_g = ln1_g;
    bp.ln_b = ln1_b;
    bp.xo = x1;
    bp.h = h;
    rc = launch_block(true, dtype, bp, st);
    // a = attn(h)
    if (rc == BRA_OK) rc = layer_device(s, h, w_qkv, b_qkv, w_o, b_o, lce_w, lce_b, a, r_idx, r_weight, st, lbuf);
    // x2 = x1 + a, h = norm2(x2)
    if (rc == BRA_OK) {
        bp.x = x1;
        bp.a = a;
        bp.ln_g = ln2_g;
        bp.ln_b = ln2_b;
        bp.xo = x2;
        bp.h = h;
        rc = launch_block(false, dtype, bp, st);
    }
    // out = x2 + mlp(h): Linear(C, 3C) + GELU, then Linear(3C, C) with the residual
    void *mp[1] = {m}, *op[1] = {out};
    if (rc == BRA_OK) rc = launch_linear(h, mlp_w1, mlp_b1, (int)T, C, 3 * C, 1, mp, dtype, st, kEpiGelu);
    if (rc == BRA_OK) rc = launch_linear(m, mlp_w2, mlp_b2, (int)T, 3 * C, C, 1, op, dtype, st, kEpiResidual, x2);
    if (cudaFreeAsync(buf, st) != cudaSuccess && rc == BRA_OK) rc = BRA_ERR_CUDA;
    return rc;
}

// Device address of the library's out-of-range flag (g_bra_index_flag) on the current device.
static int index_flag(int **out) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bra_index_flag) != cudaSuccess || p == nullptr) return BRA_ERR_CUDA;
    *out = static_cast<int *>(p);
    return BRA_OK;
}

// The backward on the tensor cores (bf16 maps, 32 channels per head), deterministic: the
// transposed routing, the LCE part of dv, the query-side pass (dq and the per-query
// statistics), the key-side pass (dk, and dv added to its LCE part), the LCE parameter
// gradients (partials, then a fixed-order sum). Scratch from the library's pool outside a
// capture. Synchronises `stream` to read the out-of-range flag, as the other backward.
static int backward_tc(const Shape &s, const void *q, const void *k, const void *v, const void *lce_w,
                       const int32_t *r_idx, const void *dout, float *dq, float *dk, float *dv, float *dlce_w,
                       float *dlce_b, cudaStream_t st, bool sync) {
    const int nw = (s.w2 + 15) / 16;
    if (nw > kBwdTcMaxWarps) return BRA_ERR_SHAPE;
    const int L = s.topk * s.w2;
    int sms = 0;
    int rc = sm_count(&sms);
    if (rc) return rc;
    // LCE gradients: ng channel groups of pg pairs, G CTAs per group
    // groups of pg channel pairs, pg the largest of 64, 48, 32, 16 that divides the pairs
    // (C is a multiple of 32, so 16 always does)
    const int pairs = s.C / 2;
    const int pg = pairs % 64 == 0 ? 64 : pairs % 48 == 0 ? 48 : pairs % 32 == 0 ? 32 : 16;
    const int ng = pairs / pg;
    const int lce_tiles = s.N * ((s.H + kLceTH - 1) / kLceTH) * ((s.W + kLceTW - 1) / kLceTW);
    const int G = std::max(1, std::min(lce_tiles, sms / ng));  // one wave (one CTA per SM)
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t b_off = up((size_t)s.N * (s.P + 1) * 4), b_list = up((size_t)s.N * s.P * s.topk * 4);
    const size_t b_stats = up((size_t)s.N * s.P * s.heads * s.w2 * 8);
    const size_t b_part = up((size_t)ng * G * kLceGroup * 2 * 26 * 4);
    unsigned char *buf = nullptr;
    if ((rc = scratch_alloc(&buf, b_off + b_list + b_stats + b_part + 256, st))) return rc;
    BwdTcParams p{};
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.k = static_cast<const __nv_bfloat16 *>(k);
    p.v = static_cast<const __nv_bfloat16 *>(v);
    p.dout = static_cast<const __nv_bfloat16 *>(dout);
    p.r_idx = r_idx;
    p.kv_off = reinterpret_cast<int *>(buf);
    p.kv_list = reinterpret_cast<int *>(buf + b_off);
    p.stats = reinterpret_cast<float *>(buf + b_off + b_list);
    float *part = reinterpret_cast<float *>(buf + b_off + b_list + b_stats);
    // the out-of-range flag: per call (read back here) or the library's device flag
    p.bad = reinterpret_cast<int *>(buf + b_off + b_list + b_stats + b_part);
    if (!sync && (rc = index_flag(&p.bad))) {
        cudaFreeAsync(buf, st);
        return rc;
    }
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.N = s.N;
    p.H = s.H;
    p.W = s.W;
    p.C = s.C;
    p.heads = s.heads;
    p.S = s.S;
    p.topk = s.topk;
    p.P = s.P;
    p.hr = s.hr;
    p.wr = s.wr;
    p.w2 = s.w2;
    p.L = L;
    p.nw = nw;
    p.scale = 1.0f / sqrtf((float)s.d);
    p.sl2 = p.scale * 1.4426950408889634f;
    p.div_S = FastDiv((uint32_t)s.S);
    p.div_wr = FastDiv((uint32_t)s.wr);
    p.div_w2 = FastDiv((uint32_t)s.w2);
    p.div_topk = FastDiv((uint32_t)s.topk);
    p.div_heads = FastDiv((uint32_t)s.heads);
    p.div_P = FastDiv((uint32_t)s.P);
    {
        const int tr_smem = s.P * 4;
        const int q_smem = bwd_tc_query_smem(nw, L, s.topk), k_smem = bwd_tc_key_smem(nw, s.w2);
        const int l_smem = bwd_tc_lce_smem(pg);
        auto lce_kern = pg == 16 ? bwd_tc_lce_kernel<16> : pg == 32 ? bwd_tc_lce_kernel<32>
                        : pg == 48 ? bwd_tc_lce_kernel<48> : bwd_tc_lce_kernel<64>;
        const unsigned units = (unsigned)((size_t)s.N * s.P * s.heads);
        if ((sync && cudaMemsetAsync(p.bad, 0, sizeof(int), st) != cudaSuccess) ||
            allow_smem(bwd_tc_query_kernel, q_smem) != cudaSuccess ||
            allow_smem(bwd_tc_key_kernel, k_smem) != cudaSuccess ||
            allow_smem(lce_kern, l_smem) != cudaSuccess) {
            rc = BRA_ERR_CUDA;
        } else {
            {
                LaunchScope ls(BRA_KERNEL_BACKWARD, st);
                bwd_tc_transpose_kernel<<<s.N, 256, tr_smem, st>>>(p);
            }
            {  // the LCE part of dv (the key kernel adds the attention part) and the LCE partials
                LaunchScope ls(BRA_KERNEL_BACKWARD, st);
                lce_kern<<<ng * G, kLceThreads, l_smem, st>>>(p, static_cast<const __nv_bfloat16 *>(lce_w), part, G);
            }
            {
                LaunchScope ls(BRA_KERNEL_BACKWARD, st);
                bwd_tc_query_kernel<<<units, 32 * nw, q_smem, st>>>(p);
            }
            {
                LaunchScope ls(BRA_KERNEL_BACKWARD, st);
                bwd_tc_key_kernel<<<units, 32 * nw, k_smem, st>>>(p);
            }
            {
                LaunchScope ls(BRA_KERNEL_BACKWARD, st);
                bwd_tc_lce_final_kernel<<<(s.C * 26 * 32 + 255) / 256, 256, 0, st>>>(part, G, s.C, pg, dlce_w, dlce_b);
            }
            if (cudaGetLastError() != cudaSuccess) rc = BRA_ERR_CUDA;
        }
    }
    int host_flag = 0;
    if (sync && rc == BRA_OK &&
        cudaMemcpyAsync(&host_flag, p.bad, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        rc = BRA_ERR_CUDA;
    if (cudaFreeAsync(buf, st) != cudaSuccess && rc == BRA_OK) rc = BRA_ERR_CUDA;
    if (sync && cudaStreamSynchronize(st) != cudaSuccess && rc == BRA_OK) rc = BRA_ERR_CUDA;
    if (rc == BRA_OK && host_flag) rc = BRA_ERR_INDEX;
    return rc;
}

static int backward_impl(const void *q, const void *k, const void *v, const void *lce_w, const int32_t *r_idx,
                         const void *dout, int N, int H, int W, int C, int heads, int S, int topk, int dtype,
                         float *dq, float *dk, float *dv, float *dlce_w, float *dlce_b, bra_stream_t stream,
                         bool sync) {
    const Shape s = make_shape(N, H, W, C, heads, S, topk, dtype);
    int rc = check_shape(s);
    if (rc) return rc;
    if (s.padded()) return BRA_ERR_SHAPE;  // the backward runs on multiples of S only
    if (!lce_w || !dlce_w || !dlce_b) return BRA_ERR_NULL;
    if (!aligned(dlce_w, 4) || !aligned(dlce_b, 4)) return BRA_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (N == 0) {  // the parameter gradients of an empty batch are zero
        if (cudaMemsetAsync(dlce_w, 0, (size_t)C * 25 * sizeof(float), st) != cudaSuccess ||
            cudaMemsetAsync(dlce_b, 0, (size_t)C * sizeof(float), st) != cudaSuccess)
            return BRA_ERR_CUDA;
        return BRA_OK;
    }
    if (!q || !k || !v || !r_idx || !dout || !dq || !dk || !dv) return BRA_ERR_NULL;
    const size_t es = dtype == BRA_BF16 ? 2 : 4;
    if (!aligned(q, es) || !aligned(k, es) || !aligned(v, es) || !aligned(dout, es) || !aligned(lce_w, es) ||
        !aligned(r_idx, 4) || !aligned(dq, 4) || !aligned(dk, 4) || !aligned(dv, 4))
        return BRA_ERR_ALIGN;
    int sms = 0;
    if ((rc = sm_count(&sms))) return rc;
    // the tensor-core kernels move 16-byte pieces of q, k, v, dout and dv and store float2 gradients
    const bool tc = dtype == BRA_BF16 && s.d == 32 && aligned(q, 16) && aligned(k, 16) && aligned(v, 16) &&
                    aligned(dout, 16) && aligned(dq, 8) && aligned(dk, 8) && aligned(dv, 16);
    if (tc) return backward_tc(s, q, k, v, lce_w, r_idx, dout, dq, dk, dv, dlce_w, dlce_b, st, sync);
    int *flag = nullptr;  // per call (read back here), or the library's device flag
    if (sync ? cudaMallocAsync(reinterpret_cast<void **>(&flag), sizeof(int), st) != cudaSuccess
             : index_flag(&flag) != BRA_OK)
        return BRA_ERR_CUDA;
    const BwdParams p = make_bwd_params(q, k, v, dout, lce_w, r_idx, N, H, W, C, heads, S, topk, dtype == BRA_BF16,
                                        dq, dk, dv, dlce_w, dlce_b, flag);
    const size_t elems = bwd_elems(p), items = bwd_attn_items(p);
    rc = (!sync || cudaMemsetAsync(flag, 0, sizeof(int), st) == cudaSuccess) &&
                 cudaMemsetAsync(dk, 0, elems * sizeof(float), st) == cudaSuccess
             ? BRA_OK
             : BRA_ERR_CUDA;
    if (rc == BRA_OK) {
        {
            LaunchScope ls(BRA_KERNEL_BACKWARD, st);
            bwd_lce_dv_kernel<<<(unsigned)std::min<size_t>((elems + 255) / 256, (size_t)sms * 8), 256, 0, st>>>(p);
        }
        {
            LaunchScope ls(BRA_KERNEL_BACKWARD, st);
            bwd_attn_kernel<<<(unsigned)std::min<size_t>((items + 127) / 128, (size_t)sms * 16), 128, 0, st>>>(p);
        }
        {
            LaunchScope ls(BRA_KERNEL_BACKWARD, st);
            bwd_lce_param_kernel<<<C * 26, 256, 0, st>>>(p);
        }
        if (cudaGetLastError() != cudaSuccess) rc = BRA_ERR_CUDA;
    }
    if (!sync) return rc;
    int host_flag = 0;
    if (rc == BRA_OK &&
        cudaMemcpyAsync(&host_flag, flag, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        rc = BRA_ERR_CUDA;
    if (cudaFreeAsync(flag, st) != cudaSuccess && rc == BRA_OK) rc = BRA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess && rc == BRA_OK) rc = BRA_ERR_CUDA;
    if (rc == BRA_OK && host_flag) rc = BRA_ERR_INDEX;
    return rc;
}

int bra_backward(const void *q, const void *k, const void *v, const void *lce_w, const int32_t *r_idx,
                 const void *dout, int N, int H, int W, int C, int heads, int S, int topk, int dtype, float *dq,
                 float *dk, float *dv, float *dlce_w, float *dlce_b, bra_stream_t stream) {
    return backward_impl(q, k, v, lce_w, r_idx, dout, N, H, W, C, heads, S, topk, dtype, dq, dk, dv, dlce_w, dlce_b,
                         stream, true);
}

int bra_backward_async(const void *q, const void *k, const void *v, const void *lce_w, const int32_t *r_idx,
                       const void *dout, int N, int H, int W, int C, int heads, int S, int topk, int dtype,
                       float *dq, float *dk, float *dv, float *dlce_w, float *dlce_b, bra_stream_t stream) {
    return backward_impl(q, k, v, lce_w, r_idx, dout, N, H, W, C, heads, S, topk, dtype, dq, dk, dv, dlce_w, dlce_b,
                         stream, false);
}

int bra_attend(const void *q, const void *k, const void *v, const void *lce_w, const void *lce_b, int N,
               int H, int W, int C, int heads, int S, int topk, int dtype, const int32_t *r_idx, void *out,
               bra_stream_t stream) {
    const Shape s = make_shape(N, H, W, C, heads, S, topk, dtype);
    int rc = check_plan(s);
    if (rc) return rc;
    if (N == 0) return BRA_OK;
    if (!q || !k || !v || !lce_w || !lce_b || !out || !r_idx) return BRA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(r_idx, 4))
        return BRA_ERR_ALIGN;
    const size_t es = dtype == BRA_BF16 ? 2 : 4;
    if (!aligned(lce_w, es) || !aligned(lce_b, es)) return BRA_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int *flag = nullptr;
    if (cudaMallocAsync(reinterpret_cast<void **>(&flag), sizeof(int), st) != cudaSuccess) return BRA_ERR_CUDA;
    int host_flag = 0;
    rc = cudaMemsetAsync(flag, 0, sizeof(int), st) == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
    if (rc == BRA_OK && s.padded()) {
        // the padded grid: zero-padded copies of q, k, v, the attention on them, the crop
        const size_t map = padded_map_bytes(s);
        unsigned char *buf = nullptr;
        if (cudaMallocAsync(reinterpret_cast<void **>(&buf), 4 * map, st) != cudaSuccess) {
            rc = BRA_ERR_CUDA;
        } else {
            const void *src[3] = {q, k, v};
            void *dst[3] = {buf, buf + map, buf + 2 * map};
            rc = launch_pad(s, 3, src, dst, st);
            if (rc == BRA_OK)
                rc = launch_attend(padded_shape(s), dst[0], dst[1], dst[2], lce_w, lce_b, buf + 3 * map, r_idx, flag,
                                   st);
            if (rc == BRA_OK) rc = launch_crop(s, buf + 3 * map, out, st);
            if (cudaFreeAsync(buf, st) != cudaSuccess && rc == BRA_OK) rc = BRA_ERR_CUDA;
        }
    } else if (rc == BRA_OK) {
        rc = launch_attend(s, q, k, v, lce_w, lce_b, out, r_idx, flag, st);
    }
    if (rc == BRA_OK &&
        cudaMemcpyAsync(&host_flag, flag, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        rc = BRA_ERR_CUDA;
    if (cudaFreeAsync(flag, st) != cudaSuccess && rc == BRA_OK) rc = BRA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess && rc == BRA_OK) rc = BRA_ERR_CUDA;
    if (rc == BRA_OK && host_flag) rc = BRA_ERR_INDEX;
    return rc;
}

int bra_forward_host(const void *q, const void *k, const void *v, const void *lce_w, const void *lce_b, int N,
                     int H, int W, int C, int heads, int S, int topk, int dtype, void *out, int32_t *r_idx,
                     float *r_weight, bra_stream_t stream) {
    const Shape s = make_shape(N, H, W, C, heads, S, topk, dtype);
    int rc = check_plan(s);
    if (rc) return rc;
    if (N == 0) return BRA_OK;
    if (!q || !k || !v || !lce_w || !lce_b || !out || !r_idx || !r_weight) return BRA_ERR_NULL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t es = dtype == BRA_BF16 ? 2 : 4;
    const size_t img = (size_t)H * W * C * es, map = (size_t)N * img, wb = (size_t)C * 25 * es, bb = (size_t)C * es;
    const size_t rimg = (size_t)s.P * topk * 4, route = (size_t)N * rimg;
    const size_t scratch = 2 * (size_t)N * s.P * C * sizeof(float);
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t total = 4 * up(map) + up(wb) + up(bb) + 2 * up(route) + up(scratch);
    cudaMemPool_t pool = nullptr;
    cudaStream_t up_st = nullptr, back = nullptr;
    if (host_call_pool(&pool, &up_st, &back) != BRA_OK) return BRA_ERR_CUDA;
    char *base = nullptr;
    if (cudaMallocFromPoolAsync(reinterpret_cast<void **>(&base), total, pool, st) != cudaSuccess) return BRA_ERR_CUDA;
    char *dq = base, *dk = dq + up(map), *dv = dk + up(map), *dout = dv + up(map), *dw = dout + up(map);
    char *db = dw + up(wb), *di = db + up(bb), *dr = di + up(route);
    float *dws = reinterpret_cast<float *>(dr + up(route));
    // Images are independent: the batch goes in chunks over three streams. The inputs
    // stream in back to back on one copy stream, chunk c is computed on `stream` once its
    // inputs are in, and its results go back on a second copy stream while later chunks
    // are still coming in.
    const int nchunk = N < 8 ? N : 8, per = (N + nchunk - 1) / nchunk;
    std::vector<cudaEvent_t> ev;
    auto event = [&](cudaEvent_t *e) {
        if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return false;
        ev.push_back(*e);
        return true;
    };
    rc = BRA_OK;
    cudaEvent_t e_alloc = nullptr;
    if (!event(&e_alloc) || cudaEventRecord(e_alloc, st) != cudaSuccess ||
        cudaStreamWaitEvent(up_st, e_alloc, 0) != cudaSuccess ||
        cudaMemcpyAsync(dw, lce_w, wb, cudaMemcpyHostToDevice, up_st) != cudaSuccess ||
        cudaMemcpyAsync(db, lce_b, bb, cudaMemcpyHostToDevice, up_st) != cudaSuccess)
        rc = BRA_ERR_CUDA;
    for (int n0 = 0; n0 < N && rc == BRA_OK; n0 += per) {
        const int nb = N - n0 < per ? N - n0 : per;
        const size_t o = (size_t)n0 * img, ob = (size_t)nb * img, ro = (size_t)n0 * rimg, rb = (size_t)nb * rimg;
        cudaEvent_t e_in = nullptr, e_out = nullptr;
        if (!event(&e_in) || !event(&e_out) ||
            cudaMemcpyAsync(dq + o, static_cast<const char *>(q) + o, ob, cudaMemcpyHostToDevice, up_st) != cudaSuccess ||
            cudaMemcpyAsync(dk + o, static_cast<const char *>(k) + o, ob, cudaMemcpyHostToDevice, up_st) != cudaSuccess ||
            cudaMemcpyAsync(dv + o, static_cast<const char *>(v) + o, ob, cudaMemcpyHostToDevice, up_st) != cudaSuccess ||
            cudaEventRecord(e_in, up_st) != cudaSuccess || cudaStreamWaitEvent(st, e_in, 0) != cudaSuccess) {
            rc = BRA_ERR_CUDA;
            break;
        }
        Shape sc = s;
        sc.N = nb;
        rc = forward_device(sc, dq + o, dk + o, dv + o, dw, db, dout + o, reinterpret_cast<int32_t *>(di + ro),
                            reinterpret_cast<float *>(dr + ro), st, dws + (size_t)n0 * 2 * s.P * C);
        if (rc != BRA_OK) break;
        if (cudaEventRecord(e_out, st) != cudaSuccess || cudaStreamWaitEvent(back, e_out, 0) != cudaSuccess ||
            cudaMemcpyAsync(static_cast<char *>(out) + o, dout + o, ob, cudaMemcpyDeviceToHost, back) != cudaSuccess ||
            cudaMemcpyAsync(reinterpret_cast<char *>(r_idx) + ro, di + ro, rb, cudaMemcpyDeviceToHost, back) !=
                cudaSuccess ||
            cudaMemcpyAsync(reinterpret_cast<char *>(r_weight) + ro, dr + ro, rb, cudaMemcpyDeviceToHost, back) !=
                cudaSuccess)
            rc = BRA_ERR_CUDA;
    }
    // `stream` takes over both copy streams, then releases the buffers
    cudaEvent_t e_up = nullptr, e_back = nullptr;
    if (!event(&e_up) || !event(&e_back) || cudaEventRecord(e_up, up_st) != cudaSuccess ||
        cudaEventRecord(e_back, back) != cudaSuccess || cudaStreamWaitEvent(st, e_up, 0) != cudaSuccess ||
        cudaStreamWaitEvent(st, e_back, 0) != cudaSuccess)
        rc = rc == BRA_OK ? BRA_ERR_CUDA : rc;
    if (cudaFreeAsync(base, st) != cudaSuccess && rc == BRA_OK) rc = BRA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess && rc == BRA_OK) rc = BRA_ERR_CUDA;
    for (cudaEvent_t e : ev) cudaEventDestroy(e);
    return rc;
}

// ----------------------------------------------------------------------------- no-allocation variant
//
// bra_forward_noalloc keeps its scratch (the pooled region means of q and k) in
// this file-scope device array instead of the memory pool. Host code must not
// pass the symbol itself to a kernel: on the host it names a host-side shadow,
// so the device address is looked up with cudaGetSymbolAddress on the current
// device. The lookup is repeated on every call (it is cheap once the module is
// loaded) rather than cached, so that a context created anew on the device (after
// cudaDeviceReset) never receives an address from the old one.

static __device__ __align__(256) float g_static_scratch[BRA_STATIC_SCRATCH_FLOATS];

// Device address of g_static_scratch on the current device.
static int static_scratch(float **out) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return BRA_ERR_CUDA;
    *out = static_cast<float *>(p);
    return BRA_OK;
}

int bra_forward_noalloc(const void *q, const void *k, const void *v, const void *lce_w, const void *lce_b,
                        int N, int H, int W, int C, int heads, int S, int topk, int dtype, void *out,
                        int32_t *r_idx, float *r_weight, bra_stream_t stream) {
    const Shape s = make_shape(N, H, W, C, heads, S, topk, dtype);
    int rc = check_plan(s);
    if (rc) return rc;
    if (N == 0) return BRA_OK;
    if (!q || !k || !v || !lce_w || !lce_b || !out || !r_idx || !r_weight) return BRA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(r_idx, 4) ||
        !aligned(r_weight, 4))
        return BRA_ERR_ALIGN;
    const size_t es = dtype == BRA_BF16 ? 2 : 4;
    if (!aligned(lce_w, es) || !aligned(lce_b, es)) return BRA_ERR_ALIGN;
    if (2 * (size_t)N * s.P * C > (size_t)BRA_STATIC_SCRATCH_FLOATS) return BRA_ERR_SCRATCH;
    if (s.padded()) return BRA_ERR_SCRATCH;  // the padded copies would need more scratch
    float *ws = nullptr;
    rc = static_scratch(&ws);
    if (rc) return rc;
    // the same kernels as bra_forward (the one-kernel fused forms use no scratch at all),
    // with the static array standing in for the pool's scratch
    return forward_device(s, q, k, v, lce_w, lce_b, out, r_idx, r_weight, reinterpret_cast<cudaStream_t>(stream), ws);
}

}  // extern "C"
