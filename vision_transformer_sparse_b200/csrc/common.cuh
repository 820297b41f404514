// common.cuh — element types and small PTX helpers shared by the BRA kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bra {

// Set by any kernel whose bounded wait ran out; read and cleared by bra_device_status.
__device__ int g_bra_timeout_flag = 0;
// Set by bra_backward_async's kernels when an r_idx entry lies outside [0, S*S); read and
// cleared by bra_device_status.
__device__ int g_bra_index_flag = 0;

// ----------------------------------------------------------------------------- element types

template <typename T> struct Elem;

template <> struct Elem<float> {
    static constexpr int kVec = 4;  // elements per 16-byte vector
    __device__ static inline float to_f(float x) { return x; }
    __device__ static inline float from_f(float x) { return x; }
    // two consecutive elements as float2
    __device__ static inline float2 load2(const float *p) { return *reinterpret_cast<const float2 *>(p); }
    __device__ static inline void store2(float *p, float a, float b) {
        *reinterpret_cast<float2 *>(p) = make_float2(a, b);
    }
};

template <> struct Elem<__nv_bfloat16> {
    static constexpr int kVec = 8;
    __device__ static inline float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    __device__ static inline __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
    __device__ static inline float2 load2(const __nv_bfloat16 *p) {
        return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
    }
    __device__ static inline void store2(__nv_bfloat16 *p, float a, float b) {
        *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(a, b);
    }
};

// Unpack a 16-byte vector of T into floats.
__device__ inline void unpack16(const uint4 &u, float *f, const float *) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
}
__device__ inline void unpack16(const uint4 &u, float *f, const __nv_bfloat16 *) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// ----------------------------------------------------------------------------- invariant division

// Unsigned 32-bit division by a divisor fixed at launch, as a multiply-high and
// shifts (Granlund & Montgomery, "Division by invariant integers using
// multiplication", 1994): l = ceil(log2 d), m = floor(2^32 (2^l - d) / d) + 1,
// q = (t + ((n - t) >> 1)) >> (l - 1) with t = mulhi(m, n). Exact for every n < 2^32.
struct FastDiv {
    uint32_t d, m, s1;
    FastDiv() : d(1), m(0), s1(0) {}
    explicit FastDiv(uint32_t div) : d(div), m(0), s1(0) {
        if (d > 1) {
            uint32_t l = 0;
            while ((1ull << l) < d) ++l;
            m = (uint32_t)(((1ull << 32) * ((1ull << l) - d)) / d + 1);
            s1 = l - 1;
        }
    }
    __device__ __forceinline__ uint32_t div(uint32_t n) const {
        if (d == 1) return n;
        const uint32_t t = __umulhi(m, n);
        return (t + ((n - t) >> 1)) >> s1;
    }
    // n / d and n % d
    __device__ __forceinline__ uint32_t divmod(uint32_t n, uint32_t &r) const {
        const uint32_t q = div(n);
        r = n - q * d;
        return q;
    }
};

// ----------------------------------------------------------------------------- async copies

__device__ inline uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global -> shared copy; when `valid` is false the destination is zero-filled
// and the source is not read.
__device__ inline void cp_async16(void *smem_dst, const void *gmem_src, bool valid) {
    const int src_bytes = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem_dst)),
                 "l"(gmem_src), "r"(src_bytes)
                 : "memory");
}
// 16-byte copy to a shared address given as a 32-bit shared-window offset.
__device__ inline void cp_async16_s(uint32_t smem_dst, const void *gmem_src, bool valid) {
    const int src_bytes = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_dst), "l"(gmem_src), "r"(src_bytes)
                 : "memory");
}
// Arrive on `bar` once all prior cp.async of this thread have completed (the arrival
// is not pre-counted: the barrier's expected count includes it).
__device__ inline void cp_async_mbar_arrive_noinc(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(bar) : "memory");
}
__device__ inline void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N> __device__ inline void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// ----------------------------------------------------------------------------- warp MMA (bf16)

__device__ inline void ldsm_x4(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3, const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(smem_u32(p)));
}
__device__ inline void ldsm_x4_t(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3, const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(smem_u32(p)));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D, fp32 accumulate.
__device__ inline void mma_bf16_16816(float *d, const uint32_t *a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ inline uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// ----------------------------------------------------------------------------- packed fp32

// d = a * b + c on two float lanes at once (sm_100 packed FMA).
__device__ inline float2 ffma2(float2 a, float2 b, float2 c) {
    unsigned long long ai = *reinterpret_cast<unsigned long long *>(&a);
    unsigned long long bi = *reinterpret_cast<unsigned long long *>(&b);
    unsigned long long ci = *reinterpret_cast<unsigned long long *>(&c);
    unsigned long long di;
    asm("fma.rn.f32x2 %0, %1, %2, %3;\n" : "=l"(di) : "l"(ai), "l"(bi), "l"(ci));
    return *reinterpret_cast<float2 *>(&di);
}

__device__ inline float2 bf16x2_to_float2(uint32_t u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// ----------------------------------------------------------------------------- mbarrier / TMA / PDL

__device__ inline void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ inline void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ inline void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
// One arrival that also adds `bytes` to the transaction count of the current phase.
__device__ inline void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ inline bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}
// Bounded wait for phase `parity` of the barrier: gives up after `limit` polls
// (each poll may suspend the thread for a short hardware-defined time).
__device__ inline bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint32_t limit) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// 4-D tiled tensor load (no multicast) into shared memory, completing on `bar`.
__device__ inline void tma_load_4d(uint32_t dst, const void *tmap, int c0, int c1, int c2, int c3, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
        "%5}], [%6];\n" ::"r"(dst),
        "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
        : "memory");
}

// Programmatic dependent launch: wait for the preceding grid's results / let the
// next grid start its independent prologue.
__device__ inline void griddep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ inline void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

__device__ inline float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace bra
