// Host execution of the backward kernels' per-item code (csrc/backward.cuh), for the CPU
// tests: the same functions the kernels call, in the same partition (the dv pass, the
// zeroed dk, every attention item, the 256-way partial sums of the parameter gradients),
// with every memory access checked against its buffer (BRA_BWD_HOST_CHECK).
// Test infrastructure: built by tests/test_backward_host.py, not part of the library.
#include <cstdio>

#define BRA_BWD_HOST_CHECK 1
#include "../../vision_transformer_sparse_b200/csrc/backward.cuh"

namespace bra {
static long long g_bounds_failures = 0;
void bra_bwd_host_bounds_failure(const char *what, long long i, long long n) {
    if (g_bounds_failures++ == 0) fprintf(stderr, "out of bounds: %s index %lld of %lld\n", what, i, n);
}
}  // namespace bra

// Returns the number of out-of-bounds accesses (0 when every access was in range).
extern "C" long long bwd_host_run(const void *q, const void *k, const void *v, const void *dout, const void *lce_w,
                                  const int32_t *r_idx, int N, int H, int W, int C, int heads, int S, int topk,
                                  int bf16, float *dq, float *dk, float *dv, float *dw, float *db, int *bad_index) {
    using namespace bra;
    g_bounds_failures = 0;
    const BwdParams p = make_bwd_params(q, k, v, dout, lce_w, r_idx, N, H, W, C, heads, S, topk, bf16 != 0, dq, dk,
                                        dv, dw, db, bad_index);
    const size_t el = bwd_elems(p);
    for (size_t i = 0; i < el; ++i) p.dv[i] = bwd_lce_dv(p, i);  // bwd_lce_dv_kernel
    for (size_t i = 0; i < el; ++i) p.dk[i] = 0.f;               // the stream-ordered memset
    const size_t items = bwd_attn_items(p);
    for (size_t i = 0; i < items; ++i) bwd_attn_item(p, i);  // bwd_attn_kernel
    for (int c = 0; c < C; ++c)                              // bwd_lce_param_kernel: CTA (c, tap)
        for (int tap = 0; tap < 26; ++tap) {
            float acc = 0.f;
            for (int t = 0; t < 256; ++t) acc += bwd_lce_param_partial(p, c, tap, (size_t)t, 256);
            if (tap == 25)
                p.db[c] = acc;
            else
                p.dw[c * 25 + tap] = acc;
        }
    return g_bounds_failures;
}
