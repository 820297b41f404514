// pad.cuh — the padded grid for feature maps whose height or width is not a multiple
// of S (bernice.tw BiFormer notes, section "消融實驗": padding the map costs compute,
// which is why S is chosen per task).
//
// Reading taken: q, k and v are zero-padded at the bottom and the right to
// Hp = S*ceil(H/S) rows and Wp = S*ceil(W/S) columns, the forward runs on the padded
// maps (region means over whole padded regions, padded tokens taking part as keys with
// k = v = 0), and only the H x W real outputs are kept. These two kernels are the
// copies around that forward: the zero-padded copy of up to three maps in one launch,
// and the crop of the padded output. Both move whole pixels as 16-byte chunks (a pixel
// of C channels is C*es bytes, a multiple of 64 for the supported C), one CTA per
// destination row.
#pragma once

#include <cstdint>

namespace bra {

constexpr int kPadThreads = 256;

struct PadParams {
    const uint4 *src[3];
    uint4 *dst[3];
    int N, H, W, Hp, Wp;
    int cv;  // 16-byte chunks per pixel
};

// blockIdx.x = (map * N + n) * Hp + y over the padded rows of every map. A row
// below H, and the columns at or beyond W of any row, are written as zeros.
__global__ void __launch_bounds__(kPadThreads) pad_maps_kernel(const PadParams p) {
    const int row = blockIdx.x;
    const int y = row % p.Hp, img = row / p.Hp;  // img = map * N + n
    const int map = img / p.N, n = img - map * p.N;
    const int real = y < p.H ? p.W * p.cv : 0;   // chunks copied from the source row
    const int total = p.Wp * p.cv;
    uint4 *dst = p.dst[map] + ((size_t)n * p.Hp + y) * total;
    const uint4 *src = p.src[map] + ((size_t)n * p.H + (y < p.H ? y : 0)) * (size_t)p.W * p.cv;
    for (int e = threadIdx.x; e < total; e += kPadThreads)
        dst[e] = e < real ? __ldg(src + e) : make_uint4(0u, 0u, 0u, 0u);
}

// blockIdx.x = n * H + y over the real output rows: the first W pixels of padded row y.
__global__ void __launch_bounds__(kPadThreads) crop_map_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst,
                                                               int H, int W, int Hp, int Wp, int cv) {
    const int row = blockIdx.x;
    const int y = row % H, n = row / H;
    const int total = W * cv;
    const uint4 *s = src + ((size_t)n * Hp + y) * (size_t)Wp * cv;
    uint4 *d = dst + ((size_t)n * H + y) * (size_t)total;
    for (int e = threadIdx.x; e < total; e += kPadThreads) d[e] = __ldg(s + e);
}

}  // namespace bra
