// items.cuh -- walking a contiguous range of (batch, block, head) work items without division.
//
// The tensor-core prefill kernels give each persistent CTA a contiguous range of items ordered
// (batch, block, group, head within group), head fastest, so consecutive items of one
// (batch, block, group) share that block's B / C tiles.  A single issuing lane that decodes
// every item with runtime integer divisions spends ~100 cycles per division, which starves
// the tensor core; the cursor decodes the first item once and then steps by increments.
#pragma once

namespace ssd {

struct ItemCursor {
    int b, k, g, hh;  // batch, 128-token block, group, head within the group
    int nk, G, hpg;

    __device__ __forceinline__ ItemCursor(int first, int H, int G_, int nk_) : nk(nk_), G(G_), hpg(H / G_) {
        const int h = first % H, t = first / H;
        k = t % nk;
        b = t / nk;
        g = h / hpg;
        hh = h - g * hpg;
    }
    __device__ __forceinline__ int h() const { return g * hpg + hh; }
    // first / last item of its (batch, block, group) tile
    __device__ __forceinline__ bool tile_first() const { return hh == 0; }
    __device__ __forceinline__ bool tile_last() const { return hh == hpg - 1; }
    __device__ __forceinline__ void next() {
        if (++hh == hpg) {
            hh = 0;
            if (++g == G) {
                g = 0;
                if (++k == nk) {
                    k = 0;
                    ++b;
                }
            }
        }
    }
};

}  // namespace ssd
