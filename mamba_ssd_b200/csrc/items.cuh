// items.cuh -- walking a contiguous range of (sequence, block, head) work items without division.
//
// The tensor-core prefill kernels give each persistent CTA a contiguous range of items ordered
// (sequence, block, group, head within group), head fastest, so consecutive items of one
// (sequence, block, group) share that block's B / C tiles.  A single issuing lane that decodes
// every item with runtime integer divisions spends ~100 cycles per division, which starves
// the tensor core; the cursor decodes the first item once and then steps by increments.
//
// Two kinds of batch.  An equal-length batch: B sequences of L tokens, sequence b at index b
// of the tensors' batch dimension, ceil(L/128) blocks each.  A packed varlen batch: the
// non-empty sequences of one token stream (batch dimension 1), sequence j holding tokens
// tok0[j] .. tok0[j+1]-1 and workspace blocks blk0[j] .. blk0[j+1]-1.  In both, the items of
// global block gb (gb = b * nk + k, or blk0[j] + k) are gb * H .. gb * H + H - 1, and the
// workspace arrays are indexed by gb.
#pragma once

namespace ssd {

constexpr int kItemBlock = 128;  // tokens per block (the M of one tcgen05 MMA)

// The packed varlen batch's table (device memory), n + 1 entries in tok0 and blk0 (an end
// sentinel), n in seq (each sequence's index among the caller's sequences, empty ones
// included: where its h0 and h_final are).  n = 0: an equal-length batch.
struct Varlen {
    const int *tok0, *blk0, *seq;
    int n;
};

// VARLEN selects the batch kind at compile time, so that the equal-length kernels carry none
// of the table lookups.
template <bool VARLEN>
struct ItemCursor {
    int b, k, g, hh;  // sequence, 128-token block within it, group, head within the group
    int nk;           // blocks of sequence b
    int G, hpg;
    int row0;  // first token of sequence b along the tensors' token dimension
    int blk0;  // global block of (b, k = 0)
    int len;   // tokens of sequence b
    int zb;    // sequence b's index along the tensors' batch dimension
    Varlen vl;

    // first: the first item; nk_eq, L: blocks and tokens per sequence of an equal-length batch
    __device__ __forceinline__ ItemCursor(int first, int H, int G_, int nk_eq, int L, const Varlen &v)
        : G(G_), hpg(H / G_), vl(v) {
        const int h = first % H, t = first / H;  // t: global block
        g = h / hpg;
        hh = h - g * hpg;
        if (!VARLEN) {
            nk = nk_eq;
            k = t % nk_eq;
            b = t / nk_eq;
            row0 = 0;
            blk0 = b * nk_eq;
            len = L;
            zb = b;
        } else {
            int lo = 0, hi = v.n - 1;  // the last sequence whose first block is <= t
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (v.blk0[mid] <= t) lo = mid;
                else hi = mid - 1;
            }
            b = lo;
            load_sequence();
            k = t - blk0;
        }
    }
    __device__ __forceinline__ void load_sequence() {
        zb = 0;
        if (b < vl.n) {
            row0 = vl.tok0[b];
            len = vl.tok0[b + 1] - row0;
            blk0 = vl.blk0[b];
            nk = vl.blk0[b + 1] - blk0;
        }
    }
    __device__ __forceinline__ int h() const { return g * hpg + hh; }
    __device__ __forceinline__ int row() const { return row0 + k * kItemBlock; }  // the block's first token
    __device__ __forceinline__ int gblk() const { return blk0 + k; }              // the block's workspace index
    __device__ __forceinline__ int valid() const {                               // the block's real tokens
        const int v = len - k * kItemBlock;
        return v < kItemBlock ? v : kItemBlock;
    }
    // first / last item of its (sequence, block, group) tile
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
                    if (VARLEN) {
                        load_sequence();
                    } else {
                        blk0 += nk;
                        zb = b;
                    }
                }
            }
        }
    }
};

}  // namespace ssd
