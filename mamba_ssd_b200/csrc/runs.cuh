// runs.cuh -- how the fused tensor-core prefill splits a call's work over persistent CTAs.
//
// The work is cut into units (batch, head pair, 128-token block), ordered with the block
// fastest, so that the units of one (batch, head pair) -- a "chain", the two heads' states
// walked along the sequence -- are consecutive.  CTA c owns the contiguous range
// [first(c), first(c+1)).  The part of a range that lies in one chain is a "run": a CTA
// carries its two heads' states through a run on chip, and only the state at each run's end
// crosses to another CTA.  A run starts either at its chain's first block or at a CTA's
// range start; it is given a slot for its state:
//   slot = chain index                  for a run that starts a chain
//   slot = number of chains + CTA index for a run that starts inside a chain
// so slots are unique and there are at most chains + CTAs of them.
//
// Plain integer arithmetic, shared by the kernels and the host (and compiled by the host
// compiler alone in a CPU test of the run enumeration).
#pragma once

#ifdef __CUDACC__
#define SSD_HD __host__ __device__ __forceinline__
#else
#define SSD_HD inline
#endif

namespace ssd {

constexpr int kPairHeads = 2;  // heads of one unit; they share the block's C B^T
constexpr int kMaxCtas = 160;  // upper bound on the fused kernels' grid (B200: 148 SMs)

struct RunLayout {
    int U;     // units: B * (H / 2) * nk
    int grid;  // CTAs, 1 .. min(U, kMaxCtas)
    int nk;    // 128-token blocks per sequence
    int nch;   // chains: B * (H / 2)

    // first unit of CTA c (c = grid gives U)
    SSD_HD int first(int c) const { return (int)((long long)c * U / grid); }
    // the CTA whose range holds unit u: the largest c with first(c) <= u
    SSD_HD int cta_of(int u) const { return (int)(((long long)(u + 1) * grid - 1) / U); }
    // slot of the run that starts at unit u in CTA c
    SSD_HD int slot(int u, int c) const { return (u % nk == 0) ? u / nk : nch + c; }
    SSD_HD int slots() const { return nch + grid; }
};

}  // namespace ssd
