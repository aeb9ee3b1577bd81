// Expert parallelism, the expert side: the rows a rank receives arrive
// grouped by source rank (sources in rank order), within a source by local
// expert; the expert GEMMs want them grouped by local expert.  The host
// computes the small tables (per (source, expert) block: its start in the
// received order and in the grouped order); this kernel expands them to the
// per-row permutation.  (LatentMoE paper, Section 2.2 and the paragraph
// after Eq. (1): dispatch and aggregation in the latent width.)
#pragma once

#include "common.cuh"
#include "routing.cuh"

namespace lmoe {

// For every received row r < Rr: its source s (the block of s starts at
// src_start[s]), its local expert e (the (s, e) block starts at roff[s*n+e]
// in received order and at goff[e*world+s] in grouped order), and its grouped
// row g = goff[e*world+s] + (r - roff[s*n+e]).  Writes perm[g] = r (the FC1
// gather index), inv[r] = g (to return the outputs in received order) and
// gates_g[g] = gates[r] (the FC2 epilogue's row scale).
__global__ void __launch_bounds__(256) ep_perm_kernel(long Rr, int world, int n,
                                                      const int* __restrict__ src_start,
                                                      const int* __restrict__ roff,
                                                      const int* __restrict__ goff,
                                                      const float* __restrict__ gates,
                                                      int* __restrict__ perm, int* __restrict__ inv,
                                                      float* __restrict__ gates_g) {
  griddep_launch();
  griddep_wait();  // the previous kernel's outputs are visible
  for (long r = (long)blockIdx.x * blockDim.x + threadIdx.x; r < Rr;
       r += (long)gridDim.x * blockDim.x) {
    int lo = 0, hi = world - 1;  // largest s with src_start[s] <= r
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(src_start + mid) <= r) lo = mid; else hi = mid - 1;
    }
    const int s = lo;
    const int* ro = roff + (size_t)s * n;
    lo = 0;
    hi = n - 1;  // largest e with ro[e] <= r
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(ro + mid) <= r) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const long g = (long)__ldg(goff + (size_t)e * world + s) + (r - __ldg(ro + e));
    perm[g] = (int)r;
    inv[r] = (int)g;
    gates_g[g] = __ldg(gates + r);
  }
}

// The tile prefixes of the received rows' grouping over the n local experts
// (counts[e] rows each): one block runs the routing's scan.
__global__ void __launch_bounds__(256) ep_scan_kernel(const int* __restrict__ counts, int n,
                                                      int* offsets, int* tp128, int* tp256,
                                                      int* tp64, int* big256, int* small128,
                                                      int* small256) {
  griddep_launch();
  griddep_wait();  // the previous kernel's outputs are visible
  scan_loads_block(counts, n, offsets, tp128, tp256, tp64, big256, small128, small256);
}

}  // namespace lmoe
