// window.cuh -- which cached positions a query row sees under a sliding window with
// attention sinks ("项目 9-16" roadmap: sliding-window attention keeps the last W
// positions, StreamingLLM-style sinks keep the first S as well).
//
// A row with n visible positions (n = L + i + 1, causal within the new chunk) sees
// position j iff  j < n  and  (W == 0  or  j >= n - W  or  j < S).  W == 0: no window.
//
// The fixed-split kernels walk a block's positions as VIRTUAL tiles: the positions any
// row of the block can see are the sink part [0, min(S, lo)) and the window part
// [lo, n_max), lo = n_min - W, where n_min / n_max are the block's smallest / largest n.
// At tile granularity that is tiles [0, ts) and [tw0, ceil(n_max / T)); the virtual
// tile list is their concatenation (one range when they touch), so a split of the
// virtual list reads nothing outside the window and every virtual tile is a contiguous
// run of real positions.
#pragma once

#include "device_common.cuh"

namespace kvc {

struct Span {
  int ts_tok;  // virtual positions below this are real positions (the sink tiles)
  int shift;   // at or above it: real = virtual + shift (the window tiles)
  int n_virt;  // virtual positions the block reads: [0, n_virt)
  __device__ __forceinline__ int real(int v) const { return v < ts_tok ? v : v + shift; }
  // `pos` must lie in the sink part or in the window part
  __device__ __forceinline__ int virt(int pos) const { return pos < ts_tok ? pos : pos - shift; }
};

__device__ __forceinline__ Span block_span(int n_min, int n_max, int W, int S, int T) {
  Span sp{n_max, 0, n_max};
  if (W <= 0) return sp;
  const int lo = max(0, n_min - W);
  const int ts = ceil_div(min(S, lo), T);
  const int tw0 = lo / T;
  if (tw0 > ts) {
    sp.ts_tok = ts * T;
    sp.shift = (tw0 - ts) * T;
    sp.n_virt = n_max - sp.shift;
  }
  return sp;
}

__device__ __forceinline__ bool visible(int pos, int n, int W, int S) {
  return pos < n && (W <= 0 || pos >= n - W || pos < S);
}

// Every row of the block (n in [n_min, n_max]) sees all of [t0, t0 + T).
__device__ __forceinline__ bool tile_fully_visible(int t0, int T, int n_min, int n_max, int W,
                                                   int S) {
  return t0 + T <= n_min && (W <= 0 || t0 >= n_max - W || t0 + T <= S);
}

}  // namespace kvc
