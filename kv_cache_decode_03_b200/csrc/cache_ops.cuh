// cache_ops.cuh -- N4: the bookkeeping steps around a speculative verify and a shared
// prefix ("llm-perf-lab" README: two-phase append/commit, and speculative decoding keeps
// the accepted prefix of the verified tokens; "9. 推理" 9.6: a paged cache in blocks).
//
//   commit_kernel      seq_lens[b] += accepted[b]  (0 <= accepted[b] <= T_new)
//   rollback_kernel    seq_lens[b] -= drop[b]      (0 <= drop[b] <= seq_lens[b])
//   copy_pages_kernel  page dst[i] := page src[i] in every layer, K and V (the copy of
//                      copy-on-write, before an append into a page other requests share)
//
// A violation skips that request (or page pair) and sets the sticky error word; nothing
// traps.
#pragma once

#include <stdint.h>

#include "device_common.cuh"

namespace kvc {

__global__ void commit_kernel(int32_t* seq_lens, const int32_t* accepted, int B, int T_new,
                              int max_T, int* err) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int a = accepted[b];
  const int L = seq_lens[b];
  if (a < 0 || a > T_new || L < 0 || (long long)L + a > max_T) {
    flag_error(err, KVC_ERR_BOUNDS);
    return;
  }
  seq_lens[b] = L + a;
}

__global__ void rollback_kernel(int32_t* seq_lens, const int32_t* drop, int B, int* err) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int d = drop[b];
  const int L = seq_lens[b];
  if (d < 0 || d > L) {
    flag_error(err, KVC_ERR_BOUNDS);
    return;
  }
  seq_lens[b] = L - d;
}

// One CTA per (pair, layer, K or V): the page is page_vecs 16-byte vectors, contiguous
// at page * page_vecs in its pool.  pool_base: layer l's K pool at 2l * layer_vecs, V at
// (2l + 1) * layer_vecs.
__global__ void copy_pages_kernel(uint4* pool_base, size_t layer_vecs, const int32_t* src,
                                  const int32_t* dst, int n, int num_layers, int num_pages,
                                  int page_vecs, int* err) {
  const int pair = blockIdx.x;
  const int which = blockIdx.y;  // 2 * layer + (0 = K, 1 = V)
  if (pair >= n || which >= 2 * num_layers) return;
  const int s = src[pair];
  const int d = dst[pair];
  if (s < 0 || s >= num_pages || d < 0 || d >= num_pages) {
    if (threadIdx.x == 0 && which == 0) flag_error(err, KVC_ERR_BOUNDS);
    return;
  }
  const uint4* from = pool_base + (size_t)which * layer_vecs + (size_t)s * page_vecs;
  uint4* to = pool_base + (size_t)which * layer_vecs + (size_t)d * page_vecs;
#pragma unroll 4
  for (int i = threadIdx.x; i < page_vecs; i += blockDim.x) to[i] = from[i];
}

}  // namespace kvc
