// combine.cuh -- N3: merge split-K slice results by log-sum-exp.
//
// A slice s of a query row holds o_s = (sum_j e^{x_j - m_s} V_j) / l_s and
// lse_s = m_s + log2 l_s (base 2).  With M = max_s lse_s the exact result is
//   out = sum_s 2^{lse_s - M} o_s / sum_s 2^{lse_s - M},
// which is softmax over the union of the slices ("9. 推理" 9.7: tiling keeps
// attention exact up to rounding).  One warp per query row; each lane owns
// D/32 output elements.  Rows that fit in one slice were finished by the
// attend kernel and are skipped.
#pragma once

#include "device_common.cuh"
#include "params.cuh"

namespace kvc {

template <int D, typename T>
__global__ void __launch_bounds__(256) combine_kernel(const AttendParams p) {
  constexpr int E = D / 32;
  const int row = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  const int nrows = p.B * p.H_q * p.T_new;
  if (row >= nrows) return;
  const int i = row % p.T_new;
  const int b = row / (p.T_new * p.H_q);
  const int L = p.seq_lens[b];
  if (L < 0 || L + p.T_new > p.max_T) return;  // flagged by the attend kernel
  const int ns = ceil_div(L + i + 1, p.split_tokens);
  if (ns <= 1) return;
  if (ns > p.num_splits) {
    if (lane == 0) flag_error(p.err, KVC_ERR_BOUNDS);
    return;
  }
  const float* lse = p.ws_lse + (size_t)row * p.num_splits;
  float M = -INFINITY;
  for (int s = lane; s < ns; s += 32) M = fmaxf(M, lse[s]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float den = 0.f;
  for (int s = lane; s < ns; s += 32) den += exp2f(lse[s] - M);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);

  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  const float* o = p.ws_o + (size_t)row * p.num_splits * D + lane * E;
#pragma unroll 1
  for (int s = 0; s < ns; ++s) {
    const float w = exp2f(lse[s] - M);
    const float* os = o + (size_t)s * D;
    if constexpr (E == 4) {
      const float4 v = *reinterpret_cast<const float4*>(os);
      acc[0] = fmaf(w, v.x, acc[0]);
      acc[1] = fmaf(w, v.y, acc[1]);
      acc[2] = fmaf(w, v.z, acc[2]);
      acc[3] = fmaf(w, v.w, acc[3]);
    } else if constexpr (E == 2) {
      const float2 v = *reinterpret_cast<const float2*>(os);
      acc[0] = fmaf(w, v.x, acc[0]);
      acc[1] = fmaf(w, v.y, acc[1]);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(w, os[e], acc[e]);
    }
  }
  const float inv = 1.f / den;
  T* out = static_cast<T*>(p.out) + (size_t)row * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    if constexpr (Elt<T>::kCode == KVC_BF16) out[e] = __float2bfloat16_rn(acc[e] * inv);
    else out[e] = __float2half_rn(acc[e] * inv);
  }
}

}  // namespace kvc
