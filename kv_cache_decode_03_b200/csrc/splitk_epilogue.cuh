// splitk_epilogue.cuh -- N3: finishing a split-K slice and merging slices.
//
// Every attend kernel ends the same way.  Its warps leave, per query row of
// the CTA's row block, an unnormalised weighted V sum, a running max m (base
// 2) and a running sum l in shared memory.  This code
//   1. merges the warps with the log-sum-exp rule,
//   2. writes the row's output directly when the row's visible range fits in
//      one slice, and otherwise writes the slice's normalised partial o_s and
//      lse_s = m_s + log2 l_s, and
//   3. lets the last CTA of the (request, KV head, row block) to finish merge
//      the partials: with M = max_s lse_s,
//         out = sum_s 2^(lse_s - M) o_s / sum_s 2^(lse_s - M),
//      which is exact softmax over the union of the slices ("9. 推理" 9.7).
// The last CTA is found with an atomic ticket taken after a release fence;
// nothing waits.  The ticket is reset for the next launch by the CTA that
// merged.
#pragma once

#include "device_common.cuh"
#include "params.cuh"
#include "window.cuh"

namespace kvc {

template <typename T>
__device__ __forceinline__ void store_elt(T* ptr, float v) {
  if constexpr (Elt<T>::kCode == KVC_BF16) *ptr = __float2bfloat16_rn(v);
  else *ptr = __float2half_rn(v);
}

// red_acc: [W][R] rows of D fp32, LD floats apart; red_m / red_l: [W][R].
// scratch: >= R * num_splits floats of shared memory that nothing else uses.
// flags: one shared int.  sp: the block's virtual tile span (window.cuh); slices
// count virtual positions.  All NT threads of the CTA call this together after
// red_* are written and synced.
template <typename T, int D, int R, int W, int NT, int LD = D>
__device__ __forceinline__ void finish_slice(const AttendParams& p, const float* red_acc,
                                             const float* red_m, const float* red_l,
                                             float* scratch, int* flag, int b, int g, int rb,
                                             int s, int r0, int nr, int L, int ns_blk,
                                             const Span& sp) {
  const int tid = threadIdx.x;
  T* out = static_cast<T*>(p.out);
  const size_t row_base = ((size_t)b * p.H_q + (size_t)g * p.group) * p.T_new + r0;
  // slices holding a row's positions: its last visible position, L + i, decides
  auto row_slices = [&](int i) { return ceil_div(sp.virt(L + i) + 1, p.split_tokens); };
#pragma unroll 1
  for (int idx = tid; idx < R * D; idx += NT) {
    const int rr = idx / D;
    const int d = idx - rr * D;
    if (rr >= nr) break;  // rows are the outer index
    const int i = (r0 + rr) % p.T_new;
    const int ns_row = row_slices(i);
    if (s >= ns_row) continue;  // the slice is past this row's last position
    const size_t orow = row_base + rr;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < W; ++w) M = fmaxf(M, red_m[w * R + rr]);
    if (M == -INFINITY) {  // the row sees nothing here (left of its window): empty partial
      p.ws_o[(orow * p.num_splits + s) * D + d] = 0.f;
      if (d == 0) p.ws_lse[orow * p.num_splits + s] = -INFINITY;
      continue;
    }
    float lsum = 0.f, o = 0.f;
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const float f = exp2f(red_m[w * R + rr] - M);
      lsum = fmaf(red_l[w * R + rr], f, lsum);
      o = fmaf(red_acc[(w * R + rr) * LD + d], f, o);
    }
    if (ns_row == 1) {
      store_elt<T>(out + orow * D + d, o / lsum);
    } else {
      p.ws_o[(orow * p.num_splits + s) * D + d] = o / lsum;
      if (d == 0) p.ws_lse[orow * p.num_splits + s] = M + log2f(lsum);
    }
  }
  if (ns_blk == 1) return;  // every row was finished in place

  // ---------------------------------------------------- cross-slice merge
  __threadfence();  // release this CTA's partials before taking a ticket
  named_barrier_sync(1, NT);
  int* ticket = p.counters + ((size_t)b * p.H_kv + g) * p.row_blocks + rb;
  if (tid == 0) *flag = (atomicAdd(ticket, 1) == ns_blk - 1);
  named_barrier_sync(1, NT);
  if (!*flag) return;
  __threadfence();  // acquire the other CTAs' partials

  // weights of every (row, slice): lse values first, all loads in flight together
  const int nsl = ns_blk;
#pragma unroll 1
  for (int idx = tid; idx < R * nsl; idx += NT) {
    const int rr = idx / nsl;
    const int k = idx - rr * nsl;
    float v = -INFINITY;
    if (rr < nr) {
      const int i = (r0 + rr) % p.T_new;
      if (k < row_slices(i)) v = __ldcg(p.ws_lse + (row_base + rr) * p.num_splits + k);
    }
    scratch[idx] = v;
  }
  named_barrier_sync(1, NT);
  if (tid < R) {
    float* w = scratch + tid * nsl;
    float M = -INFINITY;
    for (int k = 0; k < nsl; ++k) M = fmaxf(M, w[k]);
    float den = 0.f;
    for (int k = 0; k < nsl; ++k) {
      const float e = (w[k] == -INFINITY) ? 0.f : exp2f(w[k] - M);
      w[k] = e;
      den += e;
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    for (int k = 0; k < nsl; ++k) w[k] *= inv;
  }
  named_barrier_sync(1, NT);
#pragma unroll 1
  for (int idx = tid; idx < R * D; idx += NT) {
    const int rr = idx / D;
    const int d = idx - rr * D;
    if (rr >= nr) break;
    const int i = (r0 + rr) % p.T_new;
    const int ns_row = row_slices(i);
    if (ns_row <= 1) continue;
    const float* po = p.ws_o + (row_base + rr) * p.num_splits * D + d;
    const float* w = scratch + rr * nsl;
    float o = 0.f;
    int k = 0;
#pragma unroll 1
    for (; k + 8 <= ns_row; k += 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldcg(po + (size_t)(k + u) * D);
#pragma unroll
      for (int u = 0; u < 8; ++u) o = fmaf(w[k + u], v[u], o);
    }
    for (; k < ns_row; ++k) o = fmaf(w[k], __ldcg(po + (size_t)k * D), o);
    store_elt<T>(out + (row_base + rr) * D + d, o);
  }
  if (tid == 0) *ticket = 0;  // ready for the next launch
}

}  // namespace kvc
