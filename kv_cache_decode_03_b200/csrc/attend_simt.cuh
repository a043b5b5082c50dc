// attend_simt.cuh -- N2 (CUDA-core variant): split-K decode attention.
//
// Computes, for every query row r = (query head h of KV head g, new row i) of
// request b, exact-softmax attention over positions 0 .. L_b + i ("项目 9-16"
// projects 11 and 15: scores q.K^T * scale, softmax, times V; "9. 推理" 9.7:
// the tiled form is the same attention up to rounding).
//
// Decomposition (flash-decoding): one CTA per (KV-length slice s, KV head g,
// block of <= R query rows, request b).  The CTA streams its slice of K and V
// once through a 4-stage shared-memory ring filled by 1-D bulk async copies
// (a dedicated producer warp; full/empty mbarriers), and every K/V row it
// loads serves all R query rows of the GQA group.  The slice's result is
// written as a normalised partial output plus its base-2 log-sum-exp; a
// request whose rows fit in one slice gets its final output directly.
//
// Inside a consumer warp each lane owns one 16-byte vector (8 elements) of a
// K/V row: D/8 lanes cover a row and the warp covers 256/D rows per pass.
// q.k partial sums are reduced over the row's lanes with xor shuffles; the
// running max m, running sum l and the weighted V sum are kept per lane in
// fp32 (online softmax), so no score ever leaves registers.  Warps and then
// slices are merged with the log-sum-exp rule.
//
// CUDA cores are the right unit here: with R <= 4 rows per K/V element the
// work is ~R flop per byte of K/V, far below the tensor-core ridge, and the
// kernel is bound by HBM bandwidth.
#pragma once

#include <math.h>

#include "device_common.cuh"
#include "params.cuh"

namespace kvc {

template <int D>
struct SimtCfg {
  static constexpr int kVec = 8;                      // elements per 16-byte vector
  static constexpr int kLpt = D / kVec;               // lanes per K/V row
  static constexpr int kTpp = 32 / kLpt;              // rows per warp pass
  static constexpr int kConsumerWarps = 4;
  static constexpr int kThreads = (kConsumerWarps + 1) * 32;
  static constexpr int kTileBytes = 8192;             // K bytes per stage (V the same)
  static constexpr int kTile = kTileBytes / (D * 2);  // tokens per stage
  static constexpr int kStages = 4;
  static constexpr int kWarpTokens = kTile / kConsumerWarps;
  static constexpr int kPasses = kWarpTokens / kTpp;
  static_assert(kPasses * kTpp * kConsumerWarps == kTile, "tile split");

  template <int R>
  static constexpr size_t smem_bytes() {
    return 2 * kStages * kTileBytes                          // K and V rings
           + kConsumerWarps * R * D * sizeof(float)          // warp partial outputs
           + kConsumerWarps * R * 2 * sizeof(float)          // warp m and l
           + 2 * kStages * sizeof(uint64_t) + 16;            // barriers + abort flag
  }
};

template <int D, int R, typename T, bool PAGED>
__global__ void __launch_bounds__(SimtCfg<D>::kThreads)
    attend_simt_kernel(const AttendParams p) {
  using C = SimtCfg<D>;
  constexpr int W = C::kConsumerWarps;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* sk = smem;
  unsigned char* sv = smem + C::kStages * C::kTileBytes;
  float* red_acc = reinterpret_cast<float*>(smem + 2 * C::kStages * C::kTileBytes);
  float* red_m = red_acc + W * R * D;
  float* red_l = red_m + W * R;
  uint64_t* full = reinterpret_cast<uint64_t*>(red_l + W * R);
  uint64_t* empty = full + C::kStages;
  int* abort_flag = reinterpret_cast<int*>(empty + C::kStages);

  const int s = blockIdx.x;
  const int g = blockIdx.y / p.row_blocks;
  const int rb = blockIdx.y - g * p.row_blocks;
  const int b = blockIdx.z;
  const int L = p.seq_lens[b];
  const int r0 = rb * R;
  const int nr = min(R, p.rows - r0);

  // Largest new-row index in this block decides how far the block must read.
  int i_max = 0;
#pragma unroll
  for (int rr = 0; rr < R; ++rr)
    if (rr < nr) i_max = max(i_max, (r0 + rr) % p.T_new);
  const int n_blk = L + i_max + 1;
  const int t_begin = s * p.split_tokens;
  if (t_begin >= n_blk) return;  // slice lies wholly past every row's horizon
  if (L < 0 || L + p.T_new > p.max_T ||
      (PAGED && ((L + p.T_new - 1) >> p.page_shift) >= p.max_pages)) {
    if (threadIdx.x == 0) flag_error(p.err, KVC_ERR_BOUNDS);
    return;
  }
  const int t_stop = min(t_begin + p.split_tokens, n_blk);
  const int ntiles = ceil_div(t_stop - t_begin, C::kTile);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int st = 0; st < C::kStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], W);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  // ------------------------------------------------------------ producer
  if (warp == W) {
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      const char* kp = static_cast<const char*>(p.k_pool);
      const char* vp = static_cast<const char*>(p.v_pool);
      constexpr uint32_t row_bytes = D * 2;
      int issued = 0;
      bool ok = true;
#pragma unroll 1
      for (int j = 0; j < ntiles; ++j) {
        const int st = j % C::kStages;
        if (j >= C::kStages && !mbar_wait(&empty[st], ((j / C::kStages) - 1) & 1, p.err)) {
          ok = false;
          break;
        }
        const int t0 = t_begin + j * C::kTile;
        const int t1 = min(t0 + C::kTile, t_stop);
        unsigned char* dk = sk + st * C::kTileBytes;
        unsigned char* dv = sv + st * C::kTileBytes;
        if (!PAGED) {
          const size_t row = ((size_t)b * p.H_kv + g) * p.max_T + t0;
          const uint32_t bytes = (uint32_t)(t1 - t0) * row_bytes;
          mbar_arrive_expect_tx(&full[st], 2 * bytes);
          bulk_g2s_hint(dk, kp + row * row_bytes, bytes, &full[st], pol);
          bulk_g2s_hint(dv, vp + row * row_bytes, bytes, &full[st], pol);
        } else {
          const int P = 1 << p.page_shift;
          const int32_t* bt = p.block_table + (size_t)b * p.max_pages;
          uint32_t bytes = 0;
#pragma unroll 1
          for (int t = t0; t < t1;) {
            const int lp = t >> p.page_shift;
            const int pend = min(t1, (lp + 1) << p.page_shift);
            const int page = bt[lp];
            if (page >= 0 && page < p.num_pages) bytes += (uint32_t)(pend - t) * row_bytes;
            t = pend;
          }
          mbar_arrive_expect_tx(&full[st], 2 * bytes);
#pragma unroll 1
          for (int t = t0; t < t1;) {
            const int lp = t >> p.page_shift;
            const int pend = min(t1, (lp + 1) << p.page_shift);
            const int page = bt[lp];
            if (page >= 0 && page < p.num_pages) {
              const size_t row = ((size_t)page * p.H_kv + g) * P + (t & (P - 1));
              const uint32_t nb = (uint32_t)(pend - t) * row_bytes;
              bulk_g2s_hint(dk + (t - t0) * row_bytes, kp + row * row_bytes, nb, &full[st], pol);
              bulk_g2s_hint(dv + (t - t0) * row_bytes, vp + row * row_bytes, nb, &full[st], pol);
            } else {
              flag_error(p.err, KVC_ERR_BOUNDS);
            }
            t = pend;
          }
        }
        issued = j + 1;
      }
      // Do not retire while copies this thread issued may still be landing.
      const int first = max(0, issued - C::kStages);
#pragma unroll 1
      for (int j = first; j < issued; ++j)
        if (!mbar_wait(&full[j % C::kStages], (j / C::kStages) & 1, p.err)) break;
      (void)ok;
    }
    return;
  }

  // ----------------------------------------------------------- consumers
  const int c = lane % C::kLpt;        // this lane's 16-byte vector of a row
  const int sub = lane / C::kLpt;      // which row of the pass
  float qf[R][8];
  int vis[R];
#pragma unroll
  for (int rr = 0; rr < R; ++rr) {
    if (rr < nr) {
      const int r = r0 + rr;
      const int hl = r / p.T_new;
      const int i = r - hl * p.T_new;
      const int h = g * p.group + hl;
      const size_t off = ((((size_t)b * p.H_q + h) * p.T_new + i) * D + c * 8) * 2;
      const uint4 u = ld_global_nc_v4(static_cast<const char*>(p.q) + off);
      Elt<T>::unpack8(u, qf[rr]);
#pragma unroll
      for (int e = 0; e < 8; ++e) qf[rr][e] *= p.scale_log2;
      vis[rr] = L + i + 1;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) qf[rr][e] = 0.f;
      vis[rr] = 0;
    }
  }

  float m[R], l[R], acc[R][8];
#pragma unroll
  for (int rr = 0; rr < R; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[rr][e] = 0.f;
  }

  bool ok = true;
#pragma unroll 1
  for (int j = 0; j < ntiles; ++j) {
    const int st = j % C::kStages;
    if (!mbar_wait(&full[st], (j / C::kStages) & 1, p.err)) {
      ok = false;
      break;
    }
    const unsigned char* tk = sk + st * C::kTileBytes;
    const unsigned char* tv = sv + st * C::kTileBytes;
    const int t0 = t_begin + j * C::kTile;
    const int valid = min(C::kTile, t_stop - t0);

    float sc[C::kPasses][R];
#pragma unroll
    for (int pp = 0; pp < C::kPasses; ++pp) {
      const int tok = warp * C::kWarpTokens + pp * C::kTpp + sub;
      const uint4 u = ld_shared_v4(tk + (tok * D + c * 8) * 2);
      float kf[8];
      Elt<T>::unpack8(u, kf);
      float part[R];
#pragma unroll
      for (int rr = 0; rr < R; ++rr) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaf(qf[rr][e], kf[e], a);
        part[rr] = a;
      }
#pragma unroll
      for (int off = C::kLpt / 2; off > 0; off >>= 1)
#pragma unroll
        for (int rr = 0; rr < R; ++rr) part[rr] += __shfl_xor_sync(0xffffffffu, part[rr], off);
      const int pos = t0 + tok;
#pragma unroll
      for (int rr = 0; rr < R; ++rr) sc[pp][rr] = (pos < vis[rr]) ? part[rr] : -INFINITY;
    }

    // online softmax update, per row
#pragma unroll
    for (int rr = 0; rr < R; ++rr) {
      float mx = sc[0][rr];
#pragma unroll
      for (int pp = 1; pp < C::kPasses; ++pp) mx = fmaxf(mx, sc[pp][rr]);
#pragma unroll
      for (int off = C::kLpt; off < 32; off <<= 1)
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m[rr], mx);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = exp2f(m[rr] - m_use);
      m[rr] = m_new;
      l[rr] *= alpha;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[rr][e] *= alpha;
#pragma unroll
      for (int pp = 0; pp < C::kPasses; ++pp) {
        sc[pp][rr] = exp2f(sc[pp][rr] - m_use);
        l[rr] += sc[pp][rr];
      }
    }

    // weighted V sum
#pragma unroll
    for (int pp = 0; pp < C::kPasses; ++pp) {
      const int tok = warp * C::kWarpTokens + pp * C::kTpp + sub;
      if (tok < valid) {
        const uint4 u = ld_shared_v4(tv + (tok * D + c * 8) * 2);
        float vf[8];
        Elt<T>::unpack8(u, vf);
#pragma unroll
        for (int rr = 0; rr < R; ++rr)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[rr][e] = fmaf(sc[pp][rr], vf[e], acc[rr][e]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }
  if (!ok) atomicOr(abort_flag, 1);

  // merge the warp's row groups (lanes that own the same vector of different rows)
#pragma unroll
  for (int off = C::kLpt; off < 32; off <<= 1) {
#pragma unroll
    for (int rr = 0; rr < R; ++rr) {
      l[rr] += __shfl_xor_sync(0xffffffffu, l[rr], off);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[rr][e] += __shfl_xor_sync(0xffffffffu, acc[rr][e], off);
    }
  }
  if (sub == 0) {
#pragma unroll
    for (int rr = 0; rr < R; ++rr)
#pragma unroll
      for (int e = 0; e < 8; ++e) red_acc[(warp * R + rr) * D + c * 8 + e] = acc[rr][e];
  }
  if (lane == 0) {
#pragma unroll
    for (int rr = 0; rr < R; ++rr) {
      red_m[warp * R + rr] = m[rr];
      red_l[warp * R + rr] = l[rr];
    }
  }
  named_barrier_sync(1, W * 32);
  if (*abort_flag) return;

  // merge the warps and write the slice result
#pragma unroll 1
  for (int idx = threadIdx.x; idx < R * D; idx += W * 32) {
    const int rr = idx / D;
    const int d = idx - rr * D;
    if (rr >= nr) continue;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < W; ++w) M = fmaxf(M, red_m[w * R + rr]);
    if (M == -INFINITY) continue;  // no visible position of this row in the slice
    float lsum = 0.f, o = 0.f;
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const float f = exp2f(red_m[w * R + rr] - M);
      lsum = fmaf(red_l[w * R + rr], f, lsum);
      o = fmaf(red_acc[(w * R + rr) * D + d], f, o);
    }
    const int r = r0 + rr;
    const int hl = r / p.T_new;
    const int i = r - hl * p.T_new;
    const int h = g * p.group + hl;
    const size_t row = ((size_t)b * p.H_q + h) * p.T_new + i;
    const int ns_row = ceil_div(L + i + 1, p.split_tokens);
    if (ns_row == 1) {
      T* out = static_cast<T*>(p.out);
      const float val = o / lsum;
      if constexpr (Elt<T>::kCode == KVC_BF16) out[row * D + d] = __float2bfloat16_rn(val);
      else out[row * D + d] = __float2half_rn(val);
    } else {
      p.ws_o[(row * p.num_splits + s) * D + d] = o / lsum;
      if (d == 0) p.ws_lse[row * p.num_splits + s] = M + log2f(lsum);
    }
  }
}

}  // namespace kvc
