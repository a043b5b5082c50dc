// attend_decode.cuh -- N2 + N3 (CUDA-core variant): split-K decode attention with a
// fused log-sum-exp combine.
//
// For every query row r = (query head h of KV head g, new row i) of request b
// the kernel computes exact-softmax attention over positions 0 .. L_b + i
// ("项目 9-16" projects 11 and 15: scores q.K^T * scale, softmax, times V;
// "9. 推理" 9.7: a tiled evaluation is the same attention up to rounding).
//
// Decomposition (flash-decoding): one CTA per (KV-length slice s, KV head g,
// block of <= R query rows, request b).  Lane 0 of warp 0 streams the slice's
// K and V tiles once through a 3-stage shared-memory ring with 1-D bulk async
// copies (full/empty mbarriers, bounded waits); the four warps each take a
// quarter of every tile.  Each K/V row read serves all R rows of the GQA
// group, which is the point of grouping: K/V bytes are read once per KV head.
//
// Lane layout: a K/V row of D elements is split over D/16 lanes, 16 elements
// (two 16-byte vectors) per lane; a warp covers 512/D rows per pass.  The two
// vectors of a lane are loaded in a per-lane order chosen so that every
// quarter-warp's 16-byte shared loads hit 8 distinct bank groups.  q.k and p.v
// use packed fp32x2 FMAs; q.k partial sums are reduced over the row's lanes
// with xor shuffles.  Scores stay in registers in base-2 units (q is
// pre-scaled by scale*log2 e); the running max m, sum l and weighted V sum are
// per lane (online softmax) and rescaled only when m grows.
//
// Slice results: a row whose visible range fits in one slice is finished in
// place.  Otherwise each CTA writes its normalised partial output o_s and
// lse_s = m_s + log2 l_s; the last CTA of the (request, KV head, row block) to
// finish -- decided by an atomic ticket after a release fence, no waiting --
// merges them: out = sum_s 2^(lse_s - M) o_s / sum_s 2^(lse_s - M).
//
// CUDA cores, not tensor cores: with R <= 4 rows per K/V element this is ~R
// flop per K/V byte, far below the tensor ridge; the kernel is HBM-bound once
// its instruction count per K/V row is low enough.  It serves the caches the
// tensor-core kernels have no TMA tensor maps for: D = 32, pages of fewer than
// 8 tokens.
#pragma once

#include <math.h>

#include "device_common.cuh"
#include "params.cuh"
#include "splitk_epilogue.cuh"

#ifndef KVC_DECODE_TILE_BYTES
#define KVC_DECODE_TILE_BYTES 16384
#endif
#ifndef KVC_DECODE_STAGES
#define KVC_DECODE_STAGES 3
#endif

namespace kvc {

template <int D>
struct DecodeCfg {
  static constexpr int kEpl = 16;                     // elements per lane
  static constexpr int kLpt = D / kEpl;               // lanes per K/V row: 2, 4, 8
  static constexpr int kTpp = 32 / kLpt;              // rows per warp pass: 16, 8, 4
  static constexpr int kWarps = 4;                    // warps per CTA
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kTileBytes = KVC_DECODE_TILE_BYTES;  // K bytes per stage (V the same)
  static constexpr int kTile = kTileBytes / (2 * D);  // tokens per stage: 256, 128, 64
  static constexpr int kStages = KVC_DECODE_STAGES;
  static constexpr int kWarpTokens = kTile / kWarps;
  static constexpr int kPasses = kWarpTokens / kTpp;  // 4
  static_assert(kPasses * kTpp * kWarps == kTile, "tile split");

  // Quarter-warp bank spreading: which bit of the lane's row-in-pass index
  // swaps the load order of its two vectors (none when a quarter-warp reads
  // one 256-byte row).
  static constexpr int kSwapShift = (D == 64) ? 0 : (D == 32) ? 1 : -1;

  template <int R>
  static constexpr size_t smem_bytes() {
    return 2 * kStages * kTileBytes                   // K and V rings (reused for merging)
           + kWarps * R * 2 * sizeof(float)           // warp m and l
           + 2 * kStages * sizeof(uint64_t) + 16;     // barriers, flags
  }
};

// Packed fp32 pair helpers (fma.rn.f32x2 / mul.rn.f32x2 on sm_100).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  return __ffma2_rn(a, b, c);
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

template <typename T>
__device__ __forceinline__ void unpack_pairs(const uint4& u, float2* f);

template <>
__device__ __forceinline__ void unpack_pairs<__nv_bfloat16>(const uint4& u, float2* f) {
  f[0] = make_float2(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u));
  f[1] = make_float2(__uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
  f[2] = make_float2(__uint_as_float(u.z << 16), __uint_as_float(u.z & 0xffff0000u));
  f[3] = make_float2(__uint_as_float(u.w << 16), __uint_as_float(u.w & 0xffff0000u));
}

template <>
__device__ __forceinline__ void unpack_pairs<__half>(const uint4& u, float2* f) {
  const __half2* h = reinterpret_cast<const __half2*>(&u);
  f[0] = __half22float2(h[0]);
  f[1] = __half22float2(h[1]);
  f[2] = __half22float2(h[2]);
  f[3] = __half22float2(h[3]);
}

// Four warps and no dedicated producer warp: with ~200 registers per thread,
// two such CTAs fill an SM (the register file is split across the four SM
// sub-partitions, 16K registers each, two warps apiece).
template <int D, int R, typename T, bool PAGED>
__global__ void __launch_bounds__(DecodeCfg<D>::kThreads, 2)
    attend_decode_kernel(const AttendParams p) {
  using C = DecodeCfg<D>;
  constexpr int W = C::kWarps;
  constexpr int NT = W * 32;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* sk = smem;
  unsigned char* sv = smem + C::kStages * C::kTileBytes;
  float* red_m = reinterpret_cast<float*>(smem + 2 * C::kStages * C::kTileBytes);
  float* red_l = red_m + W * R;
  uint64_t* full = reinterpret_cast<uint64_t*>(red_l + W * R);
  uint64_t* empty = full + C::kStages;
  int* flags = reinterpret_cast<int*>(empty + C::kStages);  // [0] abort, [1] last
  // after the tile loop the ring is free: warp partials, then merge weights
  float* red_acc = reinterpret_cast<float*>(smem);

  // Row blocks vary fastest: the CTAs that read the same K/V slice for
  // different query rows launch together, so L2 serves all but the first read.
  const int s = blockIdx.x / p.row_blocks;
  const int rb = blockIdx.x - s * p.row_blocks;
  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int L = p.seq_lens[b];
  const int r0 = rb * R;
  const int nr = min(R, p.rows - r0);

  int i_max = 0, i_min = 1 << 30;
#pragma unroll
  for (int rr = 0; rr < R; ++rr)
    if (rr < nr) {
      const int i = (r0 + rr) % p.T_new;
      i_max = max(i_max, i);
      i_min = min(i_min, i);
    }
  const int n_blk = L + i_max + 1;  // positions the block must read
  const int vis_min = L + i_min + 1;
  const Span sp = block_span(vis_min, n_blk, p.window, p.sink, C::kTile);
  const int t_begin = s * p.split_tokens;  // virtual positions (window.cuh)
  if (t_begin >= sp.n_virt) return;  // the slice is past every row's horizon
  if (L < 0 || L + p.T_new > p.max_T ||
      (PAGED && ((L + p.T_new - 1) >> p.page_shift) >= p.max_pages)) {
    if (threadIdx.x == 0) flag_error(p.err, KVC_ERR_BOUNDS);
    return;
  }
  const int t_stop = min(t_begin + p.split_tokens, sp.n_virt);
  const int ntiles = ceil_div(t_stop - t_begin, C::kTile);
  const int ns_blk = ceil_div(sp.n_virt, p.split_tokens);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
#pragma unroll
    for (int st = 0; st < C::kStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], W);
    }
    flags[0] = 0;
    flags[1] = 0;
    fence_barrier_init();
  }
  __syncthreads();

  // ------------------------------------------------------- tile producer
  // Lane 0 of warp 0 issues the bulk copies: the first kStages tiles up front,
  // then tile j + kStages - 1 at the top of iteration j, into the stage that
  // every warp released after tile j - 1.
  const uint64_t pol = l2_policy_evict_first();
  auto issue = [&](int j) {
    const int st = j % C::kStages;
    const int t0v = t_begin + j * C::kTile;
    const int t0 = sp.real(t0v);
    const int t1 = t0 + min(C::kTile, t_stop - t0v);
    unsigned char* dk = sk + st * C::kTileBytes;
    unsigned char* dv = sv + st * C::kTileBytes;
    const char* kp = static_cast<const char*>(p.k_pool);
    const char* vp = static_cast<const char*>(p.v_pool);
    constexpr uint32_t row_bytes = D * 2;
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
  };
  const bool producer = (threadIdx.x == 0);
  int issued = 0;
  if (producer) {
    for (; issued < min(C::kStages, ntiles); ++issued) issue(issued);
  }

  // ----------------------------------------------------------- consumers
  const int c = lane % C::kLpt;  // this lane's vector pair within a row
  const int sub = lane / C::kLpt;
  int swap = 0;
  if constexpr (C::kSwapShift >= 0) swap = (sub >> C::kSwapShift) & 1;
  const int va = swap ? c + C::kLpt : c;  // first-loaded vector index (16-byte units)
  const int vb = swap ? c : c + C::kLpt;

  float2 q2[R][8];
#pragma unroll
  for (int rr = 0; rr < R; ++rr) {
    if (rr < nr) {
      const int r = r0 + rr;
      const int hl = r / p.T_new;
      const int i = r - hl * p.T_new;
      const int h = g * p.group + hl;
      const char* qrow =
          static_cast<const char*>(p.q) + (((size_t)b * p.H_q + h) * p.T_new + i) * D * 2;
      unpack_pairs<T>(ld_global_nc_v4(qrow + va * 16), &q2[rr][0]);
      unpack_pairs<T>(ld_global_nc_v4(qrow + vb * 16), &q2[rr][4]);
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
#pragma unroll
      for (int k = 0; k < 8; ++k) q2[rr][k] = fmul2(q2[rr][k], sc2);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) q2[rr][k] = make_float2(0.f, 0.f);
    }
  }
  int vis[R];
#pragma unroll
  for (int rr = 0; rr < R; ++rr) vis[rr] = (rr < nr) ? L + (r0 + rr) % p.T_new + 1 : 0;

  float m[R], l[R];
  float2 acc[R][8];
#pragma unroll
  for (int rr = 0; rr < R; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[rr][k] = make_float2(0.f, 0.f);
  }

  bool ok = true;
  int consumed = 0;
#pragma unroll 1
  for (int j = 0; j < ntiles; ++j) {
    const int st = j % C::kStages;
    if (producer && j >= 1 && issued < ntiles) {
      // refill the stage tile j - 1 used, once every warp has released it
      if (mbar_wait(&empty[(j - 1) % C::kStages], ((j - 1) / C::kStages) & 1, p.err)) {
        issue(issued);
        ++issued;
      } else {
        ok = false;
      }
    }
    if (!ok || !mbar_wait(&full[st], (j / C::kStages) & 1, p.err)) {
      ok = false;
      break;
    }
    consumed = j + 1;
    const unsigned char* tk = sk + st * C::kTileBytes;
    const unsigned char* tv = sv + st * C::kTileBytes;
    const int t0v = t_begin + j * C::kTile;
    const int t0 = sp.real(t0v);
    const int valid = min(C::kTile, t_stop - t0v);
    const bool unmasked =  // every row sees the whole tile
        tile_fully_visible(t0, C::kTile, vis_min, n_blk, p.window, p.sink);

    float sc[C::kPasses][R];
#pragma unroll
    for (int pp = 0; pp < C::kPasses; ++pp) {
      const int tok = warp * C::kWarpTokens + pp * C::kTpp + sub;
      const unsigned char* row = tk + tok * (D * 2);
      float2 kf[8];
      unpack_pairs<T>(ld_shared_v4(row + va * 16), &kf[0]);
      unpack_pairs<T>(ld_shared_v4(row + vb * 16), &kf[4]);
      float part[R];
#pragma unroll
      for (int rr = 0; rr < R; ++rr) {
        float2 a = fmul2(q2[rr][0], kf[0]);
#pragma unroll
        for (int k = 1; k < 8; ++k) a = ffma2(q2[rr][k], kf[k], a);
        part[rr] = a.x + a.y;
      }
#pragma unroll
      for (int off = C::kLpt / 2; off > 0; off >>= 1)
#pragma unroll
        for (int rr = 0; rr < R; ++rr) part[rr] += __shfl_xor_sync(0xffffffffu, part[rr], off);
      if (unmasked) {
#pragma unroll
        for (int rr = 0; rr < R; ++rr) sc[pp][rr] = part[rr];
      } else {
        const int pos = t0 + tok;
#pragma unroll
        for (int rr = 0; rr < R; ++rr)
          sc[pp][rr] = visible(pos, vis[rr], p.window, p.sink) ? part[rr] : -INFINITY;
      }
    }

    // online softmax: the warp's running max per row, rescale only if it grew
#pragma unroll
    for (int rr = 0; rr < R; ++rr) {
      float mx = sc[0][rr];
#pragma unroll
      for (int pp = 1; pp < C::kPasses; ++pp) mx = fmaxf(mx, sc[pp][rr]);
#pragma unroll
      for (int off = C::kLpt; off < 32; off <<= 1)
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      if (mx > m[rr]) {  // warp-uniform
        const float alpha = exp2f(m[rr] - mx);
        m[rr] = mx;
        l[rr] *= alpha;
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[rr][k] = fmul2(acc[rr][k], a2);
      }
      const float mu = (m[rr] == -INFINITY) ? 0.f : m[rr];
#pragma unroll
      for (int pp = 0; pp < C::kPasses; ++pp) {
        sc[pp][rr] = exp2f(sc[pp][rr] - mu);
        l[rr] += sc[pp][rr];
      }
    }

    // weighted V sum
#pragma unroll
    for (int pp = 0; pp < C::kPasses; ++pp) {
      const int tok = warp * C::kWarpTokens + pp * C::kTpp + sub;
      if (valid == C::kTile || tok < valid) {
        const unsigned char* row = tv + tok * (D * 2);
        float2 vf[8];
        unpack_pairs<T>(ld_shared_v4(row + va * 16), &vf[0]);
        unpack_pairs<T>(ld_shared_v4(row + vb * 16), &vf[4]);
#pragma unroll
        for (int rr = 0; rr < R; ++rr) {
          const float2 p2 = make_float2(sc[pp][rr], sc[pp][rr]);
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[rr][k] = ffma2(p2, vf[k], acc[rr][k]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }
  if (!ok) {
    atomicOr(&flags[0], 1);
    // Do not retire while copies issued here may still be landing in the ring.
    if (producer)
#pragma unroll 1
      for (int j = consumed; j < issued; ++j)
        if (!mbar_wait(&full[j % C::kStages], (j / C::kStages) & 1, p.err)) break;
  }

  // Back to one register order for every lane (vector c first, then c + kLpt)
  // before lanes of different row groups are added together.
  if (swap) {
#pragma unroll
    for (int rr = 0; rr < R; ++rr)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 t = acc[rr][k];
        acc[rr][k] = acc[rr][k + 4];
        acc[rr][k + 4] = t;
      }
  }
  // merge the warp's row groups (lanes owning the same vectors of different rows)
#pragma unroll
  for (int off = C::kLpt; off < 32; off <<= 1) {
#pragma unroll
    for (int rr = 0; rr < R; ++rr) {
      l[rr] += __shfl_xor_sync(0xffffffffu, l[rr], off);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        acc[rr][k].x += __shfl_xor_sync(0xffffffffu, acc[rr][k].x, off);
        acc[rr][k].y += __shfl_xor_sync(0xffffffffu, acc[rr][k].y, off);
      }
    }
  }
  named_barrier_sync(1, NT);  // every warp is done with the stage buffers
  if (flags[0]) return;      // a wait gave up: copies may still land in the ring
  if (sub == 0) {  // row group 0 never swaps: vector c, then vector c + kLpt
#pragma unroll
    for (int rr = 0; rr < R; ++rr) {
      float* dst = red_acc + (warp * R + rr) * D;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        reinterpret_cast<float2*>(dst + c * 8)[k] = acc[rr][k];
        reinterpret_cast<float2*>(dst + (c + C::kLpt) * 8)[k] = acc[rr][4 + k];
      }
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int rr = 0; rr < R; ++rr) {
      red_m[warp * R + rr] = m[rr];
      red_l[warp * R + rr] = l[rr];
    }
  }
  named_barrier_sync(1, NT);

  finish_slice<T, D, R, W, NT>(p, red_acc, red_m, red_l, red_acc + W * R * D, &flags[1], b, g,
                               rb, s, r0, nr, L, ns_blk, sp);
}

}  // namespace kvc
