// attend_mma.cuh -- N2 (tensor-core variant): split-K attention for GQA groups and
// speculative-verify chunks, on warp-level mma.sync.
//
// Same contract as attend_decode.cuh: for every query row (query head h of KV
// head g, new row i) of request b, exact-softmax attention over positions
// 0 .. L_b + i ("项目 9-16" projects 11/15; causal within the new chunk).
//
// Per KV head the work is a small dense contraction: the block's query rows
// (R = 8*NT of them, GQA group x new rows) against every K/V row.  On CUDA
// cores it costs ~70-100 instructions per K/V row (measured), which keeps a
// CUDA-core kernel issue-bound well below the HBM roofline; mma.m16n8k16 does
// the same work in about four warp instructions per K/V row.  The operands are
// swapped so that the K/V tokens are the M dimension and the query rows the N
// dimension (padding only to 8 rows):
//     S^T[16 tok x 8 rows] = K[16 x D] . Q^T[D x 8]          (bf16/fp16 in, fp32 out)
//     O^T[D x 8 rows]     += V^T[D x 16 tok] . P^T[16 x 8]
// The score fragment becomes the P^T operand through one movmatrix transpose
// per 8x8 block.  Softmax (max, exp2, sums, rescaling) stays in fp32 registers.
//
// Data path: lane 0 of warp 0 loads each 64-token K and V tile with 2-D TMA
// tensor-map copies (no multicast) into a 3-stage shared-memory ring, 128-byte
// swizzled so that ldmatrix reads are bank-conflict free; full/empty
// mbarriers with bounded waits.  Tokens past the request's last page are
// loaded from outside the tensor (zero fill), so every tile is finite.
// Each of the four warps owns 16 tokens of every tile.
#pragma once

#include <cuda.h>
#include <math.h>

#include "device_common.cuh"
#include "params.cuh"
#include "splitk_epilogue.cuh"

#ifndef KVC_MMA_STAGES_D128
#define KVC_MMA_STAGES_D128 3
#endif
#ifndef KVC_MMA_STAGES_D64
#define KVC_MMA_STAGES_D64 5
#endif

namespace kvc {

template <int D>
struct MmaCfg {
  static constexpr int kWarps = 4;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kTile = 64;                  // tokens per stage, 16 per warp
  static constexpr int kHalves = D / 64;            // 128-byte TMA boxes across a row
  static constexpr int kBoxBytes = kTile * 128;     // one box column of a tile
  static constexpr int kTileBytes = kTile * D * 2;  // K (or V) bytes per stage
  static constexpr int kStages = D == 128 ? KVC_MMA_STAGES_D128 : KVC_MMA_STAGES_D64;
  static constexpr int kKSteps = D / 16;            // k-steps of q.k
  static constexpr int kMTiles = D / 16;            // m-tiles of p.v
  static constexpr int kRing = 2 * kStages * kTileBytes;

  template <int NT>
  static constexpr size_t smem_bytes() {
    return 1024                                          // alignment slack for the swizzle
           + kRing                                       // K and V rings (reused to merge)
           + kWarps * NT * 8 * 2 * sizeof(float)         // warp m and l
           + 2 * kStages * sizeof(uint64_t) + 16;        // barriers, flags
  }
  // merge scratch available after the loop, in floats
  template <int NT>
  static constexpr int scratch_floats() {
    return (kRing - kWarps * NT * 8 * D * (int)sizeof(float)) / (int)sizeof(float);
  }
};

// byte offset of 16-byte chunk `chunk` (of D/8) of tile row `row` in a swizzled tile
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  const int h = chunk >> 3;
  const int j = chunk & 7;
  return h * MmaCfg<D>::kBoxBytes + row * 128 + ((j ^ (row & 7)) << 4);
}

template <int D, int NT, typename T, bool PAGED>
__global__ void __launch_bounds__(MmaCfg<D>::kThreads)
    attend_mma_kernel(const AttendParams p, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv) {
  using C = MmaCfg<D>;
  constexpr int W = C::kWarps;
  constexpr int NTH = C::kThreads;
  constexpr int R = NT * 8;  // query rows per CTA (padded)
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sk = smem;
  unsigned char* sv = smem + C::kStages * C::kTileBytes;
  float* red_m = reinterpret_cast<float*>(smem + C::kRing);
  float* red_l = red_m + W * R;
  uint64_t* full = reinterpret_cast<uint64_t*>(red_l + W * R);
  uint64_t* empty = full + C::kStages;
  int* flags = reinterpret_cast<int*>(empty + C::kStages);  // [0] abort, [1] last
  float* red_acc = reinterpret_cast<float*>(smem);         // ring, after the loop

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
  for (int rr = 0; rr < nr; ++rr) {
    const int i = (r0 + rr) % p.T_new;
    i_max = max(i_max, i);
    i_min = min(i_min, i);
  }
  const int n_blk = L + i_max + 1;
  const int vis_min = L + i_min + 1;
  const Span sp = block_span(vis_min, n_blk, p.window, p.sink, C::kTile);
  const int t_begin = s * p.split_tokens;  // virtual positions (window.cuh)
  if (t_begin >= sp.n_virt) return;
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
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
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
  const bool producer = (threadIdx.x == 0);
  // K/V read once: evict first; read by several row blocks: keep them in L2
  const uint64_t pol = p.row_blocks > 1 ? l2_policy_evict_normal() : l2_policy_evict_first();
  auto issue = [&](int j) {
    const int st = j % C::kStages;
    const int t0v = t_begin + j * C::kTile;
    const int t0 = sp.real(t0v);
    const int t_end = t0 + (t_stop - t0v);  // real end of the slice within this tile's run
    unsigned char* dk = sk + st * C::kTileBytes;
    unsigned char* dv = sv + st * C::kTileBytes;
    mbar_arrive_expect_tx(&full[st], 2 * C::kTileBytes);  // every box is full (zero fill)
    if (!PAGED) {
      const int y = (b * p.H_kv + g) * p.max_T + t0;
#pragma unroll
      for (int h = 0; h < C::kHalves; ++h) {
        tma_load_2d(dk + h * C::kBoxBytes, &tmk, h * 64, y, &full[st], pol);
        tma_load_2d(dv + h * C::kBoxBytes, &tmv, h * 64, y, &full[st], pol);
      }
    } else {
      const int P = 1 << p.page_shift;
      const int box_rows = P < C::kTile ? P : C::kTile;
      const int32_t* bt = p.block_table + (size_t)b * p.max_pages;
      const int beyond = p.num_pages * p.H_kv * P;  // first row past the pool: zero fill
#pragma unroll 1
      for (int t = t0; t < t0 + C::kTile; t += box_rows) {
        int y = beyond;
        if (t < t_end) {
          const int page = bt[t >> p.page_shift];
          if (page >= 0 && page < p.num_pages)
            y = (page * p.H_kv + g) * P + (t & (P - 1));
          else
            flag_error(p.err, KVC_ERR_BOUNDS);
        }
        const int off = (t - t0) * 128;
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h) {
          tma_load_2d(dk + h * C::kBoxBytes + off, &tmk, h * 64, y, &full[st], pol);
          tma_load_2d(dv + h * C::kBoxBytes + off, &tmv, h * 64, y, &full[st], pol);
        }
      }
    }
  };
  int issued = 0;
  if (producer)
    for (; issued < min(C::kStages, ntiles); ++issued) issue(issued);

  // ------------------------------------------------------------- consumers
  // Q^T fragments (B operand of q.k): row n = nt*8 + lane/4, d = kk*16 + 2(lane%4) (+8)
  uint32_t qb[C::kKSteps][NT][2];
  {
    const char* qblk =
        static_cast<const char*>(p.q) + ((((size_t)b * p.H_q + (size_t)g * p.group) * p.T_new) +
                                         r0) * D * 2;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int row = nt * 8 + (lane >> 2);
#pragma unroll
      for (int kk = 0; kk < C::kKSteps; ++kk) {
        if (row < nr) {
          const char* src = qblk + (size_t)row * D * 2 + (kk * 16 + (lane & 3) * 2) * 2;
          qb[kk][nt][0] = __ldg(reinterpret_cast<const unsigned int*>(src));
          qb[kk][nt][1] = __ldg(reinterpret_cast<const unsigned int*>(src + 16));
        } else {
          qb[kk][nt][0] = 0u;
          qb[kk][nt][1] = 0u;
        }
      }
    }
  }
  // this thread's score columns: rows nt*8 + 2(lane%4) + c
  int vis[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int rr = nt * 8 + (lane & 3) * 2 + c;
      vis[nt][c] = rr < nr ? L + (r0 + rr) % p.T_new + 1 : 0;
    }

  float m[NT][2], l[NT][2];
  float o[C::kMTiles][NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m[nt][0] = m[nt][1] = -INFINITY;
    l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < C::kMTiles; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[mt][nt][e] = 0.f;
  }

  // ldmatrix row addresses (before the stage offset): K non-transposed, V transposed
  const int mi = lane >> 3;
  const int wrow = warp * 16;
  const int k_row = wrow + (mi & 1) * 8 + (lane & 7);  // token row of this lane's matrix
  const int k_cs = mi >> 1;                             // chunk offset within a k-step
  const int v_row = wrow + (mi >> 1) * 8 + (lane & 7);
  const int v_cs = mi & 1;
  const uint32_t sk_addr = smem_addr(sk);
  const uint32_t sv_addr = smem_addr(sv);

  bool ok = true;
  int consumed = 0;
#pragma unroll 1
  for (int j = 0; j < ntiles; ++j) {
    const int st = j % C::kStages;
    if (producer && j >= 1 && issued < ntiles) {
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
    const uint32_t kb = sk_addr + st * C::kTileBytes;
    const uint32_t vb = sv_addr + st * C::kTileBytes;
    const int t0 = sp.real(t_begin + j * C::kTile);

    // S^T = K . Q^T for this warp's 16 tokens
    float sacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < C::kKSteps; ++kk) {
      uint32_t a[4];
      ldmatrix_x4(a, kb + swz<D>(k_row, 2 * kk + k_cs));
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_16816<T>(sacc[nt], a, qb[kk][nt][0], qb[kk][nt][1]);
    }

    // scale to base-2 units, mask, online softmax per score column (query row)
    const int tok0 = t0 + wrow + (lane >> 2);
    const bool unmasked = tile_fully_visible(t0, C::kTile, vis_min, n_blk, p.window, p.sink);
    bool grew = false;
    float alpha[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float s0 = sacc[nt][c] * p.scale_log2;
        float s1 = sacc[nt][2 + c] * p.scale_log2;
        if (!unmasked) {
          s0 = visible(tok0, vis[nt][c], p.window, p.sink) ? s0 : -INFINITY;
          s1 = visible(tok0 + 8, vis[nt][c], p.window, p.sink) ? s1 : -INFINITY;
        }
        float mx = fmaxf(s0, s1);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m[nt][c], mx);
        const float mu = (m_new == -INFINITY) ? 0.f : m_new;
        alpha[nt][c] = exp2f(m[nt][c] - mu);
        grew |= (m_new > m[nt][c]);
        m[nt][c] = m_new;
        const float p0 = exp2f(s0 - mu);
        const float p1 = exp2f(s1 - mu);
        l[nt][c] = fmaf(l[nt][c], alpha[nt][c], p0 + p1);
        sacc[nt][c] = p0;
        sacc[nt][2 + c] = p1;
      }
    }
    if (__any_sync(0xffffffffu, grew)) {
#pragma unroll
      for (int mt = 0; mt < C::kMTiles; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          o[mt][nt][0] *= alpha[nt][0];
          o[mt][nt][1] *= alpha[nt][1];
          o[mt][nt][2] *= alpha[nt][0];
          o[mt][nt][3] *= alpha[nt][1];
        }
    }
    // P^T fragments: transpose each 8x8 (token x row) block into (row x token)
    uint32_t pb[NT][2], pl[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint32_t h0 = Elt<T>::pack2(sacc[nt][0], sacc[nt][1]);
      const uint32_t h1 = Elt<T>::pack2(sacc[nt][2], sacc[nt][3]);
      pb[nt][0] = movmatrix_trans(h0);
      pb[nt][1] = movmatrix_trans(h1);
      if constexpr (SplitP<T>::kOn) {  // bf16: the weights' rounding remainders
        pl[nt][0] = movmatrix_trans(bf16_remainder2(sacc[nt][0], sacc[nt][1], h0));
        pl[nt][1] = movmatrix_trans(bf16_remainder2(sacc[nt][2], sacc[nt][3], h1));
      }
    }
    // O^T += V^T . P^T
#pragma unroll
    for (int mt = 0; mt < C::kMTiles; ++mt) {
      uint32_t a[4];
      ldmatrix_x4_trans(a, vb + swz<D>(v_row, 2 * mt + v_cs));
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        mma_16816<T>(o[mt][nt], a, pb[nt][0], pb[nt][1]);
        if constexpr (SplitP<T>::kOn) mma_16816<T>(o[mt][nt], a, pl[nt][0], pl[nt][1]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }
  if (!ok) {
    atomicOr(&flags[0], 1);
    if (producer)
#pragma unroll 1
      for (int j = consumed; j < issued; ++j)
        if (!mbar_wait(&full[j % C::kStages], (j / C::kStages) & 1, p.err)) break;
  }

  // row sums over the lanes that hold the other tokens of each column
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      l[nt][c] += __shfl_xor_sync(0xffffffffu, l[nt][c], 4);
      l[nt][c] += __shfl_xor_sync(0xffffffffu, l[nt][c], 8);
      l[nt][c] += __shfl_xor_sync(0xffffffffu, l[nt][c], 16);
    }
  named_barrier_sync(1, NTH);  // the ring is free
  if (flags[0]) return;
#pragma unroll
  for (int mt = 0; mt < C::kMTiles; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = nt * 8 + (lane & 3) * 2 + (e & 1);
        const int d = mt * 16 + (lane >> 2) + (e >> 1) * 8;
        red_acc[(warp * R + row) * D + d] = o[mt][nt][e];
      }
  if (lane < 4) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int row = nt * 8 + lane * 2 + c;
        red_m[warp * R + row] = m[nt][c];
        red_l[warp * R + row] = l[nt][c];
      }
  }
  named_barrier_sync(1, NTH);
  finish_slice<T, D, R, W, NTH>(p, red_acc, red_m, red_l, red_acc + W * R * D, &flags[1], b, g,
                                rb, s, r0, nr, L, ns_blk, sp);
}

}  // namespace kvc
