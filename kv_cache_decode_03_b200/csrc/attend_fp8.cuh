// attend_fp8.cuh -- N2 for the FP8 cache (fp8.cuh): split-K attention whose K/V tiles
// arrive as E4M3 codes with one fp32 scale per (token, KV head).
//
// Same contract and structure as attend_mma.cuh (tensor cores, mma.m16n8k16 with the
// K/V tokens as M and the query rows as N, fixed split-K, the shared slice epilogue,
// windows through window.cuh); what differs is the data path:
//   - thread 0 loads each 64-token tile's codes with 2-D TMA (one D-byte row per token,
//     no swizzle, no multicast) and the tile's K and V scales with 1-D bulk copies;
//   - each warp converts its own 16 tokens of codes to bf16 (exact: E4M3 has 3
//     mantissa bits) into a 128-byte-swizzled buffer, releases the stage at once, and
//     runs the bf16 MMAs from the buffer;
//   - the K scale multiplies the token's score, the V scale the token's softmax
//     weight in the p.V product (never the running sum l), so the result is attention
//     over code * scale exactly, up to fp32 rounding.
// bf16 q/out only; weights are split hi + lo like every bf16 tensor-core path.
#pragma once

#include <cuda.h>
#include <math.h>

#include "attend_mma.cuh"
#include "device_common.cuh"
#include "fp8.cuh"
#include "params.cuh"
#include "splitk_epilogue.cuh"
#include "window.cuh"

namespace kvc {

template <int D>
struct Fp8Cfg {
  static constexpr int kWarps = 4;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kTile = 64;                 // tokens per stage, 16 per warp
  static constexpr int kCodeBytes = kTile * D;     // K (or V) codes per stage
  static constexpr int kStages = 4;
  static constexpr int kRing = 2 * kStages * kCodeBytes;
  static constexpr int kScaleBytes = 2 * kTile * 4;                   // K and V scales
  static constexpr int kConvBytes = MmaCfg<D>::kTileBytes;             // one bf16 tile
  static constexpr int kData = kRing + kStages * kScaleBytes + 2 * kConvBytes;
  static constexpr int kKSteps = D / 16;
  static constexpr int kMTiles = D / 16;

  template <int NT>
  static constexpr size_t smem_bytes() {
    return 1024 + kData + kWarps * NT * 8 * 2 * sizeof(float) + 2 * kStages * sizeof(uint64_t) +
           16;
  }
  template <int NT>
  static constexpr int scratch_floats() {
    return (kData - kWarps * NT * 8 * D * (int)sizeof(float)) / (int)sizeof(float);
  }
  static_assert(kRing >= kWarps * 32 * D * 4, "the result buffer must fit the rings");
};

struct Fp8Scales {
  const float* k;  // contiguous (B, H_kv, T_pad); paged (num_pages, H_kv, P)
  const float* v;
  int T_pad;
};

template <int D, int NT, bool PAGED>
__global__ void __launch_bounds__(Fp8Cfg<D>::kThreads)
    attend_fp8_kernel(const AttendParams p, const Fp8Scales sc,
                      const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv) {
  using C = Fp8Cfg<D>;
  using T = __nv_bfloat16;
  constexpr int W = C::kWarps;
  constexpr int NTH = C::kThreads;
  constexpr int R = NT * 8;  // query rows per CTA (padded)
  constexpr int S = C::kStages;
  extern __shared__ unsigned char fp8_smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(fp8_smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ck = smem;                          // K code stages
  unsigned char* cv = smem + S * C::kCodeBytes;      // V code stages
  float* scl = reinterpret_cast<float*>(smem + C::kRing);  // [S][K 64 | V 64]
  unsigned char* bk = smem + C::kRing + S * C::kScaleBytes;  // bf16 K tile (swizzled)
  unsigned char* bv = bk + C::kConvBytes;                    // bf16 V tile
  float* red_m = reinterpret_cast<float*>(smem + C::kData);
  float* red_l = red_m + W * R;
  uint64_t* full = reinterpret_cast<uint64_t*>(red_l + W * R);
  uint64_t* empty = full + S;
  int* flags = reinterpret_cast<int*>(empty + S);  // [0] abort, [1] last
  float* red_acc = reinterpret_cast<float*>(smem);  // code rings, after the loop

  const int s = blockIdx.x / p.row_blocks;  // row blocks vary fastest (shared K/V in L2)
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
    for (int st = 0; st < S; ++st) {
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
  const uint64_t pol = p.row_blocks > 1 ? l2_policy_evict_normal() : l2_policy_evict_first();
  auto issue = [&](int j) {
    const int st = j % S;
    const int t0v = t_begin + j * C::kTile;
    const int t0 = sp.real(t0v);
    const int t_end = t0 + (t_stop - t0v);  // real end of the slice within this tile's run
    unsigned char* dk = ck + st * C::kCodeBytes;
    unsigned char* dv = cv + st * C::kCodeBytes;
    float* ds = scl + st * (2 * C::kTile);
    // every code box is full (zero fill past the tensor); every scale copy is 4 B a token
    mbar_arrive_expect_tx(&full[st], 2 * C::kCodeBytes + C::kScaleBytes);
    if (!PAGED) {
      const int y = (b * p.H_kv + g) * p.max_T + t0;
      tma_load_2d(dk, &tmk, 0, y, &full[st], pol);
      tma_load_2d(dv, &tmv, 0, y, &full[st], pol);
      const size_t srow = ((size_t)b * p.H_kv + g) * sc.T_pad + t0;  // T_pad: whole tiles
      bulk_g2s_hint(ds, sc.k + srow, C::kTile * 4, &full[st], pol);
      bulk_g2s_hint(ds + C::kTile, sc.v + srow, C::kTile * 4, &full[st], pol);
    } else {
      const int P = 1 << p.page_shift;
      const int box_rows = P < C::kTile ? P : C::kTile;
      const int32_t* bt = p.block_table + (size_t)b * p.max_pages;
      const int beyond = p.num_pages * p.H_kv * P;  // first row past the pool: zero fill
#pragma unroll 1
      for (int t = t0; t < t0 + C::kTile; t += box_rows) {
        int y = beyond;
        size_t srow = 0;  // past the slice: any finite scales (page 0); weights are zero
        if (t < t_end) {
          const int page = bt[t >> p.page_shift];
          if (page >= 0 && page < p.num_pages) {
            y = (page * p.H_kv + g) * P + (t & (P - 1));
            srow = (size_t)y;
          } else {
            flag_error(p.err, KVC_ERR_BOUNDS);
          }
        }
        const int off = t - t0;
        tma_load_2d(dk + off * D, &tmk, 0, y, &full[st], pol);
        tma_load_2d(dv + off * D, &tmv, 0, y, &full[st], pol);
        bulk_g2s_hint(ds + off, sc.k + srow, box_rows * 4, &full[st], pol);
        bulk_g2s_hint(ds + C::kTile + off, sc.v + srow, box_rows * 4, &full[st], pol);
      }
    }
  };
  int issued = 0;
  if (producer)
    for (; issued < min(S, ntiles); ++issued) issue(issued);

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
  int vis[NT][2];  // this thread's score columns: rows nt*8 + 2(lane%4) + c
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

  const int mi = lane >> 3;
  const int wrow = warp * 16;
  const int k_row = wrow + (mi & 1) * 8 + (lane & 7);
  const int k_cs = mi >> 1;
  const int v_row = wrow + (mi >> 1) * 8 + (lane & 7);
  const int v_cs = mi & 1;
  const uint32_t kb = smem_addr(bk);
  const uint32_t vb = smem_addr(bv);
  constexpr int kChunks = 16 * D / 16;  // 16-code chunks in this warp's 16 rows

  bool ok = true;
  int consumed = 0;
#pragma unroll 1
  for (int j = 0; j < ntiles; ++j) {
    const int st = j % S;
    if (producer && j >= 1 && issued < ntiles) {
      if (mbar_wait(&empty[(j - 1) % S], ((j - 1) / S) & 1, p.err)) {
        issue(issued);
        ++issued;
      } else {
        ok = false;
      }
    }
    if (!ok || !mbar_wait(&full[st], (j / S) & 1, p.err)) {
      ok = false;
      break;
    }
    consumed = j + 1;
    const int t0 = sp.real(t_begin + j * C::kTile);

    // this warp's 16 tokens: codes -> bf16 (swizzled), scales -> registers
    {
      const unsigned char* srck = ck + st * C::kCodeBytes + wrow * D;
      const unsigned char* srcv = cv + st * C::kCodeBytes + wrow * D;
#pragma unroll
      for (int c = lane; c < kChunks; c += 32) {
        const int row = wrow + c / (D / 16);
        const int col = c % (D / 16);  // 16 codes = two 16-byte bf16 chunks
        uint4 lo, hi;
        e4m3x16_to_bf16(ld_shared_v4(srck + c * 16), lo, hi);
        st_shared_v4(bk + swz<D>(row, 2 * col), lo);
        st_shared_v4(bk + swz<D>(row, 2 * col + 1), hi);
        e4m3x16_to_bf16(ld_shared_v4(srcv + c * 16), lo, hi);
        st_shared_v4(bv + swz<D>(row, 2 * col), lo);
        st_shared_v4(bv + swz<D>(row, 2 * col + 1), hi);
      }
    }
    const float* ssc = scl + st * (2 * C::kTile);
    const int ta = wrow + (lane >> 2);  // this thread's two tokens: ta and ta + 8
    const float ska = ssc[ta], skb = ssc[ta + 8];
    const float sva = ssc[C::kTile + ta], svb = ssc[C::kTile + ta + 8];
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);  // the codes are consumed: refill early

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

    // K scales and base-2 units, mask, online softmax per score column (query row)
    const int tok0 = t0 + ta;
    const bool unmasked = tile_fully_visible(t0, C::kTile, vis_min, n_blk, p.window, p.sink);
    const float fa = p.scale_log2 * ska, fb = p.scale_log2 * skb;
    bool grew = false;
    float alpha[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float s0 = sacc[nt][c] * fa;
        float s1 = sacc[nt][2 + c] * fb;
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
        sacc[nt][c] = p0 * sva;  // the V scale enters the weight, not the sum
        sacc[nt][2 + c] = p1 * svb;
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
    // P^T fragments (bf16 hi and lo): transpose each 8x8 (token x row) block
    uint32_t pb[NT][2], pl[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint32_t h0 = Elt<T>::pack2(sacc[nt][0], sacc[nt][1]);
      const uint32_t h1 = Elt<T>::pack2(sacc[nt][2], sacc[nt][3]);
      pb[nt][0] = movmatrix_trans(h0);
      pb[nt][1] = movmatrix_trans(h1);
      pl[nt][0] = movmatrix_trans(bf16_remainder2(sacc[nt][0], sacc[nt][1], h0));
      pl[nt][1] = movmatrix_trans(bf16_remainder2(sacc[nt][2], sacc[nt][3], h1));
    }
    // O^T += V^T . P^T
#pragma unroll
    for (int mt = 0; mt < C::kMTiles; ++mt) {
      uint32_t a[4];
      ldmatrix_x4_trans(a, vb + swz<D>(v_row, 2 * mt + v_cs));
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        mma_16816<T>(o[mt][nt], a, pb[nt][0], pb[nt][1]);
        mma_16816<T>(o[mt][nt], a, pl[nt][0], pl[nt][1]);
      }
    }
    __syncwarp();  // this warp's bf16 rows are rewritten by its next tile
  }
  if (!ok) {
    atomicOr(&flags[0], 1);
    if (producer)
#pragma unroll 1
      for (int j = consumed; j < issued; ++j)
        if (!mbar_wait(&full[j % S], (j / S) & 1, p.err)) break;
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
  named_barrier_sync(1, NTH);  // the rings are free
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
