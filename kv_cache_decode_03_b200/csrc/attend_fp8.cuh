// attend_fp8.cuh -- N2 for the FP8 cache (fp8.cuh): split-K attention whose K/V tiles
// arrive as E4M3 codes with one fp32 scale per (token, KV head).
//
// Same contract and structure as attend_mma.cuh (mma.m16n8k16 with the K/V tokens as M
// and the query rows as N, fixed split-K, the shared slice epilogue, windows through
// window.cuh).  The codes never pass through shared memory as wider values:
//   - thread 0 loads each 64-token tile's codes with 2-D TMA (one D-byte row a token,
//     128-byte swizzle for D = 128, 64-byte for D = 64, no multicast) and the tile's K
//     and V scales with 1-D bulk copies;
//   - K: ldmatrix reads 16-byte code chunks; each 32-bit fragment register holds codes
//     4c..4c+3 of a row, which two cvt.f16x2.e4m3x2 turn into the f16 A-fragment
//     halves for k = 2c, 2c+1 and k = 8+2c, 9+2c -- a fixed permutation of the k index
//     that the Q fragments (built once) follow, so q.k is unchanged;
//   - V: the same loads and conversions, then movmatrix.trans of each 8x8 f16 block
//     gives V^T fragments whose 16 D-rows come in a fixed permuted order (codes
//     0,1,4,5,8,9,12,13 then 2,3,6,7,10,11,14,15 of each chunk), undone when the
//     accumulators are written out;
//   - the MMAs run in f16 (E4M3 converts to f16 exactly).  Each query row is scaled by a
//     power of two into f16 range (exact; folded back into the score).  The K scale
//     multiplies the token's score; the V scale enters the p.V weight through a second
//     running maximum over s + log2(v_scale), so the f16 weights stay <= 1, while the
//     sum l keeps its own maximum; out = O * 2^(mo - m) / l is attention over
//     code * scale exactly, up to fp32 rounding and the 11-bit f16 weights.
// bf16 q/out only.
#pragma once

#include <cuda.h>
#include <math.h>

#include "device_common.cuh"
#include "fp8.cuh"
#include "params.cuh"
#include "splitk_epilogue.cuh"
#include "window.cuh"

namespace kvc {

template <int D>
struct Fp8Cfg {
  static_assert(D == 64 || D == 128, "FP8 attend: D must be 64 or 128");
  static constexpr int kWarps = 4;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kTile = 64;                 // tokens per stage, 16 per warp
  static constexpr int kCodeBytes = kTile * D;     // K (or V) codes per stage
  static constexpr int kChunks = D / 16;           // 16-code chunks in a row
  static constexpr int kStages = 4;
  static constexpr int kRing = 2 * kStages * kCodeBytes;
  static constexpr int kScaleBytes = 2 * kTile * 4;  // K and V scales of a tile
  static constexpr int kData = kRing + kStages * kScaleBytes;

  template <int NT>
  static constexpr size_t smem_bytes() {
    return 1024 + kData + kWarps * NT * 8 * 2 * sizeof(float) + NT * 8 * sizeof(int) +
           2 * kStages * sizeof(uint64_t) + 16;
  }
  template <int NT>
  static constexpr int scratch_floats() {
    return (kData - kWarps * NT * 8 * D * (int)sizeof(float)) / (int)sizeof(float);
  }
  static_assert(kRing >= kWarps * 32 * D * 4, "the result buffer must fit the rings");
};

// Byte offset of 16-byte chunk `chunk` of code row `row` in a swizzled tile: TMA's
// 128-byte swizzle (D = 128: one row is one 128-byte line) or 64-byte swizzle (D = 64).
template <int D>
__device__ __forceinline__ uint32_t swz8(int row, int chunk) {
  if constexpr (D == 128) return row * 128 + ((chunk ^ (row & 7)) << 4);
  else return row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4);
}

__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)two_codes));
  return h2;
}

__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Row of chunk `chunk`'s 16 d-values that V^T row rho (0..15) of an m-tile holds.
__device__ __forceinline__ int vt_row_to_d(int rho) {
  const int j = rho & 7;
  return 4 * (j >> 1) + (j & 1) + (rho >= 8 ? 2 : 0);
}

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
  constexpr int KC = C::kChunks;
  extern __shared__ unsigned char fp8_smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(fp8_smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ck = smem;                               // K code stages
  unsigned char* cv = smem + S * C::kCodeBytes;           // V code stages
  float* scl = reinterpret_cast<float*>(smem + C::kRing);  // [S][K 64 | V 64]
  float* red_m = reinterpret_cast<float*>(smem + C::kData);
  float* red_l = red_m + W * R;
  int* qexp = reinterpret_cast<int*>(red_l + W * R);      // [R] query-row exponents
  uint64_t* full = reinterpret_cast<uint64_t*>(qexp + R);
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

  // ------------------------------------------------------------- query rows
  // Q^T fragments (B operand, f16), row n = nt*8 + lane/4, under the k permutation of
  // the K fragments: k = 2c, 2c+1 <-> d = 16kk + 4c, +1; k = 8+2c, 9+2c <-> d = 16kk+4c+2, +3
  // (c = lane % 4).  Row n is first scaled by 2^-e_n, e_n putting its largest |q| in
  // [2^14, 2^15) (exact; e_n is folded back into the row's scores).
  uint32_t qb[KC][NT][2];
  {
    const __nv_bfloat16* qblk = static_cast<const __nv_bfloat16*>(p.q) +
                                ((((size_t)b * p.H_q + (size_t)g * p.group) * p.T_new) + r0) * D;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int row = nt * 8 + (lane >> 2);
      float qv[KC][4];
      float amax = 0.f;
#pragma unroll
      for (int kk = 0; kk < KC; ++kk) {
        uint2 w = make_uint2(0u, 0u);
        if (row < nr)
          w = __ldg(reinterpret_cast<const uint2*>(qblk + (size_t)row * D + kk * 16 +
                                                   (lane & 3) * 4));
        qv[kk][0] = __uint_as_float(w.x << 16);
        qv[kk][1] = __uint_as_float(w.x & 0xFFFF0000u);
        qv[kk][2] = __uint_as_float(w.y << 16);
        qv[kk][3] = __uint_as_float(w.y & 0xFFFF0000u);
#pragma unroll
        for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(qv[kk][e]));
      }
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      // e = exponent of amax - 14 (0 for a zero row), at least -126 so that 2^-e and 2^e
      // are normal floats built by exponent arithmetic
      const int e =
          amax > 0.f ? max((int)((__float_as_uint(amax) >> 23) & 0xFF) - 127 - 14, -126) : 0;
      const float inv = __uint_as_float((uint32_t)(127 - e) << 23);
#pragma unroll
      for (int kk = 0; kk < KC; ++kk) {
        qb[kk][nt][0] = f32x2_to_f16x2(qv[kk][0] * inv, qv[kk][1] * inv);
        qb[kk][nt][1] = f32x2_to_f16x2(qv[kk][2] * inv, qv[kk][3] * inv);
      }
      if (warp == 0 && (lane & 3) == 0) qexp[row] = e;
    }
  }
  __syncthreads();  // barriers initialised, row exponents published

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
  int vis[NT][2];    // this thread's score columns: rows nt*8 + 2(lane%4) + c
  float fcol[NT][2];  // their score factors: scale * log2(e) * 2^e_row
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int rr = nt * 8 + (lane & 3) * 2 + c;
      vis[nt][c] = rr < nr ? L + (r0 + rr) % p.T_new + 1 : 0;
      fcol[nt][c] = p.scale_log2 * __uint_as_float((uint32_t)(127 + qexp[rr]) << 23);
    }

  // per column: m / l for the softmax sum, mo for the weights of O (s + log2 v_scale)
  float m[NT][2], l[NT][2], mo[NT][2];
  float o[KC][NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m[nt][0] = m[nt][1] = -INFINITY;
    mo[nt][0] = mo[nt][1] = -INFINITY;
    l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < KC; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[mt][nt][e] = 0.f;
  }

  // ldmatrix row addresses: matrices (tokens 0-7 | 8-15) x (chunk j | j+1) of this warp
  const int wrow = warp * 16;
  const int mi = lane >> 3;
  const int ld_row = wrow + (mi & 1) * 8 + (lane & 7);
  const int ld_cs = mi >> 1;
  const uint32_t ck_addr = smem_addr(ck);
  const uint32_t cv_addr = smem_addr(cv);

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
    const uint32_t kb = ck_addr + st * C::kCodeBytes;
    const uint32_t vb = cv_addr + st * C::kCodeBytes;
    const int t0 = sp.real(t_begin + j * C::kTile);
    const float* ssc = scl + st * (2 * C::kTile);
    const int ta = wrow + (lane >> 2);  // this thread's two tokens: ta and ta + 8
    const float ska = ssc[ta], skb = ssc[ta + 8];
    const float lva = __log2f(ssc[C::kTile + ta]), lvb = __log2f(ssc[C::kTile + ta + 8]);

    // S^T = K . Q^T for this warp's 16 tokens, K converted in registers
    float sacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
    for (int kp = 0; kp < KC; kp += 2) {
      uint32_t r[4];
      ldmatrix_x4(r, kb + swz8<D>(ld_row, kp + ld_cs));
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // chunk kp + h: registers r[2h] (tokens 0-7), r[2h+1]
        const uint32_t a[4] = {e4m3x2_to_f16x2(r[2 * h]), e4m3x2_to_f16x2(r[2 * h + 1]),
                               e4m3x2_to_f16x2(r[2 * h] >> 16),
                               e4m3x2_to_f16x2(r[2 * h + 1] >> 16)};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_16816<__half>(sacc[nt], a, qb[kp + h][nt][0], qb[kp + h][nt][1]);
      }
    }

    // scores (base 2), mask, two running maxima per score column (query row)
    const int tok0 = t0 + ta;
    const bool unmasked = tile_fully_visible(t0, C::kTile, vis_min, n_blk, p.window, p.sink);
    bool grew = false;
    float alpha_o[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float s0 = sacc[nt][c] * fcol[nt][c] * ska;
        float s1 = sacc[nt][2 + c] * fcol[nt][c] * skb;
        if (!unmasked) {
          s0 = visible(tok0, vis[nt][c], p.window, p.sink) ? s0 : -INFINITY;
          s1 = visible(tok0 + 8, vis[nt][c], p.window, p.sink) ? s1 : -INFINITY;
        }
        // the sum l, referenced to m
        float mx = fmaxf(s0, s1);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m[nt][c], mx);
        const float mu = (m_new == -INFINITY) ? 0.f : m_new;
        l[nt][c] = fmaf(l[nt][c], exp2f(m[nt][c] - mu), exp2f(s0 - mu) + exp2f(s1 - mu));
        m[nt][c] = m_new;
        // the weights of O, referenced to mo: 2^(s + log2 v_scale - mo) <= 1
        const float w0 = s0 + lva, w1 = s1 + lvb;
        float mxo = fmaxf(w0, w1);
        mxo = fmaxf(mxo, __shfl_xor_sync(0xffffffffu, mxo, 4));
        mxo = fmaxf(mxo, __shfl_xor_sync(0xffffffffu, mxo, 8));
        mxo = fmaxf(mxo, __shfl_xor_sync(0xffffffffu, mxo, 16));
        const float mo_new = fmaxf(mo[nt][c], mxo);
        const float muo = (mo_new == -INFINITY) ? 0.f : mo_new;
        alpha_o[nt][c] = exp2f(mo[nt][c] - muo);
        grew |= (mo_new > mo[nt][c]);
        mo[nt][c] = mo_new;
        sacc[nt][c] = exp2f(w0 - muo);
        sacc[nt][2 + c] = exp2f(w1 - muo);
      }
    }
    if (__any_sync(0xffffffffu, grew)) {
#pragma unroll
      for (int mt = 0; mt < KC; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          o[mt][nt][0] *= alpha_o[nt][0];
          o[mt][nt][1] *= alpha_o[nt][1];
          o[mt][nt][2] *= alpha_o[nt][0];
          o[mt][nt][3] *= alpha_o[nt][1];
        }
    }
    // P^T fragments (f16): transpose each 8x8 (token x row) block
    uint32_t pb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      pb[nt][0] = movmatrix_trans(f32x2_to_f16x2(sacc[nt][0], sacc[nt][1]));
      pb[nt][1] = movmatrix_trans(f32x2_to_f16x2(sacc[nt][2], sacc[nt][3]));
    }
    // O^T += V^T . P^T, V^T from the codes: convert, then transpose each 8x8 block
#pragma unroll
    for (int kp = 0; kp < KC; kp += 2) {
      uint32_t r[4];
      ldmatrix_x4(r, vb + swz8<D>(ld_row, kp + ld_cs));
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // m-tile kp + h: d rows of chunk kp + h
        const uint32_t a[4] = {movmatrix_trans(e4m3x2_to_f16x2(r[2 * h])),
                               movmatrix_trans(e4m3x2_to_f16x2(r[2 * h] >> 16)),
                               movmatrix_trans(e4m3x2_to_f16x2(r[2 * h + 1])),
                               movmatrix_trans(e4m3x2_to_f16x2(r[2 * h + 1] >> 16))};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_16816<__half>(o[kp + h][nt], a, pb[nt][0], pb[nt][1]);
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
  // O referenced to m: O * 2^(mo - m); V^T row rho of m-tile mt is d = 16 mt + vt_row_to_d(rho)
  float f[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int c = 0; c < 2; ++c)
      f[nt][c] = (m[nt][c] == -INFINITY || mo[nt][c] == -INFINITY) ? 0.f
                                                                  : exp2f(mo[nt][c] - m[nt][c]);
#pragma unroll
  for (int mt = 0; mt < KC; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = nt * 8 + (lane & 3) * 2 + (e & 1);
        const int d = mt * 16 + vt_row_to_d((lane >> 2) + (e >> 1) * 8);
        red_acc[(warp * R + row) * D + d] = o[mt][nt][e] * f[nt][e & 1];
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
