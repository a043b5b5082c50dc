// attend_tc.cuh -- N2 (5th-generation tensor cores): split-K attention for many
// query rows per KV head (MQA verify chunks, large GQA groups, chunked prefill).
//
// Same contract as the other attend kernels: for every query row (query head h
// of KV head g, new row i) of request b, exact-softmax attention over positions
// 0 .. L_b + i ("项目 9-16" projects 11/15; "9. 推理" 9.7).  With 64 or more rows
// sharing each K/V row the work is a real dense contraction, so a CTA takes a
// block of 128 query rows as the MMA M dimension:
//     S[128 x 64]  = Q[128 x D] . K_tile^T        tcgen05.mma, fp32 in TMEM
//     O[128 x D]  += P[128 x 64] . V_tile          tcgen05.mma, fp32 in TMEM
// Thread 0 issues the TMA loads and the MMAs; thread t owns TMEM lane t, i.e.
// query row t, for the softmax: it reads its 64 scores with tcgen05.ld, keeps
// the running max and sum in registers and writes its row of P back over the
// scores in TMEM, where the second MMA takes it as its A operand.
//
// Precision of P: a bf16 P (8-bit significand) moves short-context outputs by
// up to ~2^-9 max|v|, several times the 2e-3 bound on the output.  For bf16
// caches P is therefore split as P = P_hi + P_lo (both bf16, P_lo the rounded
// remainder) and O accumulates P_hi.V + P_lo.V, leaving ~2^-17 relative error.
// fp16 (11-bit significand) takes P in one piece.
//
// Rescaling is lazy: a row's reference max only moves when a tile's max
// exceeds it by more than 2^8 (then that row of O is rescaled in TMEM by its own
// thread), so P stays below 2^8 and the sum l and the accumulator O always share
// one reference; the result is exact softmax either way.
//
// Shared-memory operands use the canonical 128-byte-swizzled layouts the TMA
// tiles already have: Q and K are K-major (8-row groups of 1024 bytes,
// 16-element k-steps of 32 bytes inside a row), V is MN-major (64-element boxes
// along D, 8-token groups of 1024 bytes).  TMEM: S in columns [0, 64), then P
// over it (two 16-bit values per column: P_hi in [0, 32), P_lo in [32, 64)),
// O in [64, 64 + D).
//
// Every wait is bounded; a timeout raises KVC_ERR_TIMEOUT, all threads leave
// the loop together (barrier with a vote), thread 0 waits (bounded) for its
// copies and MMAs in flight, and the TMEM is released before the CTA exits.
#pragma once

#include <cuda.h>
#include <math.h>

#include "device_common.cuh"
#include "params.cuh"
#include "splitk_epilogue.cuh"

#ifndef KVC_TC_STAGES
#define KVC_TC_STAGES 2
#endif

namespace kvc {

template <int D>
struct TcCfg {
  static_assert(D == 64 || D == 128, "tcgen05 attend: D must be 64 or 128");
  static constexpr int kThreads = 128;           // one thread per query row (TMEM lane)
  static constexpr int kRows = 128;              // MMA M
  static constexpr int kTile = 64;               // tokens per K/V tile (MMA N of S)
  static constexpr int kHalves = D / 64;         // 64-element boxes across a row
  static constexpr int kBoxBytes = kTile * 128;  // one box of a K/V tile
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kStages = KVC_TC_STAGES;
  static constexpr int kRing = 2 * kStages * kTileBytes;  // K stages, then V stages
  static constexpr int kQBox = kRows * 128;               // one 64-element box of Q
  static constexpr int kQBytes = kRows * D * 2;
  static constexpr int kTmemCols = D == 64 ? 128 : 256;   // S/P + O, a power of two
  static constexpr int kData = kRing + kQBytes;           // 1024-aligned operand area
  // after the loop the operand area holds the per-row results:
  static constexpr int kAccLd = D + 4;  // padded rows: conflict-free float4 stores
  static constexpr int kAccBytes = kRows * kAccLd * 4;
  static constexpr int kScratchOff = kAccBytes + 2 * kRows * 4;
  static constexpr int kScratchFloats = (kData - kScratchOff) / 4;
  static_assert(kScratchOff + kRows * 4 <= kData, "result area too small");

  static constexpr size_t smem_bytes() {
    return 1024 /* alignment slack */ + kData + (kStages + 3) * sizeof(uint64_t) + 16;
  }
};

// UMMA shared-memory descriptor for a 128-byte-swizzled operand whose atoms
// start on 1024-byte boundaries (base offset 0).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  const uint32_t lo = ((saddr >> 4) & 0x3FFFu) | (((lbo >> 4) & 0x3FFFu) << 16);
  const uint32_t hi = ((sbo >> 4) & 0x3FFFu) | (1u << 14)  // descriptor version 1
                      | (2u << 29);                        // layout: 128-byte swizzle
  return (uint64_t(hi) << 32) | lo;
}

// Instruction descriptor, kind::f16 with fp32 accumulation; A K-major.
template <typename T>
__host__ __device__ constexpr uint32_t umma_idesc(int M, int N, bool b_mn_major) {
  return (1u << 4)                                              // D: f32
         | ((Elt<T>::kCode == KVC_BF16 ? 1u : 0u) << 7)          // A: bf16 / f16
         | ((Elt<T>::kCode == KVC_BF16 ? 1u : 0u) << 10)         // B: same type as A
         | ((b_mn_major ? 1u : 0u) << 16) | (uint32_t(N >> 3) << 17) |
         (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                         bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate ? 1 : 0)
      : "memory");
}

// The same with the A operand in TMEM (K-major: row m in lane m, two 16-bit
// elements per 32-bit column).
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t b,
                                                uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(b), "r"(idesc), "r"(accumulate ? 1 : 0)
      : "memory");
}

// Arrive on `bar` once every tcgen05.mma this thread issued before has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Generic-proxy shared-memory writes become visible to the tensor cores.
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

template <int D, typename T, bool PAGED>
__global__ void __launch_bounds__(TcCfg<D>::kThreads)
    attend_tc_kernel(const AttendParams p, const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv) {
  using C = TcCfg<D>;
  constexpr int R = C::kRows;
  constexpr int NTH = C::kThreads;
  constexpr int S = C::kStages;
  constexpr bool kSplitP = Elt<T>::kCode == KVC_BF16;
  extern __shared__ __align__(1024) unsigned char tc_smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sk = smem;                      // K stages
  unsigned char* sv = smem + S * C::kTileBytes;  // V stages
  unsigned char* sq = smem + C::kRing;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kData);
  uint64_t* sbar = full + S;  // S = Q.K^T done
  uint64_t* obar = sbar + 1;  // O += P.V done
  uint64_t* dbar = obar + 1;  // drain after an abort
  uint32_t* tslot = reinterpret_cast<uint32_t*>(dbar + 1);
  int* flags = reinterpret_cast<int*>(tslot + 1);  // [0] abort [1] last
  float* red_acc = reinterpret_cast<float*>(smem);  // operand area, after the loop
  float* red_m = reinterpret_cast<float*>(smem + C::kAccBytes);
  float* red_l = red_m + R;
  float* scratch = reinterpret_cast<float*>(smem + C::kScratchOff);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int s = blockIdx.x / p.row_blocks;  // row blocks vary fastest (shared K/V in L2)
  const int rb = blockIdx.x - s * p.row_blocks;
  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int L = p.seq_lens[b];
  const int r0 = rb * R;
  const int nr = min(R, p.rows - r0);

  // last new row of the block: the block sees positions [0, L + i_max]
  int i_max = p.T_new - 1;
  if (nr < p.T_new) {
    const int i0 = r0 % p.T_new, i1 = (r0 + nr - 1) % p.T_new;
    if (i1 >= i0) i_max = i1;
  }
  const int n_blk = L + i_max + 1;
  const int t_begin = s * p.split_tokens;
  if (t_begin >= n_blk) return;
  if (L < 0 || L + p.T_new > p.max_T ||
      (PAGED && ((L + p.T_new - 1) >> p.page_shift) >= p.max_pages)) {
    if (tid == 0) flag_error(p.err, KVC_ERR_BOUNDS);
    return;
  }
  const int t_stop = min(t_begin + p.split_tokens, n_blk);
  const int ntiles = ceil_div(t_stop - t_begin, C::kTile);
  const int ns_blk = ceil_div(n_blk, p.split_tokens);

  // ---- TMEM, barriers, and Q: row tid in 64-element boxes, 128-byte swizzled
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tslot)),
                 "r"(C::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
#pragma unroll
    for (int st = 0; st < S; ++st) mbar_init(&full[st], 1);
    mbar_init(sbar, 1);
    mbar_init(obar, 1);
    mbar_init(dbar, 1);
    flags[0] = 0;
    flags[1] = 0;
    fence_barrier_init();
  }
  {
    const char* qrow =
        static_cast<const char*>(p.q) +
        ((((size_t)b * p.H_q + (size_t)g * p.group) * p.T_new) + r0 + tid) * D * 2;
#pragma unroll
    for (int ch = 0; ch < D / 8; ++ch) {
      const uint4 v = tid < nr ? ld_global_nc_v4(qrow + ch * 16) : make_uint4(0, 0, 0, 0);
      st_shared_v4(sq + (ch >> 3) * C::kQBox + tid * 128 + (((ch & 7) ^ (tid & 7)) << 4), v);
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tS = tmem;                           // columns [0, 64)
  const uint32_t tO = tmem + 64;                      // columns [64, 64 + D)
  const uint32_t lane = (uint32_t)(warp * 32) << 16;  // this warp's 32 TMEM lanes

  volatile int* abort_word = flags;
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*abort_word) return false;
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t_start = global_timer_ns();
#pragma unroll 1
    while (true) {
      if (mbar_try_wait(bar, parity)) return true;
      if (*abort_word) return false;
      if (global_timer_ns() - t_start > kWaitLimitNs) {
        flag_error(p.err, KVC_ERR_TIMEOUT);
        *abort_word = 1;
        return false;
      }
    }
  };

  // ---- producer (thread 0): K and V tiles of 64 tokens by TMA, no multicast
  const uint64_t pol = p.row_blocks > 1 ? l2_policy_evict_normal() : l2_policy_evict_first();
  int issued = 0, consumed = 0;
  bool mma_issued = false;
  auto issue = [&](int j) {
    const int st = j % S;
    const int t0 = t_begin + j * C::kTile;
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
      const int Pg = 1 << p.page_shift;
      const int box_rows = Pg < C::kTile ? Pg : C::kTile;
      const int32_t* bt = p.block_table + (size_t)b * p.max_pages;
      const int beyond = p.num_pages * p.H_kv * Pg;  // first row past the pool: zero fill
#pragma unroll 1
      for (int t = t0; t < t0 + C::kTile; t += box_rows) {
        int y = beyond;
        if (t < t_stop) {
          const int page = bt[t >> p.page_shift];
          if (page >= 0 && page < p.num_pages)
            y = (page * p.H_kv + g) * Pg + (t & (Pg - 1));
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
    ++issued;
  };
  if (tid == 0) {
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
    for (int j = 0; j < min(S, ntiles); ++j) issue(j);
  }

  const uint32_t idesc_s = umma_idesc<T>(R, C::kTile, false);
  const uint32_t idesc_o = umma_idesc<T>(R, D, true);
  const uint32_t sq_a = smem_addr(sq), sk_a = smem_addr(sk), sv_a = smem_addr(sv);

  // this thread's query row sees positions [0, vis)
  const int vis = tid < nr ? L + (r0 + tid) % p.T_new + 1 : 0;
  float m_ref = -INFINITY, l = 0.f;

#pragma unroll 1
  for (int j = 0; j < ntiles; ++j) {
    const int st = j % S;
    if (tid == 0 && !*abort_word) {
      if (wait(&full[st], (j / S) & 1)) {
        ++consumed;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qoff = (kk >> 2) * C::kQBox + (kk & 3) * 32;
          const uint32_t koff = st * C::kTileBytes + (kk >> 2) * C::kBoxBytes + (kk & 3) * 32;
          umma_f16(tS, umma_desc_sw128(sq_a + qoff, 16, 1024),
                   umma_desc_sw128(sk_a + koff, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit(sbar);
        mma_issued = true;
      }
    }
    // tcgen05.ld / st below are warp-collective: a warp goes on only as a whole
    const bool ok = __all_sync(0xffffffffu, wait(sbar, j & 1));
    if (ok) {
      tc_fence_after();
      // ---- softmax of this thread's row over the tile's 64 tokens
      float sc[64];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_ld16(tS + lane + c4 * 16, sc + c4 * 16);
      tmem_wait_ld();
      const int t0 = t_begin + j * C::kTile;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        sc[c] = (t0 + c < vis) ? sc[c] * p.scale_log2 : -INFINITY;
        mx = fmaxf(mx, sc[c]);
      }
      // Move the reference max when the tile's max passes it by 2^8 and rescale
      // this row of O (before any visible token the row is all zero: alpha 1).
      const bool move = mx > m_ref + 8.f;
      const float alpha = (move && m_ref != -INFINITY) ? exp2f(m_ref - mx) : 1.f;
      if (__any_sync(0xffffffffu, alpha != 1.f)) {  // the warp's 32 rows together
#pragma unroll 1
        for (int c16 = 0; c16 < D / 16; ++c16) {
          float ov[16];
          tmem_ld16(tO + lane + c16 * 16, ov);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) ov[i] *= alpha;
          tmem_st16(tO + lane + c16 * 16, ov);
        }
        tmem_wait_st();
      }
      if (move) {
        l *= alpha;
        m_ref = mx;
      }
      const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
      uint32_t ph[32];
      float lsum = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float p0 = exp2f(sc[2 * c] - mu);
        const float p1 = exp2f(sc[2 * c + 1] - mu);
        lsum += p0 + p1;
        ph[c] = Elt<T>::pack2(p0, p1);
        if constexpr (kSplitP) {  // keep the rounding remainder in sc[] for P_lo
          sc[2 * c] = p0 - __uint_as_float(ph[c] << 16);
          sc[2 * c + 1] = p1 - __uint_as_float(ph[c] & 0xFFFF0000u);
        }
      }
      l += lsum;
      // P over this row's scores: 64 tokens in 32 columns (even token low half)
      tmem_st16(tS + lane, ph);
      tmem_st16(tS + lane + 16, ph + 16);
      if constexpr (kSplitP) {
        uint32_t pl[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pl[c] = Elt<T>::pack2(sc[2 * c], sc[2 * c + 1]);
        tmem_st16(tS + lane + 32, pl);
        tmem_st16(tS + lane + 48, pl + 16);
      }
      tmem_wait_st();
      tc_fence_before();
    }
    if (__syncthreads_or(!ok)) break;  // everyone leaves together

    if (tid == 0) {  // O += P . V, then refill the stage once it is free
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < C::kTile / 16; ++kk) {
        const uint64_t bv =
            umma_desc_sw128(sv_a + st * C::kTileBytes + kk * 2048, C::kBoxBytes, 1024);
        umma_f16_tmem_a(tO, tS + kk * 8, bv, idesc_o, j > 0 || kk > 0);
        if constexpr (kSplitP) umma_f16_tmem_a(tO, tS + 32 + kk * 8, bv, idesc_o, true);
      }
      umma_commit(obar);
      if (wait(obar, j & 1) && j + S < ntiles) issue(j + S);
    }
  }

  const bool bad = __syncthreads_or(*abort_word != 0);
  if (bad) {
    if (tid == 0) {  // nothing may still write this CTA's shared memory or TMEM
      if (mma_issued) {
        umma_commit(dbar);
        mbar_wait(dbar, 0, p.err);
      }
      for (int j = consumed; j < issued; ++j)
        if (!mbar_wait(&full[j % S], (j / S) & 1, p.err)) break;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(C::kTmemCols)
                   : "memory");
    return;
  }

  // ---- this row's unnormalised O, reference max and sum to shared memory
  tc_fence_after();
#pragma unroll 1
  for (int c16 = 0; c16 < D / 16; ++c16) {
    float ov[16];
    tmem_ld16(tO + lane + c16 * 16, ov);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; i += 4)
      *reinterpret_cast<float4*>(red_acc + tid * C::kAccLd + c16 * 16 + i) =
          make_float4(ov[i], ov[i + 1], ov[i + 2], ov[i + 3]);
  }
  red_m[tid] = m_ref;
  red_l[tid] = l;
  tc_fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::kTmemCols)
                 : "memory");
  finish_slice<T, D, R, 1, NTH, C::kAccLd>(p, red_acc, red_m, red_l, scratch, &flags[1], b, g, rb,
                                           s, r0, nr, L, ns_blk);
}

}  // namespace kvc
