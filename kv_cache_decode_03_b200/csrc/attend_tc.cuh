// attend_tc.cuh -- N2 (5th-generation tensor cores): split-K attention for many
// query rows per KV head (MQA verify chunks, large GQA groups, chunked prefill).
//
// Same contract as the other attend kernels: for every query row (query head h
// of KV head g, new row i) of request b, exact-softmax attention over positions
// 0 .. L_b + i ("项目 9-16" projects 11/15; "9. 推理" 9.7).  With many rows sharing
// each K/V row the work is a real dense contraction, so a CTA takes a block of 128
// query rows as the MMA M dimension (the library routes 17 or more rows per KV head
// here; with fewer than 128 the rest of the block idles and it still pays):
//     S[128 x 64]  = Q[128 x D] . K_tile^T        tcgen05.mma, fp32 in TMEM
//     O[128 x D]  += P[128 x 64] . V_tile          tcgen05.mma, fp32 in TMEM
// Roles (warp-specialised, 224 threads):
//   warps 5, 6  TMA producers of K and of V tiles (64 tokens) into two rings;
//            a K stage is free again as soon as its S MMA is done, so K runs
//            several tiles ahead of V; the page lookups of a tile are spread
//            over the warp's lanes;
//   warp 4   MMA issuer (one lane): S(j+1) = Q.K(j+1)^T is issued while the
//            softmax of tile j runs (S double-buffered in TMEM), then
//            O += P(j).V(j) once P(j) is written;
//   warps 0-3 softmax: thread t owns TMEM lane t, i.e. query row t: it reads
//            its 64 scores with tcgen05.ld, keeps the running max and sum in
//            registers and writes its row of P back over the scores in TMEM,
//            where the P.V MMA takes it as its A operand.
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
// along D, 8-token groups of 1024 bytes).  TMEM: two S buffers in columns
// [0, 64) and [64, 128), each overwritten by its P (two 16-bit values per
// column: P_hi in the first 32 columns, P_lo in the next 32), O in
// [128, 128 + D).
//
// Every wait is bounded; a timeout raises KVC_ERR_TIMEOUT and sets the CTA's
// abort word, which ends every role's loop; the CTA then agrees on the abort
// with a barrier vote, the producer and the MMA lane wait (bounded) for their
// copies and MMAs in flight, and the TMEM is released before the CTA exits.
#pragma once

#include <cuda.h>
#include <math.h>

#include "device_common.cuh"
#include "params.cuh"
#include "splitk_epilogue.cuh"


#ifndef KVC_TC_KSTAGES_D128
#define KVC_TC_KSTAGES_D128 3
#endif
#ifndef KVC_TC_VSTAGES_D128
#define KVC_TC_VSTAGES_D128 2
#endif

namespace kvc {

template <int D>
struct TcCfg {
  static_assert(D == 64 || D == 128, "tcgen05 attend: D must be 64 or 128");
  static constexpr int kSoftmaxThreads = 128;    // one thread per query row (TMEM lane)
  static constexpr int kMmaWarp = 4;
  static constexpr int kKWarp = 5;               // K producer
  static constexpr int kVWarp = 6;               // V producer
  static constexpr int kThreads = 224;
  static constexpr int kRows = 128;              // MMA M
  static constexpr int kTile = 64;               // tokens per K/V tile (MMA N of S)
  static constexpr int kHalves = D / 64;         // 64-element boxes across a row
  static constexpr int kBoxBytes = kTile * 128;  // one box of a K/V tile
  static constexpr int kTileBytes = kTile * D * 2;
  // stages sized so that two CTAs share an SM (<= 113 KB of shared memory each)
  static constexpr int kKStages = D == 128 ? KVC_TC_KSTAGES_D128 : 4;
  static constexpr int kVStages = D == 128 ? KVC_TC_VSTAGES_D128 : 4;
  static constexpr int kKRing = kKStages * kTileBytes;
  static constexpr int kVRing = kVStages * kTileBytes;
  static constexpr int kQBox = kRows * 128;      // one 64-element box of Q
  static constexpr int kQBytes = kRows * D * 2;
  static constexpr int kTmemCols = 256;          // S/P x 2, O
  static constexpr int kOCol = 128;
  static constexpr int kData = kKRing + kVRing + kQBytes;  // 1024-aligned operand area
  // after the loop the operand area holds the per-row results:
  static constexpr int kAccLd = D + 4;  // padded rows: conflict-free float4 stores
  static constexpr int kAccBytes = kRows * kAccLd * 4;
  static constexpr int kScratchOff = kAccBytes + 2 * kRows * 4;
  static constexpr int kScratchFloats = (kData - kScratchOff) / 4;
  static_assert(kScratchOff + kRows * 4 <= kData, "result area too small");
  // K full/empty, V full/empty, s_full x2, p_full x2, o_done x2, drain
  static constexpr int kBarriers = 2 * kKStages + 2 * kVStages + 7;

  // The dynamic shared memory starts 1024-byte aligned (checked at run time).
  static constexpr size_t smem_bytes() { return kData + kBarriers * sizeof(uint64_t) + 16; }
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

__device__ __forceinline__ float ex2_approx(float x) {  // MUFU 2^x; 2^-inf = 0
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

template <int D, typename T, bool PAGED>
__global__ void __launch_bounds__(TcCfg<D>::kThreads, 2)
    attend_tc_kernel(const AttendParams p, const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv) {
  using C = TcCfg<D>;
  constexpr int R = C::kRows;
  constexpr int NSM = C::kSoftmaxThreads;
  constexpr int SK = C::kKStages;
  constexpr int SV = C::kVStages;
  constexpr bool kSplitP = Elt<T>::kCode == KVC_BF16;
  extern __shared__ __align__(1024) unsigned char tc_smem[];
  unsigned char* const smem = tc_smem;
  unsigned char* sk = smem;                // K stages
  unsigned char* sv = smem + C::kKRing;    // V stages
  unsigned char* sq = sv + C::kVRing;      // Q
  uint64_t* k_full = reinterpret_cast<uint64_t*>(smem + C::kData);
  uint64_t* k_empty = k_full + SK;   // K stage consumed by its S MMA
  uint64_t* v_full = k_empty + SK;
  uint64_t* v_empty = v_full + SV;   // V stage consumed by its P.V MMA
  uint64_t* s_full = v_empty + SV;   // [2] S buffer holds Q.K^T
  uint64_t* p_full = s_full + 2;     // [2] S buffer holds P (128 arrivals)
  // [2] O += P(j).V(j) done, on o_done[j & 1]: each completes a phase every other tile,
  // so a waiter is never more than one phase behind (a single barrier could be two
  // phases past a P.V still pending, and a parity wait would then match the wrong phase)
  uint64_t* o_done = p_full + 2;
  uint64_t* dbar = o_done + 2;       // drain after an abort
  uint32_t* tslot = reinterpret_cast<uint32_t*>(dbar + 1);
  int* flags = reinterpret_cast<int*>(tslot + 1);  // [0] abort [1] last
  float* red_acc = reinterpret_cast<float*>(smem);  // operand area, after the loop
  float* red_m = reinterpret_cast<float*>(smem + C::kAccBytes);
  float* red_l = red_m + R;
  float* scratch = reinterpret_cast<float*>(smem + C::kScratchOff);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane_id = tid & 31;
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
  int i_min = 0;  // first new row of the block
  if (nr < p.T_new) {
    const int i0 = r0 % p.T_new, i1 = (r0 + nr - 1) % p.T_new;
    if (i1 >= i0) i_min = i0;
  }
  const int vis_min = L + i_min + 1;
  const Span sp = block_span(vis_min, n_blk, p.window, p.sink, C::kTile);
  const int t_begin = s * p.split_tokens;  // virtual positions (window.cuh)
  if (t_begin >= sp.n_virt) return;
  if (smem_addr(smem) & 1023u) {  // swizzle atoms need 1024-byte alignment
    if (tid == 0) flag_error(p.err, KVC_ERR_UNSUPPORTED);
    return;
  }
  if (L < 0 || L + p.T_new > p.max_T ||
      (PAGED && ((L + p.T_new - 1) >> p.page_shift) >= p.max_pages)) {
    if (tid == 0) flag_error(p.err, KVC_ERR_BOUNDS);
    return;
  }
  const int t_stop = min(t_begin + p.split_tokens, sp.n_virt);
  const int ntiles = ceil_div(t_stop - t_begin, C::kTile);
  const int ns_blk = ceil_div(sp.n_virt, p.split_tokens);

  // ---- TMEM, barriers, and Q: row tid in 64-element boxes, 128-byte swizzled
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tslot)),
                 "r"(C::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int st = 0; st < SK; ++st) {
      mbar_init(&k_full[st], 1);
      mbar_init(&k_empty[st], 1);
    }
    for (int st = 0; st < SV; ++st) {
      mbar_init(&v_full[st], 1);
      mbar_init(&v_empty[st], 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&s_full[k], 1);
      mbar_init(&p_full[k], NSM);
    }
    mbar_init(&o_done[0], 1);
    mbar_init(&o_done[1], 1);
    mbar_init(dbar, 1);
    flags[0] = 0;
    flags[1] = 0;
    fence_barrier_init();
  }
  if (tid < NSM) {
    const char* qrow =
        static_cast<const char*>(p.q) +
        ((((size_t)b * p.H_q + (size_t)g * p.group) * p.T_new) + r0 + tid) * D * 2;
#pragma unroll
    for (int ch = 0; ch < D / 8; ++ch) {
      const uint4 v = tid < nr ? ld_global_nc_v4(qrow + ch * 16) : make_uint4(0, 0, 0, 0);
      st_shared_v4(sq + (ch >> 3) * C::kQBox + tid * 128 + (((ch & 7) ^ (tid & 7)) << 4), v);
    }
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tO = tmem + C::kOCol;

  volatile int* abort_word = flags;
  const unsigned long long wait_limit = p.wait_limit_ns ? p.wait_limit_ns : kWaitLimitNs;
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
      if (global_timer_ns() - t_start > wait_limit) {
        flag_error(p.err, KVC_ERR_TIMEOUT);
        *abort_word = 1;
        return false;
      }
    }
  };

  bool ok = true;
  int issued = 0;            // producer: tiles whose loads were issued
  bool mma_issued = false;   // MMA lane
  float m_ref = -INFINITY;   // softmax: the row's reference max (base 2) and
  float l = 0.f;             // sum of 2^(s - m_ref)

  if (warp == C::kKWarp || warp == C::kVWarp) {
    // ---- TMA producers (no multicast): warp 5 loads K, warp 6 loads V; lane k
    // loads box k of a paged tile
    const bool is_k = warp == C::kKWarp;
    const int NS = is_k ? SK : SV;
    unsigned char* ring = is_k ? sk : sv;
    uint64_t* full = is_k ? k_full : v_full;
    uint64_t* empty = is_k ? k_empty : v_empty;
    const CUtensorMap* tm = is_k ? &tmk : &tmv;
    const uint64_t pol = p.row_blocks > 1 ? l2_policy_evict_normal() : l2_policy_evict_first();
    if (lane_id == 0) prefetch_tmap(tm);
#pragma unroll 1
    for (int j = 0; j < ntiles && !p.stall; ++j) {  // a stall (test) issues nothing
      const int st = j % NS;
      if (j >= NS) {
        bool w = true;
        if (lane_id == 0) w = wait(&empty[st], ((j / NS) - 1) & 1);
        if (!__shfl_sync(0xffffffffu, w, 0)) {
          ok = false;
          break;
        }
      }
      const int t0v = t_begin + j * C::kTile;
      const int t0 = sp.real(t0v);
      const int t_end = t0 + (t_stop - t0v);  // real end of the slice within this tile's run
      unsigned char* dst = ring + st * C::kTileBytes;
      if (lane_id == 0) mbar_arrive_expect_tx(&full[st], C::kTileBytes);
      __syncwarp();
      if (!PAGED) {
        if (lane_id < C::kHalves)
          tma_load_2d(dst + lane_id * C::kBoxBytes, tm, lane_id * 64,
                      (b * p.H_kv + g) * p.max_T + t0, &full[st], pol);
      } else {
        const int Pg = 1 << p.page_shift;
        const int box_rows = Pg < C::kTile ? Pg : C::kTile;
        const int nbox = C::kTile / box_rows;  // <= 8 (pages of 8 or more tokens)
        if (lane_id < nbox) {
          const int t = t0 + lane_id * box_rows;
          int y = p.num_pages * p.H_kv * Pg;  // first row past the pool: zero fill
          if (t < t_end) {
            const int page = p.block_table[(size_t)b * p.max_pages + (t >> p.page_shift)];
            if (page >= 0 && page < p.num_pages)
              y = (page * p.H_kv + g) * Pg + (t & (Pg - 1));
            else
              flag_error(p.err, KVC_ERR_BOUNDS);
          }
          const int off = lane_id * box_rows * 128;
#pragma unroll
          for (int h = 0; h < C::kHalves; ++h)
            tma_load_2d(dst + h * C::kBoxBytes + off, tm, h * 64, y, &full[st], pol);
        }
      }
      ++issued;
    }
  } else if (warp == C::kMmaWarp) {
    // ---- MMA issuer: S(j+1) ahead of P(j).V(j); S buffer j&1 holds S(j), then P(j)
    if (lane_id == 0) {
      const uint32_t idesc_s = umma_idesc<T>(R, C::kTile, false);
      const uint32_t idesc_o = umma_idesc<T>(R, D, true);
      const uint32_t sq_a = smem_addr(sq), sk_a = smem_addr(sk), sv_a = smem_addr(sv);
      auto issue_s = [&](int j) -> bool {
        const int st = j % SK;
        if (!wait(&k_full[st], (j / SK) & 1)) return false;
        tc_fence_after();
        const uint32_t tS = tmem + (j & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qoff = (kk >> 2) * C::kQBox + (kk & 3) * 32;
          const uint32_t koff = st * C::kTileBytes + (kk >> 2) * C::kBoxBytes + (kk & 3) * 32;
          umma_f16(tS, umma_desc_sw128(sq_a + qoff, 16, 1024),
                   umma_desc_sw128(sk_a + koff, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit(&s_full[j & 1]);
        umma_commit(&k_empty[st]);
        mma_issued = true;
        return true;
      };
      ok = issue_s(0);
#pragma unroll 1
      for (int j = 0; ok && j < ntiles; ++j) {
        if (j + 1 < ntiles) {
          // buffer (j+1)&1 still holds P(j-1) until its P.V MMA is done
          if (j >= 1 && !wait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1)) {
            ok = false;
            break;
          }
          if (!issue_s(j + 1)) {
            ok = false;
            break;
          }
        }
        const int st = j % SV;
        if (!wait(&p_full[j & 1], (j >> 1) & 1) || !wait(&v_full[st], (j / SV) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tP = tmem + (j & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < C::kTile / 16; ++kk) {
          const uint64_t bv =
              umma_desc_sw128(sv_a + st * C::kTileBytes + kk * 2048, C::kBoxBytes, 1024);
          umma_f16_tmem_a(tO, tP + kk * 8, bv, idesc_o, j > 0 || kk > 0);
          if constexpr (kSplitP) umma_f16_tmem_a(tO, tP + 32 + kk * 8, bv, idesc_o, true);
        }
        umma_commit(&v_empty[st]);
        umma_commit(&o_done[j & 1]);
      }
    }
    __syncwarp();
  } else {
    // ---- softmax: thread tid owns query row tid (TMEM lane tid)
    const uint32_t lane = (uint32_t)(warp * 32) << 16;  // this warp's 32 TMEM lanes
    const int vis = tid < nr ? L + (r0 + tid) % p.T_new + 1 : 0;  // positions [0, vis)
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
#pragma unroll 1
    for (int j = 0; j < ntiles; ++j) {
      const int buf = j & 1;
      const uint32_t tS = tmem + buf * 64 + lane;
      // tcgen05.ld / st are warp-collective: a warp goes on only as a whole
      ok = __all_sync(0xffffffffu, wait(&s_full[buf], (j >> 1) & 1));
      if (!ok) break;
      tc_fence_after();
      float2 sc[32];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_ld16(tS + c4 * 16, reinterpret_cast<float*>(sc) + c4 * 16);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; ++c) sc[c] = __fmul2_rn(sc[c], sc2);
      const int t0 = sp.real(t_begin + j * C::kTile);
      if (!tile_fully_visible(t0, C::kTile, vis_min, n_blk, p.window, p.sink)) {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (!visible(t0 + 2 * c, vis, p.window, p.sink)) sc[c].x = -INFINITY;
          if (!visible(t0 + 2 * c + 1, vis, p.window, p.sink)) sc[c].y = -INFINITY;
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 32; ++c) mx = fmaxf(mx, fmaxf(sc[c].x, sc[c].y));
      // Move the reference max when the tile's max passes it by 2^8 and rescale
      // this row of O (before any visible token the row is all zero: alpha 1).
      const bool move = mx > m_ref + 8.f;
      const float alpha = (move && m_ref != -INFINITY) ? ex2_approx(m_ref - mx) : 1.f;
      if (__any_sync(0xffffffffu, alpha != 1.f)) {  // the warp's 32 rows together
        // O must hold P(j-1).V(j-1) first
        ok = __all_sync(0xffffffffu, wait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1));
        if (!ok) break;
        tc_fence_after();
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
      const float2 mu2 = make_float2(-mu, -mu);
      uint32_t ph[32];
      float2 lsum = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float2 e = __fadd2_rn(sc[c], mu2);
        const float2 pp = make_float2(ex2_approx(e.x), ex2_approx(e.y));
        lsum = __fadd2_rn(lsum, pp);
        ph[c] = Elt<T>::pack2(pp.x, pp.y);
        if constexpr (kSplitP)  // keep the rounding remainder in sc[] for P_lo
          sc[c] = __fadd2_rn(pp, make_float2(-__uint_as_float(ph[c] << 16),
                                             -__uint_as_float(ph[c] & 0xFFFF0000u)));
      }
      l += lsum.x + lsum.y;
      // P over this row's scores: 64 tokens in 32 columns (even token low half)
      tmem_st16(tS, ph);
      tmem_st16(tS + 16, ph + 16);
      if constexpr (kSplitP) {
        uint32_t pl[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pl[c] = Elt<T>::pack2(sc[c].x, sc[c].y);
        tmem_st16(tS + 32, pl);
        tmem_st16(tS + 48, pl + 16);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[buf]);
    }
    if (ok && ntiles > 0)
      ok = __all_sync(0xffffffffu,
                      wait(&o_done[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1));
  }

  const bool bad = __syncthreads_or(*abort_word != 0);
  if (bad) {
    if ((warp == C::kKWarp || warp == C::kVWarp) && lane_id == 0) {  // loads in flight
      const int NS = warp == C::kKWarp ? SK : SV;
      uint64_t* full = warp == C::kKWarp ? k_full : v_full;
      for (int j = max(0, issued - NS); j < issued; ++j)
        if (!mbar_wait(&full[j % NS], (j / NS) & 1, p.err, wait_limit)) break;
    }
    if (warp == C::kMmaWarp && lane_id == 0 && mma_issued) {  // MMAs still in flight
      umma_commit(dbar);
      mbar_wait(dbar, 0, p.err, wait_limit);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(C::kTmemCols)
                   : "memory");
    return;
  }
  if (warp >= C::kMmaWarp) return;  // producers and MMA issuer are done

  // ---- this row's unnormalised O, reference max and sum to shared memory (every
  // MMA and load has completed: the ring and Q are idle)
  tc_fence_after();
  red_m[tid] = m_ref;
  red_l[tid] = l;
  {
    const uint32_t lane = (uint32_t)(warp * 32) << 16;
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
  }
  tc_fence_before();
  named_barrier_sync(1, NSM);
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::kTmemCols)
                 : "memory");
  finish_slice<T, D, R, 1, NSM, C::kAccLd>(p, red_acc, red_m, red_l, scratch, &flags[1], b, g,
                                           rb, s, r0, nr, L, ns_blk, sp);
}

}  // namespace kvc
