// attend_tc_streamk.cuh -- N2 + N3 (tcgen05, persistent): stream-K split attention for
// 17 or more query rows per KV head (MQA verify chunks, large GQA groups, chunked prefill).
//
// The per-tile arithmetic is that of attend_tc.cuh (S = Q.K^T and O += P.V on tcgen05
// with fp32 accumulators in TMEM, one softmax thread per query row, lazy rescaling,
// bf16 weights split in two); the work is organised as in attend_streamk.cuh:
//
// * Segments are (request b, KV head g, 128-row block rb) in that order, each of
//   ceil((L_b + i_max + 1) / 64) tiles, preceded by `sk_penalty` virtual tiles that
//   charge the fixed cost of a piece (Q reload, TMEM readout, partial write, ticket)
//   to the CTA that pays it.  The G persistent CTAs (G = SMs x 2, TMEM-bound) take equal
//   contiguous ranges of the virtual tiles, so every CTA does the same work whatever
//   the mix of lengths, and none waits for a second wave.
// * TMEM is allocated once per CTA and the K and V rings stream across piece
//   boundaries: the producers walk the range without stopping; at a piece end the
//   softmax threads read the row's O out of TMEM, stage the next piece's Q, and only
//   then write the piece's result, so the MMA issuer starts the next piece at once.
// * A piece that covers its whole segment writes the output rows directly; otherwise
//   it writes a normalised partial (o / l, base-2 log-sum-exp) to one of its CTA's two
//   workspace slots and takes a release-acquire ticket; the segment's last finisher
//   merges the pieces by log-sum-exp ("9. 推理" 9.7: exact up to rounding), or, when the
//   plan's segments carry large partials (p.sk_combine), leaves a descriptor for the
//   dependent combine_kernel launch, which merges them over many CTAs.
// * The range is planned before the dependency wait (shared memory only) and checked
//   against the lengths after it; it is planned again if any changed.
// * With k_new / v_new (kvc_append_attend) the K and V copy warps store a tile's new
//   rows into the pool before its TMA copy reads them (the append, fused).
//
// Roles (224 threads): warps 0-3 softmax (thread t = TMEM lane t = query row t of the
// block; they also load Q and run the epilogue and the merge), warp 4 lane 0 issues the
// MMAs, warps 5 and 6 load K and V tiles with TMA (no multicast).  Every wait is bounded;
// after a wait runs out the softmax threads keep one control path (they meet at named
// barriers), the other roles stop, and the CTA drains its copies and MMAs and frees its
// TMEM before it exits.
#pragma once

#include <cuda.h>
#include <math.h>

#include "attend_streamk.cuh"
#include "attend_tc.cuh"
#include "device_common.cuh"
#include "params.cuh"

namespace kvc {

// ints of a segment's combine descriptor (in the workspace after the lse values):
// generation, valid rows, first range, pieces, first piece in its range's second slot,
// output row (2 ints), pad
constexpr int kCombineDescInts = 8;

template <int D>
struct TcSkCfg {
  using C = TcCfg<D>;
  // K full/empty, V full/empty, s_full x2, p_full x2, o_done x2, q_full, drain
  static constexpr int kBarriers = 2 * C::kKStages + 2 * C::kVStages + 8;
  // after the barriers: the TMEM slot (16 bytes), then 32 ints of flags: [0] abort,
  // [1] last finisher, [2] final merge pending, [4..7] two merge mbarriers, [8..14] scan
  // sums, [16..23] the final merge's parameters
  static constexpr size_t smem_bytes() {
    return C::kData + kBarriers * sizeof(uint64_t) + 16 + 32 * sizeof(int);
  }
  // the final merge's weights: up to kMergeMaxPieces pieces of 128 rows at the end of the
  // operand area; the rest holds two windows of partial rows
  static constexpr int kMergeMaxPieces = 32;
  static constexpr int kMergeWeightBytes = C::kRows * kMergeMaxPieces * (int)sizeof(float);
  static constexpr int kMergeHalf = ((C::kData - kMergeWeightBytes) / 2) & ~15;
  // the plan's scan (tile prefix and lengths, 2B + 1 ints) uses the K/V rings before any copy
  static constexpr int kMaxBatch = ((C::kKRing + C::kVRing) / (int)sizeof(int) - 1) / 2;
};

// This CTA's share of the stream-K range: the segments are those of attend_streamk.cuh
// with R query rows per segment.
template <int R>
struct SkRange {
  bool work;
  long long Wt, lo, hi;
  int G, ntiles;  // CTAs with work (the grid may be larger), real tiles of this range
  TileCursor<R> cur;
};

// Mixes one length into a thread's digest of the lengths it scanned.
__device__ __forceinline__ uint32_t len_mix(uint32_t h, int L) {
  return (h ^ (uint32_t)L) * 0x9E3779B1u + 0x7F4A7C15u;
}

// Plans this CTA's range from seq_lens with a block scan over the requests; every one of
// the NTH threads calls it.  P and Ls: 2B + 1 ints of shared memory, wsum: NTH/32 ints.
// Lengths outside the cache contribute no tiles (and flag KVC_ERR_BOUNDS when
// `authoritative`); `digest` receives this thread's digest of the lengths it read
// (requests tid * ceil(B / NTH) onwards).
template <int R, int NTH, bool PAGED>
__device__ __forceinline__ SkRange<R> sk_plan(const AttendParams& p, int* P, int* Ls, int* wsum,
                                              bool authoritative, uint32_t& digest) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = ceil_div(p.B, NTH);
  const int b_lo = min(p.B, tid * per), b_hi = min(p.B, b_lo + per);
  int sum = 0;
  digest = 0;
  for (int b = b_lo; b < b_hi; ++b) {
    const int L = p.seq_lens[b];
    digest = len_mix(digest, L);
    Ls[b] = L;
    int t = 0;
    if (length_ok(p, L, PAGED)) t = request_tiles<R>(p, L);
    else if (authoritative) flag_error(p.err, KVC_ERR_BOUNDS);
    P[b] = t;
    sum += t;
  }
  int incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += wsum[w];
  int run = base + incl - sum;
  for (int b = b_lo; b < b_hi; ++b) {
    const int t = P[b];
    P[b] = run;
    run += t;
  }
  if (tid == NTH - 1) P[p.B] = base + incl;
  __syncthreads();
  SkRange<R> r{};
  // row-block major: P covers one row block, repeated row_blocks times
  const long long W1 = P[p.B];
  r.Wt = p.sk_rb_major ? W1 * p.row_blocks : W1;
  r.G = (int)(r.Wt < (long long)gridDim.x ? r.Wt : (long long)gridDim.x);
  const int c = blockIdx.x;
  r.work = c < r.G;
  if (r.work) {
    r.lo = (long long)c * r.Wt / r.G;
    r.hi = (long long)(c + 1) * r.Wt / r.G;
    const int rb0 = p.sk_rb_major ? (int)(r.lo / W1) : 0;
    const long long lo1 = r.lo - rb0 * W1;  // the position within the row block's part
    int a = 0, z = p.B;  // largest b with P[b] <= lo1
    while (z - a > 1) {
      const int mid = (a + z) >> 1;
      if (P[mid] <= lo1) a = mid;
      else z = mid;
    }
    while (P[a + 1] == P[a]) ++a;  // requests with no tiles
    TileCursor<R>& cur = r.cur;
    cur.b = a;
    cur.L = Ls[a];
    int local = (int)(lo1 - P[a]);
    const int per_g = (P[a + 1] - P[a]) / p.H_kv;
    cur.g = local / per_g;
    local -= cur.g * per_g;
    cur.rb = rb0;  // row-block major: the (b, g) segment of this block; else the first
    while (true) {
      const int t = ceil_div(cur.L + row_block(cur.rb, R, p.rows, p.T_new).imax + 1, 64);
      if (local < t + p.sk_penalty || cur.rb == p.row_blocks - 1) {
        cur.seg_tiles = t;
        break;
      }
      local -= t + p.sk_penalty;
      ++cur.rb;
    }
    cur.seg_start = r.lo - local + p.sk_penalty;
    cur.k = max(0, local - p.sk_penalty);
    r.ntiles = 0;
    TileCursor<R> w = cur;
#pragma unroll 1
    while (w.b < p.B) {
      const long long v = w.seg_start + w.k;
      if (v >= r.hi) break;
      const long long seg_end = w.seg_start + w.seg_tiles;
      const long long stop = r.hi < seg_end ? r.hi : seg_end;
      r.ntiles += (int)(stop - v);
      if (stop < seg_end) break;
      w.k = w.seg_tiles - 1;
      w.next(p, PAGED, Ls);
    }
    r.work = r.ntiles > 0;
  }
  __syncthreads();  // P and Ls are dead: the rings may be filled
  return r;
}

// The last finisher's merge of a segment's pieces rf..rl at the end of its range, by all
// of the CTA's threads, with the operand area (`smem`, TcCfg<D>::kData bytes) free:
//   1. every (row, piece) weight 2^(lse - M) / sum, once, into the area's last bytes;
//   2. the pieces' partial rows streamed through two shared-memory windows of bulk copies
//      (each window RC rows of every piece), the next window loading while this one is
//      summed.
// More pieces than the weight area holds fall back to merge_pieces_spread.  Waits are
// bounded; after one runs out the merge finishes on garbage and KVC_ERR_TIMEOUT stands.
template <typename T, int D>
__device__ __forceinline__ void tc_merge_final(const AttendParams& p, const RangeMap& rm,
                                               long long rf, long long rl, long long s0, int nr,
                                               size_t row_base, unsigned char* smem,
                                               uint64_t* mbar, unsigned long long wait_limit) {
  using C = TcCfg<D>;
  using S = TcSkCfg<D>;
  constexpr int R = C::kRows;
  constexpr int NTH = C::kThreads;
  constexpr int Q4 = D / 4;
  const int tid = threadIdx.x;
  const int npc = (int)(rl - rf + 1);
  if (npc > S::kMergeMaxPieces) {
    merge_pieces_spread<T, D, R, NTH>(p, rm, rf, rl, s0, nr, row_base);
    return;
  }
  const bool rf_mid = rm.start(rf) < s0 - p.sk_penalty;
  auto slot_of = [&](int q) -> size_t {
    return (size_t)(rf + q) * 2 + ((q == 0 && rf_mid) ? 1 : 0);
  };
  float* w = reinterpret_cast<float*>(smem + C::kData - S::kMergeWeightBytes);  // [row][piece]
  // 1. weights
#pragma unroll 1
  for (int idx = tid; idx < nr * npc; idx += NTH) {
    const int rr = idx / npc, q = idx - rr * npc;
    w[idx] = __ldcg(p.ws_lse + slot_of(q) * p.sk_slot_rows + rr);
  }
  __syncthreads();
  if (tid < nr) {
    float* wr = w + tid * npc;
    float M = -INFINITY;
    for (int q = 0; q < npc; ++q) M = fmaxf(M, wr[q]);
    float den = 0.f;
    for (int q = 0; q < npc; ++q) {
      wr[q] = wr[q] == -INFINITY ? 0.f : exp2f(wr[q] - M);
      den += wr[q];
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    for (int q = 0; q < npc; ++q) wr[q] *= inv;
  }
  // 2. the partial rows, RC rows of every piece per window
  const int RC = min(nr, S::kMergeHalf / (npc * D * (int)sizeof(float)));
  const int nwin = ceil_div(nr, RC);
  auto issue = [&](int win) {  // thread 0
    const int half = win & 1;
    const int r0 = win * RC;
    const uint32_t bytes = (uint32_t)min(RC, nr - r0) * D * sizeof(float);
    mbar_arrive_expect_tx(&mbar[half], bytes * npc);
    for (int q = 0; q < npc; ++q)
      bulk_g2s(smem + half * S::kMergeHalf + (size_t)q * RC * D * sizeof(float),
               p.ws_o + (slot_of(q) * p.sk_slot_rows + r0) * D, bytes, &mbar[half]);
  };
  if (tid == 0) {
    // the partials were written by other CTAs through the generic proxy and acquired by
    // the ticket: order them before the bulk copies' async-proxy reads
    asm volatile("fence.proxy.async.global;" ::: "memory");
    issue(0);
    if (nwin > 1) issue(1);
  }
  __syncthreads();  // the weights are complete
  T* out = static_cast<T*>(p.out);
#pragma unroll 1
  for (int win = 0; win < nwin; ++win) {
    const int half = win & 1;
    const int r0 = win * RC;
    const int rows = min(RC, nr - r0);
    mbar_wait(&mbar[half], (win >> 1) & 1, p.err, wait_limit);
    const float* buf = reinterpret_cast<const float*>(smem + half * S::kMergeHalf);
#pragma unroll 1
    for (int e = tid; e < rows * Q4; e += NTH) {
      const int rr = e / Q4;
      const int d = (e - rr * Q4) * 4;
      const float* wr = w + (r0 + rr) * npc;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
      for (int q = 0; q < npc; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(buf + ((size_t)q * RC + rr) * D + d);
        const float wq = wr[q];
        a.x = fmaf(wq, v.x, a.x);
        a.y = fmaf(wq, v.y, a.y);
        a.z = fmaf(wq, v.z, a.z);
        a.w = fmaf(wq, v.w, a.w);
      }
      T* o = out + (row_base + r0 + rr) * D + d;
      const uint2 packed = make_uint2(Elt<T>::pack2(a.x, a.y), Elt<T>::pack2(a.z, a.w));
      *reinterpret_cast<uint2*>(o) = packed;
    }
    __syncthreads();  // the window is read: it may be refilled
    if (tid == 0 && win + 2 < nwin) issue(win + 2);
  }
}

// Combine launch (after attend_tc_streamk_kernel with p.sk_combine != 0): block
// (segment, chunk of KVC_TC_COMBINE_ROWS rows) merges that chunk of the segment's pieces
// by log-sum-exp ("9. 推理" 9.7) with merge_rows_spread.  A segment whose descriptor does
// not carry this call's generation was written whole (or has no tiles) and is skipped.
// Launched dependently: it waits for the attend grid before reading anything.  Small
// chunks keep each thread's chain of dependent partial loads short (4 rows: one quad of
// one row a thread, about nine pieces in three rounds of four loads; 16 rows took four
// such items in sequence: gamma 4 MQA verify 0.216 -> 0.185 ms a step).
#ifndef KVC_TC_COMBINE_ROWS
#define KVC_TC_COMBINE_ROWS 4
#endif
constexpr int kCombineRows = KVC_TC_COMBINE_ROWS;
template <typename T, int D>
__global__ void __launch_bounds__(128) combine_kernel(const AttendParams p) {
  griddep_launch_dependents();
  griddep_wait();
  const size_t segi = blockIdx.x;
  const int* d = p.sk_desc + segi * kCombineDescInts;
  if (d[0] != p.sk_combine) return;
  const int nr = d[1];
  const int r_off = blockIdx.y * kCombineRows;
  if (r_off >= nr) return;
  const size_t row_base = (size_t)(uint32_t)d[5] | ((size_t)(uint32_t)d[6] << 32);
  merge_rows_spread<T, D, 128>(p, d[2], d[3], d[4] != 0, r_off, min(kCombineRows, nr - r_off),
                               row_base);
}

template <int D, typename T, bool PAGED>
__global__ void __launch_bounds__(TcCfg<D>::kThreads, 2)
    attend_tc_streamk_kernel(const AttendParams p, const __grid_constant__ CUtensorMap tmk,
                             const __grid_constant__ CUtensorMap tmv) {
  using C = TcCfg<D>;
  constexpr int R = C::kRows;
  constexpr int NSM = C::kSoftmaxThreads;
  constexpr int SK = C::kKStages;
  constexpr int SV = C::kVStages;
  constexpr bool kSplitP = Elt<T>::kCode == KVC_BF16;
  extern __shared__ __align__(1024) unsigned char tc_smem[];
  unsigned char* const smem = tc_smem;
  unsigned char* sk = smem;              // K stages
  unsigned char* sv = smem + C::kKRing;  // V stages
  unsigned char* sq = sv + C::kVRing;    // Q of the current piece
  uint64_t* k_full = reinterpret_cast<uint64_t*>(smem + C::kData);
  uint64_t* k_empty = k_full + SK;
  uint64_t* v_full = k_empty + SK;
  uint64_t* v_empty = v_full + SV;
  uint64_t* s_full = v_empty + SV;  // [2]
  uint64_t* p_full = s_full + 2;    // [2] (NSM arrivals)
  uint64_t* o_done = p_full + 2;    // [2] P(j).V(j) done on o_done[j & 1] (attend_tc.cuh)
  uint64_t* q_full = o_done + 2;    // a piece's Q is staged (NSM arrivals; O was read)
  uint64_t* dbar = q_full + 1;      // drain after an abort
  uint32_t* tslot = reinterpret_cast<uint32_t*>(dbar + 1);
  int* flags = reinterpret_cast<int*>(tslot + 4);  // see TcSkCfg::smem_bytes
  uint64_t* mbar = reinterpret_cast<uint64_t*>(flags + 4);      // [2] final merge windows
  long long* fm = reinterpret_cast<long long*>(flags + 16);     // final merge parameters

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane_id = tid & 31;
  if (smem_addr(smem) & 1023u) {  // swizzle atoms need 1024-byte alignment
    if (tid == 0) flag_error(p.err, KVC_ERR_UNSUPPORTED);
    return;
  }
  griddep_launch_dependents();
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
    mbar_init(q_full, NSM);
    mbar_init(dbar, 1);
    flags[0] = 0;
    flags[1] = 0;
    flags[2] = 0;
    mbar_init(&mbar[0], 1);
    mbar_init(&mbar[1], 1);
    fence_barrier_init();
  }
  tc_fence_before();
  // Plan from the lengths as they stand while the grid ahead finishes (shared memory
  // only); after the dependency wait every thread reads the lengths it scanned again and
  // the block plans once more if any changed (or a test asked for it: p.replan).
  int* Pscan = reinterpret_cast<int*>(smem);
  SkRange<R> rg;
#pragma unroll 1
  for (int pass = 0;; ++pass) {  // pass 0 before the wait, pass 1 only if it was stale
    uint32_t digest;
    rg = sk_plan<R, C::kThreads, PAGED>(p, Pscan, Pscan + p.B + 1, flags + 8, pass > 0, digest);
    if (pass > 0) break;
    griddep_wait();
    const int per = ceil_div(p.B, C::kThreads);
    const int b_lo = min(p.B, tid * per), b_hi = min(p.B, b_lo + per);
    uint32_t h = 0;
    for (int b = b_lo; b < b_hi; ++b) {
      const int L = p.seq_lens[b];
      h = len_mix(h, L);
      if (!length_ok(p, L, PAGED)) flag_error(p.err, KVC_ERR_BOUNDS);
    }
    if (!__syncthreads_or(h != digest || p.replan != 0)) break;
  }
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t tO = tmem + C::kOCol;
  if (!rg.work) {
    if (warp == 0)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(C::kTmemCols)
                   : "memory");
    return;
  }

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

  int issued = 0;           // producers: tiles whose loads were issued
  bool mma_issued = false;  // MMA lane

  if (warp == C::kKWarp || warp == C::kVWarp) {
    // ---- TMA producers (no multicast): warp 5 loads K, warp 6 loads V, each walking the
    // range with its own cursor; lane k loads box k of a paged tile
    const bool is_k = warp == C::kKWarp;
    const int NS = is_k ? SK : SV;
    unsigned char* ring = is_k ? sk : sv;
    uint64_t* full = is_k ? k_full : v_full;
    uint64_t* empty = is_k ? k_empty : v_empty;
    const CUtensorMap* tm = is_k ? &tmk : &tmv;
    const uint64_t pol = p.row_blocks > 1 ? l2_policy_evict_normal() : l2_policy_evict_first();
    if (lane_id == 0) prefetch_tmap(tm);
    const int Pg = PAGED ? (1 << p.page_shift) : C::kTile;
    const int box_rows = Pg < C::kTile ? Pg : C::kTile;
    const int nbox = C::kTile / box_rows;  // <= 8 (pages of 8 or more tokens)
    const int beyond = p.num_pages * p.H_kv * Pg;  // first row past the pool: zero fill
    // row of this lane's box in the tile under cursor cc: past the segment, or a page id
    // outside the pool (flagged), the row past the pool (zero fill)
    auto box_y = [&](const TileCursor<R>& cc) -> int {
      const int t = cc.k * C::kTile + lane_id * box_rows;
      if (t >= cc.L + row_block(cc.rb, R, p.rows, p.T_new).imax + 1) return beyond;
      const int page = p.block_table[(size_t)cc.b * p.max_pages + (t >> p.page_shift)];
      if (page >= 0 && page < p.num_pages) return (page * p.H_kv + cc.g) * Pg + (t & (Pg - 1));
      flag_error(p.err, KVC_ERR_BOUNDS);
      return beyond;
    };
    TileCursor<R> pc = rg.cur;
#pragma unroll 1
    for (int j = 0; j < rg.ntiles && !p.stall; ++j) {  // a stall (test) issues nothing
      const int st = j % NS;
      if (j >= NS) {
        bool w = true;
        if (lane_id == 0) w = wait(&empty[st], ((j / NS) - 1) & 1);
        if (!__shfl_sync(0xffffffffu, w, 0)) break;
      }
      unsigned char* dst = ring + st * C::kTileBytes;
      const int t0 = pc.k * C::kTile;
      if (p.k_new != nullptr) {
        // Fused append: the new positions of this tile go into the pool (this warp's K
        // or V) before its copy reads them.  Every CTA that loads such a tile writes them
        // (the row blocks of a segment write the same bytes), after the dependency wait;
        // each lane's proxy fence, then the warp barrier, order the stores before the
        // copies' async-proxy reads.
        const int n_lo = max(pc.L, t0), n_hi = min(pc.L + p.T_new, t0 + C::kTile);
        if (n_lo < n_hi) {  // the same decision in every lane
          constexpr int CH = D / 8;  // 16-byte chunks a row
          const char* src = static_cast<const char*>(is_k ? p.k_new : p.v_new);
          char* pool = static_cast<char*>(const_cast<void*>(is_k ? p.k_pool : p.v_pool));
#pragma unroll 1
          for (int idx = lane_id; idx < (n_hi - n_lo) * CH; idx += 32) {
            const int rr = idx / CH;
            const int ch = idx - rr * CH;
            const int pos = n_lo + rr;
            long long row;
            if (PAGED) {
              const int page = p.block_table[(size_t)pc.b * p.max_pages + (pos >> p.page_shift)];
              if (page < 0 || page >= p.num_pages) {
                flag_error(p.err, KVC_ERR_BOUNDS);
                continue;
              }
              row = ((long long)page * p.H_kv + pc.g) * Pg + (pos & (Pg - 1));
            } else {
              row = ((long long)pc.b * p.H_kv + pc.g) * p.max_T + pos;
            }
            const size_t s_off =
                ((((size_t)pc.b * p.H_kv + pc.g) * p.T_new + (pos - pc.L)) * D + ch * 8) *
                sizeof(T);
            st_global_v4(pool + (row * D + ch * 8) * (long long)sizeof(T),
                         ld_global_nc_v4(src + s_off));
          }
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
      }
      if (lane_id == 0) mbar_arrive_expect_tx(&full[st], C::kTileBytes);
      __syncwarp();
      if (!PAGED) {
        if (lane_id < C::kHalves)
          tma_load_2d(dst + lane_id * C::kBoxBytes, tm, lane_id * 64,
                      (pc.b * p.H_kv + pc.g) * p.max_T + t0, &full[st], pol);
      } else if (lane_id < nbox) {
        const int y = box_y(pc);
        const int off = lane_id * box_rows * 128;
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h)
          tma_load_2d(dst + h * C::kBoxBytes + off, tm, h * 64, y, &full[st], pol);
      }
      ++issued;
      pc.next(p, PAGED);
    }
  } else if (warp == C::kMmaWarp) {
    // ---- MMA issuer: S(j+1) ahead of P(j).V(j) within a piece; S buffer j&1 holds S(j),
    // then P(j).  A piece's first S waits for its Q (q_full, which the softmax threads
    // arrive on only after reading the previous piece's O, so O may then be overwritten).
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
      TileCursor<R> mc = rg.cur;
      int piece = 0;
      bool ok = wait(q_full, 0);
      if (ok) {
        tc_fence_after();
        ok = issue_s(0);
      }
#pragma unroll 1
      for (int j = 0; ok && j < rg.ntiles; ++j) {
        const bool first = (j == 0) || (mc.k == 0);
        const bool last = (j == rg.ntiles - 1) || (mc.k == mc.seg_tiles - 1);
        if (j + 1 < rg.ntiles && !last) {
          // buffer (j+1)&1 still holds P(j-1) until its P.V MMA is done
          if (j >= 1 && !wait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1)) break;
          if (!issue_s(j + 1)) break;
        }
        const int st = j % SV;
        if (!wait(&p_full[j & 1], (j >> 1) & 1) || !wait(&v_full[st], (j / SV) & 1)) break;
        tc_fence_after();
        const uint32_t tP = tmem + (j & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < C::kTile / 16; ++kk) {
          const uint64_t bv =
              umma_desc_sw128(sv_a + st * C::kTileBytes + kk * 2048, C::kBoxBytes, 1024);
          umma_f16_tmem_a(tO, tP + kk * 8, bv, idesc_o, !first || kk > 0);
          if constexpr (kSplitP) umma_f16_tmem_a(tO, tP + 32 + kk * 8, bv, idesc_o, true);
        }
        umma_commit(&v_empty[st]);
        umma_commit(&o_done[j & 1]);
        if (j + 1 < rg.ntiles && last) {  // the next piece starts once its Q is staged
          ++piece;
          if (!wait(q_full, piece & 1)) break;
          tc_fence_after();
          if (!issue_s(j + 1)) break;
        }
        mc.next(p, PAGED);
      }
    }
    __syncwarp();
  } else {
    // ---- softmax, epilogue and merge: thread tid owns query row tid (TMEM lane tid)
    const uint32_t lane = (uint32_t)(warp * 32) << 16;  // this warp's 32 TMEM lanes
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
    const int c = blockIdx.x;
    RangeMap rm;
    rm.W = rg.Wt;
    rm.G = rg.G;
    T* out = static_cast<T*>(p.out);
    TileCursor<R> sc = rg.cur;
    float m_ref = -INFINITY;  // the row's reference max (base 2) and
    float l = 0.f;            // sum of 2^(s - m_ref)
    int vis = 0, vis_min = 0, r0 = 0, nr = 0, piece_first_j = 0;
    // Q of the piece under cursor qc: row tid in 64-element boxes, 128-byte swizzled
    auto stage_q = [&](const TileCursor<R>& qc) {
      const int qr0 = qc.rb * R;
      const int qnr = min(R, p.rows - qr0);
      const char* qrow =
          static_cast<const char*>(p.q) +
          ((((size_t)qc.b * p.H_q + (size_t)qc.g * p.group) * p.T_new) + qr0 + tid) * D * 2;
#pragma unroll
      for (int ch = 0; ch < D / 8; ++ch) {
        const uint4 v = tid < qnr ? ld_global_nc_v4(qrow + ch * 16) : make_uint4(0, 0, 0, 0);
        st_shared_v4(sq + (ch >> 3) * C::kQBox + tid * 128 + (((ch & 7) ^ (tid & 7)) << 4), v);
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(q_full);
    };
    stage_q(sc);
    // After a wait runs out every softmax thread still walks all tiles (on garbage) so
    // that the named barriers of the epilogue are always met.
#pragma unroll 1
    for (int j = 0; j < rg.ntiles; ++j) {
      const bool first = (j == 0) || (sc.k == 0);
      const bool last = (j == rg.ntiles - 1) || (sc.k == sc.seg_tiles - 1);
      if (first) {  // a new piece: the row's visible length, fresh running state
        piece_first_j = j;
        r0 = sc.rb * R;
        nr = min(R, p.rows - r0);
        vis = tid < nr ? sc.L + (r0 + tid) % p.T_new + 1 : 0;
        vis_min = sc.L + row_block(sc.rb, R, p.rows, p.T_new).imin + 1;
        m_ref = -INFINITY;
        l = 0.f;
      }
      const int buf = j & 1;
      const uint32_t tS = tmem + buf * 64 + lane;
      // tcgen05.ld / st are warp-collective: a warp goes on only as a whole
      __all_sync(0xffffffffu, wait(&s_full[buf], (j >> 1) & 1));
      tc_fence_after();
      float2 sv2[32];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4)
        tmem_ld16(tS + c4 * 16, reinterpret_cast<float*>(sv2) + c4 * 16);
      tmem_wait_ld();
#pragma unroll
      for (int cc = 0; cc < 32; ++cc) sv2[cc] = __fmul2_rn(sv2[cc], sc2);
      const int t0 = sc.k * C::kTile;
      if (t0 + C::kTile > vis_min) {  // some row of the block does not see the whole tile
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) {
          if (t0 + 2 * cc >= vis) sv2[cc].x = -INFINITY;
          if (t0 + 2 * cc + 1 >= vis) sv2[cc].y = -INFINITY;
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int cc = 0; cc < 32; ++cc) mx = fmaxf(mx, fmaxf(sv2[cc].x, sv2[cc].y));
      // Move the reference max when the tile's max passes it by 2^8 and rescale this row
      // of O (the first tile of a piece starts from -inf: nothing to rescale).
      const bool move = mx > m_ref + 8.f;
      const float alpha = (move && m_ref != -INFINITY) ? ex2_approx(m_ref - mx) : 1.f;
      if (__any_sync(0xffffffffu, alpha != 1.f)) {  // the warp's 32 rows together
        // O holds P(j-1).V(j-1)
        __all_sync(0xffffffffu, wait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1));
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
      for (int cc = 0; cc < 32; ++cc) {
        const float2 e = __fadd2_rn(sv2[cc], mu2);
        const float2 pp = make_float2(ex2_approx(e.x), ex2_approx(e.y));
        lsum = __fadd2_rn(lsum, pp);
        ph[cc] = Elt<T>::pack2(pp.x, pp.y);
        if constexpr (kSplitP)  // keep the rounding remainder in sv2[] for P_lo
          sv2[cc] = __fadd2_rn(pp, make_float2(-__uint_as_float(ph[cc] << 16),
                                               -__uint_as_float(ph[cc] & 0xFFFF0000u)));
      }
      l += lsum.x + lsum.y;
      tmem_st16(tS, ph);  // P over this row's scores: 64 tokens in 32 columns
      tmem_st16(tS + 16, ph + 16);
      if constexpr (kSplitP) {
        uint32_t plo[32];
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) plo[cc] = Elt<T>::pack2(sv2[cc].x, sv2[cc].y);
        tmem_st16(tS + 32, plo);
        tmem_st16(tS + 48, plo + 16);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[buf]);

      if (last) {  // ---- end of a piece: the row's result, the next Q, the ticket
        // P.V(j) done implies every earlier MMA of the piece is (tcgen05.commit tracks all
        // of the issuing thread's prior MMAs)
        __all_sync(0xffffffffu, wait(&o_done[j & 1], (j >> 1) & 1));
        tc_fence_after();
        const bool whole = (piece_first_j == j - sc.k) && (sc.k == sc.seg_tiles - 1);
        const int slot = (piece_first_j == 0) ? 0 : 1;
        const size_t row_base =
            ((size_t)sc.b * p.H_q + (size_t)sc.g * p.group) * p.T_new + r0;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        float* wso = p.ws_o + (((size_t)c * 2 + slot) * p.sk_slot_rows + tid) * D;
        T* orow = out + (row_base + tid) * D;
#pragma unroll 1
        for (int c16 = 0; c16 < D / 16; ++c16) {
          float ov[16];
          tmem_ld16(tO + lane + c16 * 16, ov);
          tmem_wait_ld();
          if (tid < nr) {
            if (whole) {
              uint32_t w[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) w[i] = Elt<T>::pack2(ov[2 * i] * inv, ov[2 * i + 1] * inv);
              st_global_v4(orow + c16 * 16, make_uint4(w[0], w[1], w[2], w[3]));
              st_global_v4(orow + c16 * 16 + 8, make_uint4(w[4], w[5], w[6], w[7]));
            } else {
#pragma unroll
              for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<float4*>(wso + c16 * 16 + i) =
                    make_float4(ov[i] * inv, ov[i + 1] * inv, ov[i + 2] * inv, ov[i + 3] * inv);
            }
          }
        }
        if (!whole && tid < nr)
          p.ws_lse[((size_t)c * 2 + slot) * p.sk_slot_rows + tid] =
              l > 0.f ? m_ref + log2f(l) : -INFINITY;
        // The row's O is read: staging the next piece's Q hands TMEM back to the MMA issuer.
        if (j + 1 < rg.ntiles) {
          TileCursor<R> nc = sc;
          nc.next(p, PAGED);
          stage_q(nc);
        }
        if (!whole && p.sk_combine) {
          // a combine launch merges the segment: the piece holding its first tile leaves
          // the descriptor (read only after this grid has completed)
          if (tid == 0 && piece_first_j == j - sc.k) {
            const long long s0 = sc.seg_start, s1 = sc.seg_start + sc.seg_tiles - 1;
            const long long rf = rm.of(s0), rl = rm.of(s1);
            const size_t segi = ((size_t)sc.b * p.H_kv + sc.g) * p.row_blocks + sc.rb;
            int* d = p.sk_desc + segi * kCombineDescInts;
            d[1] = nr;
            d[2] = (int)rf;
            d[3] = (int)(rl - rf + 1);
            d[4] = rm.start(rf) < s0 - p.sk_penalty ? 1 : 0;
            d[5] = (int)(row_base & 0xffffffffu);
            d[6] = (int)(row_base >> 32);
            d[0] = p.sk_combine;
          }
        } else if (!whole) {
          // hand the piece to the segment's last finisher: the barrier orders every
          // row's partial stores before thread 0's release-acquire ticket
          named_barrier_sync(1, NSM);
          const long long s0 = sc.seg_start, s1 = sc.seg_start + sc.seg_tiles - 1;
          const long long rf = rm.of(s0), rl = rm.of(s1);
          int* ticket = p.counters + ((size_t)sc.b * p.H_kv + sc.g) * p.row_blocks + sc.rb;
          if (tid == 0) flags[1] = ticket_add_acq_rel(ticket) == (int)(rl - rf);
          named_barrier_sync(1, NSM);
          if (j + 1 < rg.ntiles) {  // mid-range: the softmax threads merge at once
            if (flags[1]) {
              merge_pieces_spread<T, D, R, NSM>(p, rm, rf, rl, s0, nr, row_base);
              if (tid == 0) *ticket = 0;
            }
            named_barrier_sync(1, NSM);  // flags[1] is read by every thread before reuse
          } else if (tid == 0 && flags[1]) {
            // the range's last piece: every thread of the CTA merges after the loops, with
            // the operand area free for staging (tc_merge_final)
            flags[2] = 1;
            fm[0] = s0;
            fm[1] = (long long)row_base;
            fm[2] = rf | (rl << 32);
            fm[3] = nr | ((long long)(ticket - p.counters) << 32);
          }
        }
      }
      sc.next(p, PAGED);
    }
  }

  const bool bad = __syncthreads_or(*abort_word != 0);
  if (!bad && flags[2]) {  // every copy and MMA has completed: the operand area is free
    RangeMap frm;
    frm.W = rg.Wt;
    frm.G = rg.G;
    tc_merge_final<T, D>(p, frm, fm[2] & 0xffffffffll, fm[2] >> 32, fm[0],
                         (int)(fm[3] & 0xffffffffll), (size_t)fm[1], smem, mbar, wait_limit);
    if (tid == 0) p.counters[fm[3] >> 32] = 0;  // the ticket, ready for the next launch
  }
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
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::kTmemCols)
                 : "memory");
}

}  // namespace kvc
