// attend_streamk.cuh -- N2 + N3 (tensor-core, persistent): stream-K split attention.
//
// Same contract and the same per-tile arithmetic as attend_mma.cuh (mma.m16n8k16
// with tokens as M, query rows as N; fp32 online softmax), organised so that no
// SM waits for work or for memory between pieces of work:
//
// * Work is counted in 64-token tiles of "segments" s = (request b, KV head g,
//   row block rb), in that order; segment s has ceil((L_b + i_max + 1) / 64)
//   tiles, where i_max is the largest new-row index of the row block.  Each
//   segment is preceded by `sk_penalty` virtual tiles that hold no work: a CTA
//   pays a fixed cost (epilogue, ticket, a new q and a ring that restarts) for
//   every segment it enters, and the virtual tiles charge that cost to it.
//   Each of the G persistent CTAs takes the contiguous range [c*W/G,
//   (c+1)*W/G) of the W virtual tiles in total, so every CTA streams the same
//   work, costs included, whatever the mix of lengths.
//   Every CTA computes the per-request tile counts and their prefix sums from
//   seq_lens itself (a block scan), so the host needs no lengths.
// * Stage layout: K (and V) rows of 128-byte, 128-byte-swizzled chunks.  Contiguous
//   caches and pages of 64+ tokens: one 64-row box per 64-element half ([half][row]).
//   Paged D = 128 with smaller pages: the tensor maps are 4-D (64 elements, page
//   tokens, 2 halves, page blocks) so that one box brings a whole (page, head) block,
//   laid out [page][half][row in page] -- half the copies of per-half boxes, and the
//   same conflict-free ldmatrix pattern (8 consecutive rows of one half).
// * Warp 0 keeps the 3-stage TMA ring full across segment boundaries; the
//   first tile of each segment piece also carries that segment's q rows (one
//   bulk copy into a per-stage q slot).  On a paged cache lane k of warp 0
//   looks up and loads box k of a tile, and the page ids of the next tile are
//   read while the current one is consumed, so a tile costs one lookup latency
//   (hidden) rather than one per page.
// * When a piece ends, the four warps merge their partial results inside the
//   stage they just consumed, while the other stages keep streaming.  A piece
//   that covers its whole segment writes the output directly.  A CTA has at
//   most two partial pieces (its first and its last); they go to slots
//   (c, 0) and (c, 1) of the workspace, and the last CTA of a segment to
//   finish merges the segment's pieces by log-sum-exp ("9. 推理" 9.7:
//   exact up to rounding); a release-acquire ticket decides who is last (its
//   result is read only at the CTA's next piece end or after its loop), so
//   nothing ever waits on another CTA.  The merge spreads each output quad's
//   pieces over up to eight threads, so all of its loads are in flight at once,
//   and combines them with shuffles.
// * Launched with programmatic stream serialization, a CTA sets up its
//   barriers, plans its tile range from the lengths as they stand and
//   prefetches the first tiles of that range into L2 while the grid ahead
//   finishes; right after the dependency wait it issues its first stages from
//   that plan while it re-reads the lengths, and if any changed it waits for
//   those copies, resets its barriers and plans again.
// * FP8 (a compile-time variant, 1-8 rows): the stages carry E4M3 codes and
//   per-row scales; the codes are converted in registers as in attend_fp8.cuh, and
//   one running reference per row serves both the sum and the V-scaled weights.
#pragma once

#include <cuda.h>
#include <math.h>

#include "attend_fp8.cuh"
#include "attend_mma.cuh"
#include "device_common.cuh"
#include "params.cuh"
#include "splitk_epilogue.cuh"

#ifndef KVC_SK_STAGES
#define KVC_SK_STAGES 3
#endif
#ifndef KVC_SK_FP8_CHAINS  // FP8: independent S accumulator chains
#define KVC_SK_FP8_CHAINS 2
#endif
#ifndef KVC_SK_FP8_MIN_BLOCKS  // FP8, D = 128: resident CTAs an SM (a register bound)
#define KVC_SK_FP8_MIN_BLOCKS 3
#endif
#ifndef KVC_SK_STAGES_FP8  // FP8, D = 128: stages (3 CTAs of 3 stages fit an SM)
#define KVC_SK_STAGES_FP8 3
#endif
#ifndef KVC_SK_STAGES_D64
#define KVC_SK_STAGES_D64 KVC_SK_STAGES
#endif
// Tiles of its range a CTA prefetches into L2 before the dependency wait (measured on
// contiguous caches: 2 beats 0, 1, 3 and 5: more delays the CTAs that start late and
// competes with the grid ahead for HBM; paged caches: 1 beats 0 and 2).
// Paged: tiles ahead of the next copy whose page ids are already being read (measured:
// 3 is no faster than 1 once a page is one box).
#ifndef KVC_SK_LOOKAHEAD
#define KVC_SK_LOOKAHEAD 1
#endif
#ifndef KVC_SK_PREFETCH_TILES  // tiles of its range a CTA warms in L2 before the wait
#define KVC_SK_PREFETCH_TILES 2
#endif
#ifndef KVC_SK_PREFETCH_TILES_PAGED  // the same on a paged cache (measured: 1 beats 2 there)
#define KVC_SK_PREFETCH_TILES_PAGED 1
#endif

namespace kvc {

// L2 prefetch of one box: nothing lands in shared memory and nothing signals
// completion, so it changes no result whatever the coordinates name.
__device__ __forceinline__ void tma_prefetch_2d(const void* tmap, int c0, int c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];"
               ::"l"(tmap), "r"(c0), "r"(c1)
               : "memory");
}

// atomicAdd(ticket, 1) with release-acquire semantics at GPU scope: every write
// this CTA made before the barrier that precedes it is visible to whoever reads the
// new count, and the writes of the CTAs counted before it are visible to this one.
__device__ __forceinline__ int ticket_add_acq_rel(int* ticket) {
  int old;
  asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], 1;" : "=r"(old) : "l"(ticket) : "memory");
  return old;
}

// 4-D tiled load / L2 prefetch of one box (the blocked paged layout), no multicast.
__device__ __forceinline__ void tma_load_4d(void* dst, const void* tmap, int c0, int c1, int c2,
                                            int c3, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4, %5}], [%6], %7;"
      ::"r"(smem_addr(dst)), "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tma_prefetch_4d(const void* tmap, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];"
               ::"l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

// L2 prefetch of `bytes` (a multiple of 16) from a 16-byte aligned address.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// -------------------------------------------- programmatic dependent launch
// A kernel launched with programmatic stream serialization may start before the
// grid ahead of it in the stream has finished.  griddep_wait() blocks until that
// grid has completed and its writes are visible (it returns at once for a plain
// launch); griddep_launch_dependents() lets the next such grid begin launching.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// FP8 = true: the cache holds E4M3 codes (one byte an element) and one fp32 scale per
// (token, KV head); a stage then holds the K and V codes of a tile and their scales, and
// twice as many stages keep the same bytes in flight.
template <int D, bool FP8 = false>
struct StreamKCfg {
  static constexpr int kWarps = 4;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kTile = 64;
  static constexpr int kHalves = D / 64;
  static constexpr int kBoxBytes = kTile * 128;
  static constexpr int kTileBytes = kTile * D * (FP8 ? 1 : 2);  // K (equally V) of a stage
  static constexpr int kScaleBytes = FP8 ? 2 * kTile * 4 : 0;   // K and V scales of a stage
  // FP8: half-size stages; the conversions make the tile arithmetic latency-bound, so
  // D = 128 trades depth for a third resident CTA (3 x 3 stages an SM)
  static constexpr int kStages =
      FP8 ? (D == 128 ? KVC_SK_STAGES_FP8 : 6) : (D == 64 ? KVC_SK_STAGES_D64 : KVC_SK_STAGES);
  static constexpr int kKSteps = D / 16;
  static constexpr int kMTiles = D / 16;
  static constexpr int kRing = 2 * kStages * kTileBytes + kStages * kScaleBytes;

  template <int NT>
  static constexpr size_t smem_bytes() {
    return 1024 + kRing                                 // aligned K and V rings
           + kStages * NT * 8 * D * 2                   // q slots
           + kWarps * NT * 8 * 2 * sizeof(float)        // warp m and l
           + 2 * kStages * sizeof(uint64_t) + 64;       // barriers, flags
  }
  // resident CTAs an SM should hold (shared memory allows 4 at D = 64, 2 at D = 128):
  // a register bound for the compiler
  template <int NT>
  static constexpr int min_blocks() {
    return FP8 ? (D == 64 ? 3 : KVC_SK_FP8_MIN_BLOCKS) : D == 64 ? (KVC_SK_STAGES_D64 <= 3 ? (NT == 1 ? 4 : 3) : 2) : 2;
  }
  // the block scan of per-request tile counts and the lengths it read use the ring
  // before the first copy
  static constexpr int kMaxBatch = (kRing / (int)sizeof(int) - 1) / 2;
  // the piece epilogue's W x 8NT x D fp32 partials live in one stage's K and V buffers
  static_assert(!FP8 || kWarps * 8 * D * 4 <= 2 * kTileBytes, "FP8: one row group of 8");
  static_assert(!FP8 || D == 64 || KVC_SK_FP8_MIN_BLOCKS * (smem_bytes<1>() + 1024) <= 233472,
                "FP8 D = 128: the resident CTAs must fit an SM's shared memory");
};

// Row-block geometry: new-row indices covered by row block rb.
struct RowBlock {
  int imin, imax;
};

__device__ __forceinline__ RowBlock row_block(int rb, int R, int rows, int T_new) {
  const int r0 = rb * R;
  const int r1 = min(r0 + R, rows) - 1;
  if (r1 - r0 + 1 >= T_new) return {0, T_new - 1};
  const int i0 = r0 % T_new, i1 = r1 % T_new;
  return i1 >= i0 ? RowBlock{i0, i1} : RowBlock{0, T_new - 1};
}

__device__ __forceinline__ bool length_ok(const AttendParams& p, int L, bool paged) {
  return L >= 0 && L + p.T_new <= p.max_T &&
         (!paged || ((L + p.T_new - 1) >> p.page_shift) < p.max_pages);
}

// Virtual tiles of request b: its segments' tiles plus their penalty tiles (row-block
// major: those of one row block, every block having as many).
template <int R>
__device__ __forceinline__ int request_tiles(const AttendParams& p, int L) {
  int t = 0;
  const int nrb = p.sk_rb_major ? 1 : p.row_blocks;
  for (int rb = 0; rb < nrb; ++rb)
    t += ceil_div(L + row_block(rb, R, p.rows, p.T_new).imax + 1, 64) + p.sk_penalty;
  return t * p.H_kv;
}

// Walks the real tiles in the global order: request, KV head, row block, tile; or, row-block
// major (p.sk_rb_major), row block, request, KV head, tile -- then the CTAs that stream one
// K/V tile for different row blocks are a fixed number of ranges apart and stream it at
// about the same time, so that L2 serves all but the first read.
template <int R>
struct TileCursor {
  int b, g, rb, L, k, seg_tiles;
  long long seg_start;  // virtual index of the segment's first real tile

  __device__ __forceinline__ void enter_segment(const AttendParams& p) {
    seg_tiles = ceil_div(L + row_block(rb, R, p.rows, p.T_new).imax + 1, 64);
  }
  // lens: the requests' lengths (seq_lens, or a copy of them in shared memory)
  __device__ __forceinline__ void next(const AttendParams& p, bool paged, const int* lens) {
    if (++k < seg_tiles) return;
    seg_start += seg_tiles + p.sk_penalty;
    k = 0;
    if (p.sk_rb_major || ++rb == p.row_blocks) {
      if (!p.sk_rb_major) rb = 0;
      if (++g == p.H_kv) {
        g = 0;
        do {  // requests whose length is invalid contribute no tiles
          ++b;
          L = b < p.B ? lens[b] : 0;
        } while (b < p.B && !length_ok(p, L, paged));
        if (p.sk_rb_major && b >= p.B && rb + 1 < p.row_blocks) {  // the next row block
          ++rb;
          b = -1;
          do {
            ++b;
            L = b < p.B ? lens[b] : 0;
          } while (b < p.B && !length_ok(p, L, paged));
        }
      }
    }
    enter_segment(p);
  }
  __device__ __forceinline__ void next(const AttendParams& p, bool paged) {
    next(p, paged, p.seq_lens);
  }
};

// Stream-K ranges: CTA r streams the W tiles' range [r*W/G, (r+1)*W/G).
struct RangeMap {
  long long W;
  int G;
  __device__ __forceinline__ long long start(long long r) const { return r * W / G; }
  __device__ __forceinline__ long long of(long long t) const {  // range holding tile t
    return ((t + 1) * G - 1) / W;
  }
};

// Merge the partial pieces rf..rl of one segment (the CTA's rows r0.., nr of them
// valid, outputs from row_base; slots of p.sk_slot_rows rows) by log-sum-exp:
//     out = sum_q 2^(lse_q - M) o_q / sum_q 2^(lse_q - M),   M = max_q lse_q.
// Piece q lives in workspace slot 2*(rf+q) + 1 if it is the first piece and range rf
// began before the segment (its penalty tiles, before s0), else 2*(rf+q).  Each output quad (4 consecutive
// elements of a row) is handled by tpq consecutive lanes (a power of two up to 8,
// chosen so the CTA's threads cover the quads): lane `sub` of the group takes pieces
// sub, sub + tpq, ..., issuing the lse and the float4 of four pieces before using
// any, with a running maximum; the group then combines its lanes' (max, sum, acc)
// with xor shuffles.  A merge is thus about one L2 round trip, not one per piece.
// merge_rows_spread merges rows r_off .. r_off + nr - 1 of the npc pieces from range rf
// (rf_mid: piece 0 sits in its range's second slot) into outputs from row row_base +
// r_off; merge_pieces_spread merges a whole segment's rows.
template <typename T, int D, int NTH>
__device__ __forceinline__ void merge_rows_spread(const AttendParams& p, long long rf, int npc,
                                                  bool rf_mid, int r_off, int nr,
                                                  size_t row_base) {
  constexpr int Q4 = D / 4;
  const int tid = threadIdx.x;
  const int items = nr * Q4;
  int tpq = 1;
  while (tpq < 8 && tpq < npc && items * tpq * 2 <= NTH) tpq *= 2;
  T* out = static_cast<T*>(p.out);
#pragma unroll 1
  for (int base = 0; base < items * tpq; base += NTH) {  // the same trip count in every thread
    const int w = base + tid;
    const bool act = w < items * tpq;
    const int item = act ? w / tpq : 0;
    const int sub = w & (tpq - 1);
    const int rr = item / Q4;
    const int d = (item - rr * Q4) * 4;
    float m_run = -INFINITY, den = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
    for (int q0 = sub; act && q0 < npc; q0 += 4 * tpq) {
      float ls[4];
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int q = q0 + u * tpq;
        if (q < npc) {
          const size_t slot = (size_t)(rf + q) * 2 + ((q == 0 && rf_mid) ? 1 : 0);
          const size_t srow = slot * p.sk_slot_rows + r_off + rr;
          ls[u] = __ldcg(p.ws_lse + srow);
          v[u] = __ldcg(reinterpret_cast<const float4*>(p.ws_o + srow * D + d));
        } else {
          ls[u] = -INFINITY;
          v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      float mx = fmaxf(fmaxf(ls[0], ls[1]), fmaxf(ls[2], ls[3]));
      const float m_new = fmaxf(m_run, mx);
      if (m_new == -INFINITY) continue;  // nothing visible yet
      const float f = m_run == -INFINITY ? 0.f : exp2f(m_run - m_new);
      den *= f;
      acc.x *= f;
      acc.y *= f;
      acc.z *= f;
      acc.w *= f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float wq = ls[u] == -INFINITY ? 0.f : exp2f(ls[u] - m_new);
        den += wq;
        acc.x = fmaf(wq, v[u].x, acc.x);
        acc.y = fmaf(wq, v[u].y, acc.y);
        acc.z = fmaf(wq, v[u].z, acc.z);
        acc.w = fmaf(wq, v[u].w, acc.w);
      }
      m_run = m_new;
    }
    // combine the group's lanes (consecutive lanes of one warp; every lane takes part)
#pragma unroll 1
    for (int off = 1; off < tpq; off <<= 1) {
      const float m_o = __shfl_xor_sync(0xffffffffu, m_run, off);
      const float den_o = __shfl_xor_sync(0xffffffffu, den, off);
      float4 a_o;
      a_o.x = __shfl_xor_sync(0xffffffffu, acc.x, off);
      a_o.y = __shfl_xor_sync(0xffffffffu, acc.y, off);
      a_o.z = __shfl_xor_sync(0xffffffffu, acc.z, off);
      a_o.w = __shfl_xor_sync(0xffffffffu, acc.w, off);
      const float m_new = fmaxf(m_run, m_o);
      const float f1 = m_run == -INFINITY ? 0.f : exp2f(m_run - m_new);
      const float f2 = m_o == -INFINITY ? 0.f : exp2f(m_o - m_new);
      den = den * f1 + den_o * f2;
      acc.x = acc.x * f1 + a_o.x * f2;
      acc.y = acc.y * f1 + a_o.y * f2;
      acc.z = acc.z * f1 + a_o.z * f2;
      acc.w = acc.w * f1 + a_o.w * f2;
      m_run = m_new;
    }
    if (act && sub == 0) {
      const float inv = den > 0.f ? 1.f / den : 0.f;
      T* o = out + (row_base + r_off + rr) * D + d;
      store_elt<T>(o, acc.x * inv);
      store_elt<T>(o + 1, acc.y * inv);
      store_elt<T>(o + 2, acc.z * inv);
      store_elt<T>(o + 3, acc.w * inv);
    }
  }
}

template <typename T, int D, int R, int NTH>
__device__ __forceinline__ void merge_pieces_spread(const AttendParams& p, const RangeMap& rm,
                                                    long long rf, long long rl, long long s0,
                                                    int nr, size_t row_base) {
  // range rf streamed real tiles of an earlier segment first iff it began before this
  // segment's penalty tiles
  const bool rf_mid = rm.start(rf) < s0 - p.sk_penalty;
  merge_rows_spread<T, D, NTH>(p, rf, (int)(rl - rf + 1), rf_mid, 0, nr, row_base);
}

// FP8 = true (NT 1, bf16 q and out): the stages carry E4M3 codes and scales and the
// codes are converted in registers as in attend_fp8.cuh, with one running reference per
// row (the maximum of s + max(exponent of v_scale, -64)) for the sum and the weights
// v_scale * 2^(s - m); planning, the ring, pieces, epilogue and merge are the same.
template <int D, int NT, typename T, bool PAGED, bool FP8 = false>
__global__ void __launch_bounds__(StreamKCfg<D, FP8>::kThreads,
                                  StreamKCfg<D, FP8>::template min_blocks<NT>())
    attend_streamk_kernel(const AttendParams p, const __grid_constant__ CUtensorMap tmk,
                          const __grid_constant__ CUtensorMap tmv) {
  using C = StreamKCfg<D, FP8>;
  static_assert(!FP8 || (NT == 1 && Elt<T>::kCode == KVC_BF16), "FP8: 1-8 rows, bf16");
  constexpr int W = C::kWarps;
  constexpr int NTH = C::kThreads;
  constexpr int R = NT * 8;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sk = smem;
  unsigned char* sv = smem + C::kStages * C::kTileBytes;
  float* scl = reinterpret_cast<float*>(smem + 2 * C::kStages * C::kTileBytes);  // FP8: [st][K|V]
  unsigned char* sq = smem + C::kRing;  // [stage][R][D]
  float* red_m = reinterpret_cast<float*>(sq + C::kStages * R * D * 2);
  float* red_l = red_m + W * R;
  uint64_t* full = reinterpret_cast<uint64_t*>(red_l + W * R);
  uint64_t* empty = full + C::kStages;
  int* flags = reinterpret_cast<int*>(empty + C::kStages);  // [0] abort, [1] last, [4..7] scan

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int c = blockIdx.x;

  // Programmatic dependent launch: the next grid in the stream may begin as
  // this one's CTAs retire.  Before griddep_wait() this kernel writes no global
  // memory and reads seq_lens and the block table only to plan and to aim L2
  // prefetches, which change no result; every read that counts comes after it.
  griddep_launch_dependents();

  // CTA-local set-up (shared memory only): made visible by the first barrier of locate().
  if (tid == 0) {
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
#pragma unroll
    for (int st = 0; st < C::kStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], W);
    }
    flags[0] = 0;
    fence_barrier_init();
  }

  // ------------------------------------ per-request tile prefix and this CTA's range
  int* P = reinterpret_cast<int*>(smem);  // [B + 1], in the ring before any copy
  int* Ls = P + p.B + 1;                   // [B]: the lengths the scan read
  long long Wt = 0, lo = 0;
  int G = 0, ntiles = 0;
  TileCursor<R> cur;
  // this thread's requests in the scan, and a digest of the lengths it read there
  const int per_thread = ceil_div(p.B, NTH);
  const int b_lo = min(p.B, tid * per_thread), b_hi = min(p.B, b_lo + per_thread);
  auto mix = [](uint32_t h, int L) { return (h ^ (uint32_t)L) * 0x9E3779B1u + 0x7F4A7C15u; };
  uint32_t digest = 0;
  // Returns whether this CTA has tiles; ends with a barrier.  P and Ls stay valid until
  // the first copy into the ring.
  auto locate = [&](bool authoritative) -> bool {
    {
      int sum = 0;
      digest = 0;
      for (int b = b_lo; b < b_hi; ++b) {
        const int L = p.seq_lens[b];
        digest = mix(digest, L);
        Ls[b] = L;
        int t = 0;
        if (length_ok(p, L, PAGED)) t = request_tiles<R>(p, L);
        else if (authoritative) flag_error(p.err, KVC_ERR_BOUNDS);
        P[b] = t;
        sum += t;
      }
      int incl = sum;  // inclusive scan across the block
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      int* wsum = flags + 4;  // [W]
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
    }
    Wt = P[p.B];
    G = (int)(Wt < (long long)gridDim.x ? Wt : (long long)gridDim.x);
    bool work = c < G;  // the same in every thread
    if (work) {
      lo = (long long)c * Wt / G;
      ntiles = (int)((long long)(c + 1) * Wt / G - lo);
      // starting position: request (binary search), KV head, row block
      int a = 0, z = p.B;  // largest b with P[b] <= lo
      while (z - a > 1) {
        const int mid = (a + z) >> 1;
        if (P[mid] <= lo) a = mid;
        else z = mid;
      }
      while (P[a + 1] == P[a]) ++a;  // skip requests with no tiles
      cur.b = a;
      cur.L = Ls[a];
      work = length_ok(p, cur.L, PAGED);
      int local = (int)(lo - P[a]);
      const int per_g = (P[a + 1] - P[a]) / p.H_kv;
      cur.g = local / per_g;
      local -= cur.g * per_g;
      cur.rb = 0;
      while (work) {
        const int t = ceil_div(cur.L + row_block(cur.rb, R, p.rows, p.T_new).imax + 1, 64);
        if (local < t + p.sk_penalty || cur.rb == p.row_blocks - 1) {
          cur.seg_tiles = t;
          break;
        }
        local -= t + p.sk_penalty;
        ++cur.rb;
      }
      // local: the virtual offset in the segment; its penalty tiles are skipped
      cur.seg_start = lo - local + p.sk_penalty;
      cur.k = max(0, local - p.sk_penalty);
      // the real tiles of [lo, hi): walk the segments the range reaches
      const long long hi = (long long)(c + 1) * Wt / G;
      ntiles = 0;
      TileCursor<R> w = cur;
#pragma unroll 1
      while (work && w.b < p.B) {
        const long long v = w.seg_start + w.k;
        if (v >= hi) break;
        const long long seg_end = w.seg_start + w.seg_tiles;
        const long long stop = hi < seg_end ? hi : seg_end;
        ntiles += (int)(stop - v);
        if (stop < seg_end) break;
        w.k = w.seg_tiles - 1;
        w.next(p, PAGED, Ls);
      }
      work = work && ntiles > 0;
    }
    __syncthreads();
    return work;
  };

  // Paged tiles are loaded as boxes of min(page, 64) rows, one page lookup each.
  const int Pg = PAGED ? (1 << p.page_shift) : C::kTile;
  const int box_rows = Pg < C::kTile ? Pg : C::kTile;
  const int nbox = C::kTile / box_rows;         // <= 8: pages of 8 or more tokens
  const int beyond = p.num_pages * p.H_kv * Pg;  // first row past the pool: zero fill
  const bool blocked = PAGED && D == 128 && p.sk_blocked != 0;
  // byte offset in a stage of tile row `row` (its half 0, chunk 0 before the swizzle)
  auto row_part = [&](int row) -> int {
    return blocked ? (row >> p.page_shift) * (box_rows * 256) + (row & (box_rows - 1)) * 128
                   : row * 128;
  };
  const int half_stride = blocked ? box_rows * 128 : C::kBoxBytes;
  // byte offset of 16-byte chunk `chunk` (of D/8) of tile row `row`, swizzled
  auto tile_off = [&](int row, int chunk) -> uint32_t {
    return row_part(row) + (chunk >> 3) * half_stride + (((chunk & 7) ^ (row & 7)) << 4);
  };
  // Row of box `box` of the tile under cursor pc: -1 = the lookup is still to be done;
  // returns `beyond` past the segment's last position.
  auto box_page_row = [&](const TileCursor<R>& pc, int box, int page) -> int {
    const int t = pc.k * C::kTile + box * box_rows;
    if (t >= pc.L + row_block(pc.rb, R, p.rows, p.T_new).imax + 1) return beyond;
    if (page < 0 || page >= p.num_pages) return -1;
    return (page * p.H_kv + pc.g) * Pg + (t & (Pg - 1));
  };
  auto lookup_page = [&](const TileCursor<R>& pc, int box) -> int {
    const int t = pc.k * C::kTile + box * box_rows;
    if (pc.b >= p.B || box >= nbox ||
        t >= pc.L + row_block(pc.rb, R, p.rows, p.T_new).imax + 1)
      return 0;
    return p.block_table[(size_t)pc.b * p.max_pages + (t >> p.page_shift)];
  };

  // Speculative pass: plan from the lengths as they stand and warm L2 with the
  // first tiles of this CTA's range while the grid ahead finishes.  Lengths or
  // pages that change before the wait only waste a prefetch.
  const bool spec_work = locate(false);
  const uint32_t spec_digest = digest;
  const TileCursor<R> spec_cur = cur;
  if (spec_work && warp == 0) {
    // only boxes wholly inside the tensor: the cursor may walk off stale lengths
    const long long rows_total =
        PAGED ? (long long)p.num_pages * p.H_kv * Pg : (long long)p.B * p.H_kv * p.max_T;
    const int pf = min(ntiles, PAGED ? KVC_SK_PREFETCH_TILES_PAGED : KVC_SK_PREFETCH_TILES);
    TileCursor<R> pc = cur;
#pragma unroll 1
    for (int i = 0; i < max(pf, 1) && pc.b < p.B; ++i) {
      if ((i == 0 || pc.k == 0) && lane == 31) {  // the piece's q rows
        const int r0 = pc.rb * R;
        const char* qsrc = static_cast<const char*>(p.q) +
                           ((((size_t)pc.b * p.H_q + (size_t)pc.g * p.group) * p.T_new) + r0) *
                               D * 2;
        bulk_prefetch_l2(qsrc, (uint32_t)min(R, p.rows - r0) * D * 2);
      }
      if (i >= pf) break;  // no tiles prefetched: q only
      if (!PAGED) {
        const int y = (pc.b * p.H_kv + pc.g) * p.max_T + pc.k * C::kTile;
        // FP8 code maps: one box of D bytes a row
        if (lane < (FP8 ? 1 : C::kHalves) && y + C::kTile <= rows_total) {
          tma_prefetch_2d(&tmk, lane * 64, y);
          tma_prefetch_2d(&tmv, lane * 64, y);
        }
      } else if (lane < nbox) {
        const int y = box_page_row(pc, lane, lookup_page(pc, lane));
        if (y >= 0 && y != beyond && y + box_rows <= rows_total) {
          if (FP8) {
            tma_prefetch_2d(&tmk, 0, y);
            tma_prefetch_2d(&tmv, 0, y);
          } else if (blocked) {
            tma_prefetch_4d(&tmk, 0, 0, 0, y >> p.page_shift);
            tma_prefetch_4d(&tmv, 0, 0, 0, y >> p.page_shift);
          } else {
#pragma unroll
            for (int h = 0; h < C::kHalves; ++h) {
              tma_prefetch_2d(&tmk, h * 64, y);
              tma_prefetch_2d(&tmv, h * 64, y);
            }
          }
        }
      }
      pc.next(p, PAGED, Ls);
    }
  }
  if (spec_work && warp == 1 && lane == 0 && p.k_new != nullptr) {
    // the new rows of every segment this range ends: the fused append reads them
    const long long hi = (long long)(c + 1) * Wt / G;
    TileCursor<R> w = cur;
#pragma unroll 1
    while (w.b < p.B && w.seg_start < hi) {
      if (w.seg_start + w.seg_tiles <= hi) {
        const size_t off = ((size_t)w.b * p.H_kv + w.g) * p.T_new * D * 2;
        bulk_prefetch_l2(static_cast<const char*>(p.k_new) + off, (uint32_t)p.T_new * D * 2);
        bulk_prefetch_l2(static_cast<const char*>(p.v_new) + off, (uint32_t)p.T_new * D * 2);
      }
      w.k = w.seg_tiles - 1;
      w.next(p, PAGED, Ls);
    }
  }
  griddep_wait();

  // ------------------------------------------------------- tile producer
  // Warp 0 issues the copies (lane 0 the barrier and q; lane k box k).
  const bool producer = (warp == 0) && !p.stall;
  const uint64_t pol = l2_policy_evict_first();
  TileCursor<R> pc = spec_cur;  // producer's own cursor
  int issued = 0;
  // Paged: lane k < nbox holds the page ids of box k of the next kLookahead tiles to
  // issue (ids[0] for tile pc); a second cursor, kLookahead - 1 tiles ahead of pc, reads
  // them, so a lookup has that many tiles' time to land.
  constexpr int kLookahead = KVC_SK_LOOKAHEAD;
  int ids[kLookahead];
  TileCursor<R> pa = spec_cur;
  auto prime_lookups = [&]() {
    if (PAGED && producer) {
      pa = pc;
#pragma unroll
      for (int i = 0; i < kLookahead; ++i) {
        if (i > 0) pa.next(p, PAGED);
        ids[i] = lookup_page(pa, lane);
      }
    }
  };
  auto issue = [&]() {
    const int st = issued % C::kStages;
    const bool first = (issued == 0) || (pc.k == 0);
    const int r0 = pc.rb * R;
    const int nr = min(R, p.rows - r0);
    const uint32_t qbytes = first ? (uint32_t)nr * D * 2 : 0u;
    if (lane == 0) {
      mbar_arrive_expect_tx(&full[st], 2 * C::kTileBytes + C::kScaleBytes + qbytes);
      if (first) {
        const char* qsrc = static_cast<const char*>(p.q) +
                           ((((size_t)pc.b * p.H_q + (size_t)pc.g * p.group) * p.T_new) + r0) *
                               D * 2;
        bulk_g2s(sq + st * R * D * 2, qsrc, qbytes, &full[st]);
      }
    }
    __syncwarp();
    unsigned char* dk = sk + st * C::kTileBytes;
    unsigned char* dv = sv + st * C::kTileBytes;
    if constexpr (FP8) {  // codes: one box of D bytes a row; scales: 1-D bulk copies
      float* ds = scl + st * 2 * C::kTile;
      if (!PAGED) {
        const int y = (pc.b * p.H_kv + pc.g) * p.max_T + pc.k * C::kTile;
        if (lane == 0) {
          tma_load_2d(dk, &tmk, 0, y, &full[st], pol);
          tma_load_2d(dv, &tmv, 0, y, &full[st], pol);
        } else if (lane == 1) {  // T_pad holds whole tiles
          const size_t srow = ((size_t)pc.b * p.H_kv + pc.g) * p.T_pad + pc.k * C::kTile;
          bulk_g2s_hint(ds, p.k_scales + srow, C::kTile * 4, &full[st], pol);
          bulk_g2s_hint(ds + C::kTile, p.v_scales + srow, C::kTile * 4, &full[st], pol);
        }
      } else if (lane < nbox) {
        int y = box_page_row(pc, lane, ids[0]);
        if (y < 0) {  // a page id outside the pool: zero fill, reported
          flag_error(p.err, KVC_ERR_BOUNDS);
          y = beyond;
        }
        // past the segment (zero codes): any finite scales, row 0's
        const size_t srow = y == beyond ? 0 : (size_t)y;
        const int off = lane * box_rows;
        tma_load_2d(dk + off * D, &tmk, 0, y, &full[st], pol);
        tma_load_2d(dv + off * D, &tmv, 0, y, &full[st], pol);
        bulk_g2s_hint(ds + off, p.k_scales + srow, box_rows * 4, &full[st], pol);
        bulk_g2s_hint(ds + C::kTile + off, p.v_scales + srow, box_rows * 4, &full[st], pol);
      }
    } else if (!PAGED) {
      if (lane < C::kHalves) {
        const int y = (pc.b * p.H_kv + pc.g) * p.max_T + pc.k * C::kTile;
        tma_load_2d(dk + lane * C::kBoxBytes, &tmk, lane * 64, y, &full[st], pol);
        tma_load_2d(dv + lane * C::kBoxBytes, &tmv, lane * 64, y, &full[st], pol);
      }
    } else if (lane < nbox) {
      int y = box_page_row(pc, lane, ids[0]);
      if (y < 0) {  // a page id outside the pool: zero fill, reported
        flag_error(p.err, KVC_ERR_BOUNDS);
        y = beyond;
      }
      if (blocked) {  // one box: the page's block, both halves
        const int off = lane * box_rows * 256;
        tma_load_4d(dk + off, &tmk, 0, 0, 0, y >> p.page_shift, &full[st], pol);
        tma_load_4d(dv + off, &tmv, 0, 0, 0, y >> p.page_shift, &full[st], pol);
      } else {
        const int off = lane * box_rows * 128;
#pragma unroll
        for (int h = 0; h < C::kHalves; ++h) {
          tma_load_2d(dk + h * C::kBoxBytes + off, &tmk, h * 64, y, &full[st], pol);
          tma_load_2d(dv + h * C::kBoxBytes + off, &tmv, h * 64, y, &full[st], pol);
        }
      }
    }
    ++issued;
    pc.next(p, PAGED);
    if (PAGED) {  // shift the lookahead queue and read the ids kLookahead - 1 tiles ahead
#pragma unroll
      for (int i = 0; i + 1 < kLookahead; ++i) ids[i] = ids[i + 1];
      pa.next(p, PAGED);
      ids[kLookahead - 1] = lookup_page(pa, lane);
    }
  };
  // The first copies of the speculative plan go out now, after the wait (so they read
  // what the grid ahead wrote), while every thread checks the plan against the lengths
  // as they now stand; a stale plan drains them and starts over.
  if (spec_work && producer) {
    prime_lookups();
    while (issued < min(C::kStages, ntiles)) issue();
  }
  bool work;
  {
    uint32_t h = 0;
    for (int b = b_lo; b < b_hi; ++b) {
      const int L = p.seq_lens[b];
      h = mix(h, L);
      if (!length_ok(p, L, PAGED)) flag_error(p.err, KVC_ERR_BOUNDS);
    }
    const bool same_first = !spec_work || p.seq_lens[spec_cur.b] == spec_cur.L;
    if (__syncthreads_or(h != spec_digest || !same_first || p.replan)) {
      // every speculative copy lands before the barriers are reset and the ring reused
      bool drained = true;
      if (producer && lane == 0)
#pragma unroll 1
        for (int j = 0; j < issued && drained; ++j)
          drained = mbar_wait(&full[j], 0, p.err, p.wait_limit_ns ? p.wait_limit_ns
                                                                  : kWaitLimitNs);
      if (__syncthreads_or(!drained)) return;  // a copy that never landed: reported
      if (tid == 0) {
#pragma unroll
        for (int st = 0; st < C::kStages; ++st) {
          mbar_inval(&full[st]);
          mbar_inval(&empty[st]);
          mbar_init(&full[st], 1);
          mbar_init(&empty[st], W);
        }
        fence_barrier_init();
      }
      issued = 0;
      work = locate(true);  // its barriers publish the new barriers too
      if (work && producer) {
        pc = cur;
        prime_lookups();
      }
    } else {
      work = spec_work;
      cur = spec_cur;
    }
  }
  if (!work) return;
  if (producer)
    while (issued < min(C::kStages, ntiles)) issue();

  // Bounded waits that keep every thread on the same control path: a wait that
  // runs out flags the error and the CTA abort word, and from then on waits
  // return at once; the CTA finishes its loop (on garbage) instead of
  // stranding threads at a named barrier.
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

  // The producer keeps kStages tiles in flight: tile t goes into stage t % kStages
  // once tile t - kStages has been released (`released` tiles are).  Warp 0 only.
  auto refill = [&](int released) {
#pragma unroll 1
    while (issued < ntiles && issued < released + C::kStages) {
      const int t = issued - C::kStages;
      bool ready = true;
      if (lane == 0) ready = wait(&empty[t % C::kStages], (t / C::kStages) & 1);
      if (!__shfl_sync(0xffffffffu, ready, 0)) break;  // aborted: issue nothing more
      issue();
    }
  };

  // ------------------------------------------------------------- consumers
  const int mi = lane >> 3;
  const int wrow = warp * 16;
  const int k_row = wrow + (mi & 1) * 8 + (lane & 7);
  const int k_cs = mi >> 1;
  const int v_row = wrow + (mi >> 1) * 8 + (lane & 7);
  const int v_cs = mi & 1;
  const uint32_t sk_addr = smem_addr(sk);
  const uint32_t sv_addr = smem_addr(sv);
  const int k_rp = row_part(k_row), k_sw = k_row & 7;
  const int v_rp = row_part(v_row), v_sw = v_row & 7;

  uint32_t qb[C::kKSteps][NT][2];
  int vis[NT][2];
  int r0 = 0, nr = 0, vis_min = 0, piece_first_j = 0;
  float m[NT][2], l[NT][2];
  float fcol[NT][2];  // FP8: score factor of the column's row: scale * log2(e) * 2^e_row
  float o[C::kMTiles][NT][4];
  // fresh running state; reset again at the end of every piece
  auto reset_state = [&]() {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        m[nt][cc] = -INFINITY;
        l[nt][cc] = 0.f;
      }
#pragma unroll
      for (int mt = 0; mt < C::kMTiles; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[mt][nt][e] = 0.f;
    }
  };
  reset_state();

  // A partial piece's ticket (see the end of a piece) and what its merge needs.
  constexpr int kTicketThread = 32;  // warp 1: the producer warp never waits on it
  RangeMap rm;
  rm.W = Wt;
  rm.G = G;
  bool pend = false;
  long long pend_rf = 0, pend_rl = 0, pend_s0 = 0;
  int pend_nr = 0, pend_count = 0;
  size_t pend_row_base = 0;
  int* pend_ticket = nullptr;
  // Every thread: if the pending ticket was the segment's last, merge its pieces.
  auto settle = [&]() {
    if (tid == kTicketThread) flags[1] = pend_count == (int)(pend_rl - pend_rf);
    named_barrier_sync(1, NTH);
    if (flags[1]) {
      merge_pieces_spread<T, D, R, NTH>(p, rm, pend_rf, pend_rl, pend_s0, pend_nr,
                                        pend_row_base);
      if (tid == 0) *pend_ticket = 0;
    }
    named_barrier_sync(1, NTH);  // flags[1] is read by every thread before it is reused
    pend = false;
  };

#pragma unroll 1
  for (int j = 0; j < ntiles; ++j) {
    const int st = j % C::kStages;
    if (producer && j >= 1) refill(j);
    wait(&full[st], (j / C::kStages) & 1);

    if (j == 0 || cur.k == 0) {  // a new piece: its q rows, visibility, fresh state
      piece_first_j = j;
      r0 = cur.rb * R;
      nr = min(R, p.rows - r0);
      vis_min = cur.L + row_block(cur.rb, R, p.rows, p.T_new).imin + 1;
      const unsigned char* qs = sq + st * R * D * 2;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int row = nt * 8 + (lane >> 2);
        if constexpr (FP8) {
          // f16 fragments of row / 2^e (e puts the row's largest |q| in [2^14, 2^15);
          // exact), under the k permutation of the converted K codes (attend_fp8.cuh):
          // k = 2c, 2c+1 <-> d = 16kk + 4c, +1; k = 8+2c, 9+2c <-> d = 16kk + 4c + 2, +3
          float qv[C::kKSteps][4];
          float amax = 0.f;
#pragma unroll
          for (int kk = 0; kk < C::kKSteps; ++kk) {
            uint2 w = make_uint2(0u, 0u);
            if (row < nr)
              w = *reinterpret_cast<const uint2*>(qs + row * D * 2 + (kk * 16 + (lane & 3) * 4) * 2);
            qv[kk][0] = __uint_as_float(w.x << 16);
            qv[kk][1] = __uint_as_float(w.x & 0xFFFF0000u);
            qv[kk][2] = __uint_as_float(w.y << 16);
            qv[kk][3] = __uint_as_float(w.y & 0xFFFF0000u);
#pragma unroll
            for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(qv[kk][e]));
          }
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
          const int e =
              amax > 0.f ? max((int)((__float_as_uint(amax) >> 23) & 0xFF) - 127 - 14, -126) : 0;
          const float inv = __uint_as_float((uint32_t)(127 - e) << 23);
#pragma unroll
          for (int kk = 0; kk < C::kKSteps; ++kk) {
            qb[kk][nt][0] = f32x2_to_f16x2(qv[kk][0] * inv, qv[kk][1] * inv);
            qb[kk][nt][1] = f32x2_to_f16x2(qv[kk][2] * inv, qv[kk][3] * inv);
          }
          // the exponent of column row nt*8 + 2(lane%4) + cc is held by lane 4 (row % 8)
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int ec = __shfl_sync(0xffffffffu, e, (((lane & 3) * 2 + cc) & 7) << 2);
            fcol[nt][cc] = p.scale_log2 * __uint_as_float((uint32_t)(127 + ec) << 23);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < C::kKSteps; ++kk) {
            if (row < nr) {
              const unsigned char* src = qs + row * D * 2 + (kk * 16 + (lane & 3) * 2) * 2;
              qb[kk][nt][0] = *reinterpret_cast<const uint32_t*>(src);
              qb[kk][nt][1] = *reinterpret_cast<const uint32_t*>(src + 16);
            } else {
              qb[kk][nt][0] = 0u;
              qb[kk][nt][1] = 0u;
            }
          }
        }
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int rr = nt * 8 + (lane & 3) * 2 + cc;
          vis[nt][cc] = rr < nr ? cur.L + (r0 + rr) % p.T_new + 1 : 0;
        }
      }
    }

    // Fused append: the tile that holds the new positions takes them from
    // k_new / v_new (its copy from the pool may predate them) and the first row
    // block writes them into the cache; every other tile is untouched.
    if (!FP8 && p.k_new != nullptr) {
      const int ta = cur.k * C::kTile;
      const int n_lo = max(cur.L, ta), n_hi = min(cur.L + p.T_new, ta + C::kTile);
      if (n_lo < n_hi) {  // the same decision in every thread of the CTA
        constexpr int CH = D / 8;  // 16-byte chunks per row
        unsigned char* dk = sk + st * C::kTileBytes;
        unsigned char* dv = sv + st * C::kTileBytes;
        char* kpool = static_cast<char*>(const_cast<void*>(p.k_pool));
        char* vpool = static_cast<char*>(const_cast<void*>(p.v_pool));
#pragma unroll 1
        for (int idx = tid; idx < (n_hi - n_lo) * CH; idx += NTH) {
          const int rr = idx / CH;
          const int ch = idx - rr * CH;
          const int pos = n_lo + rr;
          const size_t src =
              ((((size_t)cur.b * p.H_kv + cur.g) * p.T_new + (pos - cur.L)) * D + ch * 8) * 2;
          const uint4 kv = ld_global_nc_v4(static_cast<const char*>(p.k_new) + src);
          const uint4 vv = ld_global_nc_v4(static_cast<const char*>(p.v_new) + src);
          const uint32_t off = tile_off(pos - ta, ch);
          st_shared_v4(dk + off, kv);
          st_shared_v4(dv + off, vv);
          if (cur.rb == 0) {
            long long row;
            if (PAGED) {
              const int page = p.block_table[(size_t)cur.b * p.max_pages + (pos >> p.page_shift)];
              if (page < 0 || page >= p.num_pages) {
                flag_error(p.err, KVC_ERR_BOUNDS);
                continue;
              }
              row = ((long long)page * p.H_kv + cur.g) * (1 << p.page_shift) +
                    (pos & ((1 << p.page_shift) - 1));
            } else {
              row = ((long long)cur.b * p.H_kv + cur.g) * p.max_T + pos;
            }
            st_global_v4(kpool + (row * D + ch * 8) * 2, kv);
            st_global_v4(vpool + (row * D + ch * 8) * 2, vv);
          }
        }
        named_barrier_sync(1, NTH);
      }
    }
    if (FP8 && p.k_new != nullptr) {
      // FP8: warp w quantises rows (row, K or V) w, w + 4, ... of the new positions in
      // this tile exactly as the append kernel does, into the stage (codes and scale)
      // and, first row block, into the cache
      const int ta = cur.k * C::kTile;
      const int n_lo = max(cur.L, ta), n_hi = min(cur.L + p.T_new, ta + C::kTile);
      if (n_lo < n_hi) {  // the same decision in every thread of the CTA
        constexpr int PER = D / 32;
        float* ssc = scl + st * 2 * C::kTile;
#pragma unroll 1
        for (int task = warp; task < 2 * (n_hi - n_lo); task += W) {
          const bool is_v = task & 1;
          const int pos = n_lo + (task >> 1);
          const __nv_bfloat16* src =
              static_cast<const __nv_bfloat16*>(is_v ? p.v_new : p.k_new) +
              (((size_t)cur.b * p.H_kv + cur.g) * p.T_new + (pos - cur.L)) * D;
          uint32_t codes;
          const float scale = quantize_row_warp<PER>(src, lane, codes);
          const int d = lane * PER;  // this lane's first code of the row
          unsigned char* tile = (is_v ? sv : sk) + st * C::kTileBytes;
          unsigned char* at = tile + swz8<D>(pos - ta, d >> 4) + (d & 15);
          if (PER == 4) *reinterpret_cast<uint32_t*>(at) = codes;
          else *reinterpret_cast<uint16_t*>(at) = (uint16_t)codes;
          if (lane == 0) ssc[(is_v ? C::kTile : 0) + pos - ta] = scale;
          if (cur.rb == 0) {
            long long row, srow;
            if (PAGED) {
              const int page = p.block_table[(size_t)cur.b * p.max_pages + (pos >> p.page_shift)];
              if (page < 0 || page >= p.num_pages) {
                if (lane == 0) flag_error(p.err, KVC_ERR_BOUNDS);
                continue;
              }
              row = ((long long)page * p.H_kv + cur.g) * (1 << p.page_shift) +
                    (pos & ((1 << p.page_shift) - 1));
              srow = row;
            } else {
              row = ((long long)cur.b * p.H_kv + cur.g) * p.max_T + pos;
              srow = ((long long)cur.b * p.H_kv + cur.g) * p.T_pad + pos;
            }
            unsigned char* pool =
                static_cast<unsigned char*>(const_cast<void*>(is_v ? p.v_pool : p.k_pool));
            if (PER == 4) reinterpret_cast<uint32_t*>(pool + row * D)[lane] = codes;
            else reinterpret_cast<uint16_t*>(pool + row * D)[lane] = (uint16_t)codes;
            if (lane == 0) const_cast<float*>(is_v ? p.v_scales : p.k_scales)[srow] = scale;
          }
        }
        named_barrier_sync(1, NTH);
      }
    }

    const uint32_t kb = sk_addr + st * C::kTileBytes;
    const uint32_t vb = sv_addr + st * C::kTileBytes;
    const int t0 = cur.k * C::kTile;
    if constexpr (FP8) {
      // E4M3 tile: the codes converted as in attend_fp8.cuh
      const float* ssc = scl + st * 2 * C::kTile;
      const int ta = wrow + (lane >> 2);  // this thread's two tokens: ta and ta + 8
      const float ska = ssc[ta], skb = ssc[ta + 8];
      const float vsa = ssc[C::kTile + ta], vsb = ssc[C::kTile + ta + 8];
      // the reference of the row: the running maximum of s + max(e_v, -64), e_v the binary
      // exponent of the V scale (read off its bits: 2^e_v <= v_scale < 2^(e_v + 1)), so
      // the f16 weights v_scale * 2^(s - m) stay below 2 and the sum's terms 2^(s - m)
      // below 2^64
      const float lca = fmaxf((float)(int)((__float_as_uint(vsa) >> 23) & 0xFFu) - 127.f, -64.f);
      const float lcb = fmaxf((float)(int)((__float_as_uint(vsb) >> 23) & 0xFFu) - 127.f, -64.f);
      // KVC_SK_FP8_CHAINS independent accumulator chains (chunk % chains), summed after:
      // shorter dependent MMA chains for the one n-tile
      constexpr int NCH = KVC_SK_FP8_CHAINS;
      float sacc[NT][4];
      float sch[NCH][NT][4];
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sch[ch][nt][e] = 0.f;
#pragma unroll
      for (int kp = 0; kp < C::kKSteps; kp += 2) {
        uint32_t r[4];
        ldmatrix_x4(r, kb + swz8<D>(k_row, kp + k_cs));
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // chunk kp + h: r[2h] tokens 0-7, r[2h+1] tokens 8-15
          const uint32_t a[4] = {e4m3x2_to_f16x2(r[2 * h]), e4m3x2_to_f16x2(r[2 * h + 1]),
                                 e4m3x2_to_f16x2(r[2 * h] >> 16),
                                 e4m3x2_to_f16x2(r[2 * h + 1] >> 16)};
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_16816<__half>(sch[(kp + h) % NCH][nt], a, qb[kp + h][nt][0], qb[kp + h][nt][1]);
        }
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float v = sch[0][nt][e];
#pragma unroll
          for (int ch = 1; ch < NCH; ++ch) v += sch[ch][nt][e];
          sacc[nt][e] = v;
        }
      const int tok0 = t0 + ta;
      const bool unmasked = (t0 + C::kTile <= vis_min);
      bool grew = false;
      float alpha_o[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          float s0 = sacc[nt][cc] * fcol[nt][cc] * ska;
          float s1 = sacc[nt][2 + cc] * fcol[nt][cc] * skb;
          if (!unmasked) {
            s0 = (tok0 < vis[nt][cc]) ? s0 : -INFINITY;
            s1 = (tok0 + 8 < vis[nt][cc]) ? s1 : -INFINITY;
          }
          float mx = fmaxf(s0 + lca, s1 + lcb);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          const float m_new = fmaxf(m[nt][cc], mx);
          const float mu = (m_new == -INFINITY) ? 0.f : m_new;
          alpha_o[nt][cc] = exp2f(m[nt][cc] - mu);
          grew |= (m_new > m[nt][cc]);
          m[nt][cc] = m_new;
          // the sum l and the weights of O, both referenced to m
          const float e0 = exp2f(s0 - mu), e1 = exp2f(s1 - mu);
          l[nt][cc] = fmaf(l[nt][cc], alpha_o[nt][cc], e0 + e1);
          sacc[nt][cc] = e0 * vsa;
          sacc[nt][2 + cc] = e1 * vsb;
        }
      }
      if (__any_sync(0xffffffffu, grew)) {
#pragma unroll
        for (int mt = 0; mt < C::kMTiles; ++mt)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            o[mt][nt][0] *= alpha_o[nt][0];
            o[mt][nt][1] *= alpha_o[nt][1];
            o[mt][nt][2] *= alpha_o[nt][0];
            o[mt][nt][3] *= alpha_o[nt][1];
          }
      }
      uint32_t pb[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        pb[nt][0] = movmatrix_trans(f32x2_to_f16x2(sacc[nt][0], sacc[nt][1]));
        pb[nt][1] = movmatrix_trans(f32x2_to_f16x2(sacc[nt][2], sacc[nt][3]));
      }
      // O^T += V^T . P^T; V^T rows of m-tile kp + h come in vt_row_to_d order
#pragma unroll
      for (int kp = 0; kp < C::kKSteps; kp += 2) {
        uint32_t r[4];
        ldmatrix_x4(r, vb + swz8<D>(k_row, kp + k_cs));
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t a[4] = {movmatrix_trans(e4m3x2_to_f16x2(r[2 * h])),
                                 movmatrix_trans(e4m3x2_to_f16x2(r[2 * h] >> 16)),
                                 movmatrix_trans(e4m3x2_to_f16x2(r[2 * h + 1])),
                                 movmatrix_trans(e4m3x2_to_f16x2(r[2 * h + 1] >> 16))};
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_16816<__half>(o[kp + h][nt], a, pb[nt][0], pb[nt][1]);
        }
      }
    } else {
      float sacc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < C::kKSteps; ++kk) {
        uint32_t a[4];
        ldmatrix_x4(a, kb + k_rp + (kk >> 2) * half_stride + ((((2 * kk + k_cs) & 7) ^ k_sw) << 4));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_16816<T>(sacc[nt], a, qb[kk][nt][0], qb[kk][nt][1]);
      }
      const int tok0 = t0 + wrow + (lane >> 2);
      const bool unmasked = (t0 + C::kTile <= vis_min);
      bool grew = false;
      float alpha[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          float s0 = sacc[nt][cc] * p.scale_log2;
          float s1 = sacc[nt][2 + cc] * p.scale_log2;
          if (!unmasked) {
            s0 = (tok0 < vis[nt][cc]) ? s0 : -INFINITY;
            s1 = (tok0 + 8 < vis[nt][cc]) ? s1 : -INFINITY;
          }
          float mx = fmaxf(s0, s1);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          const float m_new = fmaxf(m[nt][cc], mx);
          const float mu = (m_new == -INFINITY) ? 0.f : m_new;
          alpha[nt][cc] = exp2f(m[nt][cc] - mu);
          grew |= (m_new > m[nt][cc]);
          m[nt][cc] = m_new;
          const float p0 = exp2f(s0 - mu);
          const float p1 = exp2f(s1 - mu);
          l[nt][cc] = fmaf(l[nt][cc], alpha[nt][cc], p0 + p1);
          sacc[nt][cc] = p0;
          sacc[nt][2 + cc] = p1;
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
#pragma unroll
      for (int mt = 0; mt < C::kMTiles; ++mt) {
        uint32_t a[4];
        ldmatrix_x4_trans(a, vb + v_rp + (mt >> 2) * half_stride + ((((2 * mt + v_cs) & 7) ^ v_sw) << 4));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_16816<T>(o[mt][nt], a, pb[nt][0], pb[nt][1]);
          if constexpr (SplitP<T>::kOn) mma_16816<T>(o[mt][nt], a, pl[nt][0], pl[nt][1]);
        }
      }
    }

    const bool piece_end = (j == ntiles - 1) || (cur.k == cur.seg_tiles - 1);
    if (!piece_end) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      cur.next(p, PAGED);
      continue;
    }

    // -------------------------------------------- end of a segment piece
    // The four warps merge inside this stage's K/V buffers (every warp is done
    // reading them after the barrier) into registers; then the stage is released
    // and refilled at once, so the ring keeps streaming while the piece's result
    // is written and its ticket taken.
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        l[nt][cc] += __shfl_xor_sync(0xffffffffu, l[nt][cc], 4);
        l[nt][cc] += __shfl_xor_sync(0xffffffffu, l[nt][cc], 8);
        l[nt][cc] += __shfl_xor_sync(0xffffffffu, l[nt][cc], 16);
      }
    named_barrier_sync(1, NTH);
    float* red_acc = reinterpret_cast<float*>(sk + st * C::kTileBytes);
    float* red_acc_hi = reinterpret_cast<float*>(sv + st * C::kTileBytes);
    auto acc_at = [&](int w, int row, int d) -> float* {
      // W*R*D floats spread over this stage's K then V buffers; the column is
      // swizzled by row bits 1-2 so that the fragment stores hit 32 distinct banks
      const int idx = (w * R + row) * D + (d ^ (((row >> 1) & 3) << 3));
      constexpr int kHalfFloats = C::kTileBytes / 4;
      return idx < kHalfFloats ? red_acc + idx : red_acc_hi + (idx - kHalfFloats);
    };
    // FP8: the rows of O come in vt_row_to_d order
#pragma unroll
    for (int mt = 0; mt < C::kMTiles; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int row = nt * 8 + (lane & 3) * 2 + (e & 1);
          const int rho = (lane >> 2) + (e >> 1) * 8;
          const int d = mt * 16 + (FP8 ? vt_row_to_d(rho) : rho);
          *acc_at(warp, row, d) = o[mt][nt][e];
        }
    if (lane < 4) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int row = nt * 8 + lane * 2 + cc;
          red_m[warp * R + row] = m[nt][cc];
          red_l[warp * R + row] = l[nt][cc];
        }
    }
    reset_state();
    named_barrier_sync(1, NTH);
    // per row, once: warp w's weight 2^(m_w - M) / l in red_m, the row's base-2
    // log-sum-exp M + log2 l in red_l[row] (a row that saw nothing: weights 0, -inf)
    if (tid < R) {
      const int rr = tid;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < W; ++w) M = fmaxf(M, red_m[w * R + rr]);
      float f[W];
      float lsum = 0.f;
#pragma unroll
      for (int w = 0; w < W; ++w) {
        f[w] = M == -INFINITY ? 0.f : exp2f(red_m[w * R + rr] - M);
        lsum = fmaf(red_l[w * R + rr], f[w], lsum);
      }
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll
      for (int w = 0; w < W; ++w) red_m[w * R + rr] = f[w] * inv;
      red_l[rr] = lsum > 0.f ? M + log2f(lsum) : -INFINITY;
    }
    named_barrier_sync(1, NTH);

    // element k of this thread: row (tid + k*NTH) / D, column (tid + k*NTH) % D
    constexpr int PER = R * D / NTH;
    float res[PER];  // the row's output (whole piece) or normalised partial
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int idx = tid + k * NTH;
      const int rr = idx / D;
      const int d = idx - rr * D;
      float ov = 0.f;
      if (rr < nr) {
#pragma unroll
        for (int w = 0; w < W; ++w) ov = fmaf(*acc_at(w, rr, d), red_m[w * R + rr], ov);
      }
      res[k] = ov;
    }
    named_barrier_sync(1, NTH);  // the stage is read: release and refill it
    if (lane == 0) mbar_arrive(&empty[st]);
    if (producer) refill(j + 1);
    // a ticket taken at an earlier piece end is settled now, while the ring streams
    if (pend) settle();

    const bool whole = (piece_first_j == j - cur.k) && (cur.k == cur.seg_tiles - 1);
    const int slot = (piece_first_j == 0) ? 0 : 1;
    T* out = static_cast<T*>(p.out);
    const size_t row_base =
        ((size_t)cur.b * p.H_q + (size_t)cur.g * p.group) * p.T_new + r0;
    float* wso = p.ws_o + ((size_t)c * 2 + slot) * p.sk_slot_rows * D;
    float* wsl = p.ws_lse + ((size_t)c * 2 + slot) * p.sk_slot_rows;
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int idx = tid + k * NTH;
      const int rr = idx / D;
      const int d = idx - rr * D;
      if (rr < nr) {
        if (whole) {
          store_elt<T>(out + (row_base + rr) * D + d, res[k]);
        } else {
          wso[rr * D + d] = res[k];
          if (d == 0) wsl[rr] = red_l[rr];
        }
      }
    }
    if (!whole) {
      // Hand the piece to the segment's last finisher: the barrier orders every
      // thread's partial stores before the release-acquire ticket, whose result is
      // read only at the next piece end or after the loop (settle()), so nobody
      // waits for it here.
      named_barrier_sync(1, NTH);
      pend = true;
      pend_s0 = cur.seg_start;
      const long long s1 = cur.seg_start + cur.seg_tiles - 1;
      pend_rf = rm.of(pend_s0);
      pend_rl = rm.of(s1);
      pend_nr = nr;
      pend_row_base = row_base;
      pend_ticket = p.counters + ((size_t)cur.b * p.H_kv + cur.g) * p.row_blocks + cur.rb;
      if (tid == kTicketThread) pend_count = ticket_add_acq_rel(pend_ticket);
    }
    cur.next(p, PAGED);
  }
  if (pend) settle();
  // After an abort, do not retire while copies may still be landing.
  if (producer && lane == 0 && *abort_word)
#pragma unroll 1
    for (int j = max(0, issued - C::kStages); j < issued; ++j)
      if (!mbar_wait(&full[j % C::kStages], (j / C::kStages) & 1, p.err, wait_limit)) break;
}

}  // namespace kvc
