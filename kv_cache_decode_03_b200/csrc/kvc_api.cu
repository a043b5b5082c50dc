// kvc_api.cu -- host side of libkvc: the cache object, argument checks, the
// split-K planner and kernel dispatch behind the C ABI of include/kvc.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "append.cuh"
#include "attend_decode.cuh"
#include "attend_fp8.cuh"
#include "attend_mma.cuh"
#include "attend_streamk.cuh"
#include "attend_tc.cuh"
#include "attend_tc_streamk.cuh"
#include "cache_ops.cuh"
#include "fp8.cuh"
#include "kvc.h"

struct kvc_cache {
  int B, H_kv, D, max_T, page_size, page_shift, num_layers, num_pages;
  kvc_dtype dtype;
  bool paged;
  size_t layer_bytes;  // one layer's K (equally V) pool
  char* pool;          // layers x {K, V}
  int* d_err;
  float* ws;           // split-K workspace: partial outputs and lse
  size_t ws_bytes;
  int* tickets;        // slice tickets, zero between launches (own allocation, so that
  size_t n_tickets;    // partial layouts of different plans can never overwrite them)
  bool fp8;                        // FP8 (E4M3) codes + per-(token, head) scales (fp8.cuh)
  float* scales;                   // fp8: layers x {K, V} x scale_floats
  size_t scale_floats;             // fp8: scales of one layer's K (equally V)
  int T_pad;                       // fp8, contiguous: scale row length (whole 64-token tiles)
  bool tma;                        // tensor maps built: the tensor-core path is available
  std::vector<CUtensorMap> tmk;    // per layer: K pool as a 2-D (rows, D) tensor
  std::vector<CUtensorMap> tmv;
  bool tma4;                       // 4-D paged maps for the stream-K kernel (D 128, pages < 64)
  std::vector<CUtensorMap> tmk4;   // per layer: (64 elements, page tokens, 2 halves, blocks)
  std::vector<CUtensorMap> tmv4;
  int device;
  int num_sms;
  bool dependent_launch;           // stream-K launches with programmatic stream serialization
  unsigned long long wait_limit_ns;  // bound of the kernels' pipeline waits (0: 1 s)
  bool stall_next;                 // failure-detection test: next attend issues no copies
  bool replan_next;                // dependent-launch test: next stream-K attend replans
};

namespace {

constexpr int kEltBytes = 2;

// TMA L2 promotion: a 128-byte box column pulls the neighbouring half of the
// 256-byte K/V row into L2, where the other column's load finds it.
#ifndef KVC_TMA_L2_PROMOTION
#define KVC_TMA_L2_PROMOTION CU_TENSOR_MAP_L2_PROMOTION_L2_256B
#endif

// Query rows per KV head from which the tensor-core kernels take over from the CUDA-core
// kernel (where tensor maps exist: D 64 or 128, pages of 8 or more tokens).
#ifndef KVC_MMA_MIN_ROWS
#define KVC_MMA_MIN_ROWS 1
#endif

// Query rows per KV head from which the tcgen05 kernel (128-row blocks) takes over.  From
// 17 rows the persistent tcgen05 kernel beats the mma.sync kernels even with most of the
// MMA's 128 rows idle (GQA verify gamma 8, 32 rows: 69 % of HBM against 33 % on the
// fixed-split mma.sync kernel); up to 16 rows the mma.sync stream-K kernel is faster.
#ifndef KVC_TC_MIN_ROWS
#define KVC_TC_MIN_ROWS 17
#endif

// Split-K sizing: aim for this many waves of resident CTAs, so that the last
// wave's imbalance is a small fraction of the pass.
#ifndef KVC_SPLIT_WAVES
#define KVC_SPLIT_WAVES 4
#endif
#ifndef KVC_TC_COMBINE  // tcgen05 stream-K: partial pieces merged by a separate combine launch
#define KVC_TC_COMBINE 1
#endif
// ... when a segment's partials average more than this many bytes: one CTA merging them
// in the attend kernel takes ~20 us at 600 KB (a trace); the combine launch, with 4 rows a
// block, was measured on MQA verify at gamma 2 / 4 / 8 (300 / 600 / 300 KB a segment):
// +12 / +14 / +5 % a step, and flat on GQA verify gamma 8 (19 KB a segment)
#ifndef KVC_TC_COMBINE_MIN_BYTES
#define KVC_TC_COMBINE_MIN_BYTES (64 << 10)
#endif
#ifndef KVC_TC_RB_MAJOR
#define KVC_TC_RB_MAJOR 1
#endif
#ifndef KVC_FP8_STREAMK  // FP8, 1-8 rows per KV head, no window: the stream-K kernel
#define KVC_FP8_STREAMK 1
#endif
#ifndef KVC_SK_PENALTY_FP8  // its per-piece cost in virtual tiles
#define KVC_SK_PENALTY_FP8 3
#endif
#ifndef KVC_FP8_SPLIT_WAVES  // the FP8 kernel's tiles are cheaper to load: fewer, longer slices
#define KVC_FP8_SPLIT_WAVES 4
#endif
// A tcgen05 slice carries a large fixed cost (TMEM allocation, 32 KB of Q staged, the
// pipeline fill, its part of the merge): plan two waves and slices of at least 16 tiles.
// Measured against 4, 8 and 16 waves, 1 wave, and a model fitting whole waves, this was
// best or close on the MQA verify and MHA prefill-chunk workloads.
#ifndef KVC_TC_SPLIT_WAVES
#define KVC_TC_SPLIT_WAVES 2
#endif
#ifndef KVC_TC_MIN_SLICE_TILES
#define KVC_TC_MIN_SLICE_TILES 16
#endif
// Stream-K: virtual tiles charged per segment a CTA enters (the fixed cost of a piece:
// epilogue, ticket, a fresh q and a ring restart, measured at about two to four tiles'
// streaming time), so CTAs that cross segment boundaries get fewer real tiles.
#ifndef KVC_SK_PENALTY_D128
#define KVC_SK_PENALTY_D128 4
#endif
#ifndef KVC_SK_PENALTY_D64
#define KVC_SK_PENALTY_D64 4
#endif
// tcgen05 rows (64+ per KV head) without a window run on the persistent stream-K
// tcgen05 kernel; its penalty tiles charge a piece's Q reload, TMEM readout and partial.
#ifndef KVC_TC_STREAMK
#define KVC_TC_STREAMK 1
#endif
// Resident CTAs per SM the persistent tcgen05 grid assumes at least: the occupancy query
// reports 1 for this 224-thread kernel although registers, shared memory and TMEM hold two,
// and two do co-reside (MQA verify gamma 8: 24.6 % of HBM with 296 CTAs, 17.6 % with 148).
#ifndef KVC_TC_MIN_OCC
#define KVC_TC_MIN_OCC 2
#endif
#ifndef KVC_TC_SK_PENALTY
#define KVC_TC_SK_PENALTY 3
#endif
// Stream-K on paged D = 128 caches with pages under 64 tokens: one 4-D box per page.
#ifndef KVC_SK_BLOCKED_PAGES
#define KVC_SK_BLOCKED_PAGES 1
#endif

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int log2_exact(int v) {
  int s = 0;
  while ((1 << s) < v) ++s;
  return (1 << s) == v ? s : -1;
}

kvc_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return KVC_OK;
  if (e == cudaErrorMemoryAllocation) return KVC_ERR_OOM;
  return KVC_ERR_CUDA;
}

int tile_tokens(int D) {
  switch (D) {
    case 32: return kvc::DecodeCfg<32>::kTile;
    case 64: return kvc::DecodeCfg<64>::kTile;
    default: return kvc::DecodeCfg<128>::kTile;
  }
}

// ------------------------------------------------------------- tensor maps
// The pools are addressed by TMA as 2-D tensors of rows x D elements: rows are
// (b, g, position) for a contiguous cache and (page, g, slot) for a paged one.
// Boxes are 64 elements (128 bytes, the swizzle span) by up to 64 rows.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    else
      cudaGetLastError();
  });
  return fn;
}

bool make_tmap(CUtensorMap* m, void* base, kvc_dtype dtype, int D, long long rows, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * kEltBytes};
  const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = fn(m,
                        dtype == KVC_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                          : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, KVC_TMA_L2_PROMOTION,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Paged pools with D = 128 and pages of fewer than 64 tokens, for the stream-K kernel: a
// 4-D view (64 elements, P tokens, 2 halves, num_pages x H_kv blocks) whose box is a whole
// (page, head) block, landing in shared memory as [half][token] rows of 128 bytes.
bool make_tmap_blocked(CUtensorMap* m, void* base, kvc_dtype dtype, int P, long long blocks) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {64u, (cuuint64_t)P, 2u, (cuuint64_t)blocks};
  const cuuint64_t strides[3] = {128u * kEltBytes, 64u * kEltBytes,
                                 (cuuint64_t)P * 128u * kEltBytes};
  const cuuint32_t box[4] = {64u, (cuuint32_t)P, 2u, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  const CUresult r = fn(m,
                        dtype == KVC_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                          : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, KVC_TMA_L2_PROMOTION,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// FP8 code pools: 2-D (rows, D) bytes, one D-byte row per box row, swizzled across the
// row's 16-byte chunks (128-byte swizzle for D = 128, 64-byte for D = 64) so that the
// kernel's ldmatrix reads are conflict-free.
bool make_tmap_fp8(CUtensorMap* m, void* base, int D, long long rows, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D};
  const cuuint32_t box[2] = {(cuuint32_t)D, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                        KVC_TMA_L2_PROMOTION, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

void build_tmaps(kvc_cache* c) {
  c->tma = false;
  if (c->fp8) {
    const long long rows = c->paged ? (long long)c->num_pages * c->H_kv * c->page_size
                                    : (long long)c->B * c->H_kv * c->max_T;
    if (rows + 64 >= (1LL << 31)) return;
    const int box_rows = c->paged ? std::min(c->page_size, 64) : 64;
    c->tmk.resize(c->num_layers);
    c->tmv.resize(c->num_layers);
    for (int l = 0; l < c->num_layers; ++l)
      if (!make_tmap_fp8(&c->tmk[l], c->pool + (size_t)(2 * l) * c->layer_bytes, c->D, rows,
                         box_rows) ||
          !make_tmap_fp8(&c->tmv[l], c->pool + (size_t)(2 * l + 1) * c->layer_bytes, c->D, rows,
                         box_rows))
        return;
    c->tma = true;
    return;
  }
  if (c->D != 64 && c->D != 128) return;
  if (c->paged && c->page_size < 8) return;  // boxes must start on 1024-byte swizzle atoms
  const long long rows = c->paged ? (long long)c->num_pages * c->H_kv * c->page_size
                                  : (long long)c->B * c->H_kv * c->max_T;
  if (rows + 64 >= (1LL << 31)) return;  // TMA coordinates are 32-bit
  const int box_rows = c->paged ? std::min(c->page_size, 64) : 64;
  c->tmk.resize(c->num_layers);
  c->tmv.resize(c->num_layers);
  for (int l = 0; l < c->num_layers; ++l) {
    if (!make_tmap(&c->tmk[l], c->pool + (size_t)(2 * l) * c->layer_bytes, c->dtype, c->D,
                   rows, box_rows) ||
        !make_tmap(&c->tmv[l], c->pool + (size_t)(2 * l + 1) * c->layer_bytes, c->dtype, c->D,
                   rows, box_rows))
      return;
  }
  c->tma = true;
  c->tma4 = false;
  if (KVC_SK_BLOCKED_PAGES && c->paged && c->D == 128 && c->page_size < 64) {
    const long long blocks = (long long)c->num_pages * c->H_kv;
    c->tmk4.resize(c->num_layers);
    c->tmv4.resize(c->num_layers);
    for (int l = 0; l < c->num_layers; ++l)
      if (!make_tmap_blocked(&c->tmk4[l], c->pool + (size_t)(2 * l) * c->layer_bytes, c->dtype,
                             c->page_size, blocks) ||
          !make_tmap_blocked(&c->tmv4[l], c->pool + (size_t)(2 * l + 1) * c->layer_bytes,
                             c->dtype, c->page_size, blocks))
        return;  // the stream-K kernel keeps the 2-D maps
    c->tma4 = true;
  }
}

template <int D, int NT, typename T, bool PAGED>
int mma_occupancy() {
  static int occ = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    const size_t smem = kvc::MmaCfg<D>::template smem_bytes<NT>();
    cudaFuncSetAttribute(kvc::attend_mma_kernel<D, NT, T, PAGED>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &n, kvc::attend_mma_kernel<D, NT, T, PAGED>, kvc::MmaCfg<D>::kThreads, smem) !=
        cudaSuccess)
      n = 1;
    occ = std::max(1, n);
  });
  return occ;
}

template <int D, typename T, bool PAGED>
int mma_occ_nt(int NT) {
  switch (NT) {
    case 1: return mma_occupancy<D, 1, T, PAGED>();
    case 2: return mma_occupancy<D, 2, T, PAGED>();
    default: return mma_occupancy<D, 4, T, PAGED>();
  }
}

template <typename T>
int mma_occ(int D, int NT, bool paged) {
  if (D == 64) return paged ? mma_occ_nt<64, T, true>(NT) : mma_occ_nt<64, T, false>(NT);
  return paged ? mma_occ_nt<128, T, true>(NT) : mma_occ_nt<128, T, false>(NT);
}

template <int D, int NT, typename T, bool PAGED, bool FP8 = false>
int streamk_occupancy() {
  static int occ = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    const size_t smem = kvc::StreamKCfg<D, FP8>::template smem_bytes<NT>();
    cudaFuncSetAttribute(kvc::attend_streamk_kernel<D, NT, T, PAGED, FP8>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &n, kvc::attend_streamk_kernel<D, NT, T, PAGED, FP8>,
            kvc::StreamKCfg<D, FP8>::kThreads, smem) != cudaSuccess)
      n = 1;
    occ = std::max(1, n);
  });
  return occ;
}

// the FP8 variant: one row group of 8, bf16 queries
int streamk_fp8_occ(int D, bool paged) {
  using T = __nv_bfloat16;
  if (D == 64)
    return paged ? streamk_occupancy<64, 1, T, true, true>()
                 : streamk_occupancy<64, 1, T, false, true>();
  return paged ? streamk_occupancy<128, 1, T, true, true>()
               : streamk_occupancy<128, 1, T, false, true>();
}

template <typename T>
int streamk_occ(int D, int NT, bool paged) {
  if (D == 64)
    return paged ? (NT == 1 ? streamk_occupancy<64, 1, T, true>()
                            : streamk_occupancy<64, 2, T, true>())
                 : (NT == 1 ? streamk_occupancy<64, 1, T, false>()
                            : streamk_occupancy<64, 2, T, false>());
  return paged ? (NT == 1 ? streamk_occupancy<128, 1, T, true>()
                          : streamk_occupancy<128, 2, T, true>())
               : (NT == 1 ? streamk_occupancy<128, 1, T, false>()
                          : streamk_occupancy<128, 2, T, false>());
}

template <int D, typename T, bool PAGED>
int tc_occupancy() {
  static int occ = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    const size_t smem = kvc::TcCfg<D>::smem_bytes();
    cudaFuncSetAttribute(kvc::attend_tc_kernel<D, T, PAGED>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &n, kvc::attend_tc_kernel<D, T, PAGED>, kvc::TcCfg<D>::kThreads, smem) !=
        cudaSuccess)
      n = 1;
    // every resident CTA holds TMEM columns: never more than the 512 an SM has
    occ = std::max(1, std::min(n, 512 / kvc::TcCfg<D>::kTmemCols));
  });
  return occ;
}

template <typename T>
int tc_occ(int D, bool paged) {
  if (D == 64) return paged ? tc_occupancy<64, T, true>() : tc_occupancy<64, T, false>();
  return paged ? tc_occupancy<128, T, true>() : tc_occupancy<128, T, false>();
}

template <int D, typename T, bool PAGED>
int tc_sk_occupancy() {
  static int occ = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    const size_t smem = kvc::TcSkCfg<D>::smem_bytes();
    cudaFuncSetAttribute(kvc::attend_tc_streamk_kernel<D, T, PAGED>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &n, kvc::attend_tc_streamk_kernel<D, T, PAGED>, kvc::TcCfg<D>::kThreads, smem) !=
        cudaSuccess)
      n = 1;
    // every resident CTA holds TMEM columns: never more than the 512 an SM has
    occ = std::max(1, std::min(std::max(n, KVC_TC_MIN_OCC), 512 / kvc::TcCfg<D>::kTmemCols));
  });
  return occ;
}

template <typename T>
int tc_sk_occ(int D, bool paged) {
  if (D == 64) return paged ? tc_sk_occupancy<64, T, true>() : tc_sk_occupancy<64, T, false>();
  return paged ? tc_sk_occupancy<128, T, true>() : tc_sk_occupancy<128, T, false>();
}

template <int D, int NT, bool PAGED>
int fp8_occupancy() {
  static int occ = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    const size_t smem = kvc::Fp8Cfg<D>::template smem_bytes<NT>();
    cudaFuncSetAttribute(kvc::attend_fp8_kernel<D, NT, PAGED>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &n, kvc::attend_fp8_kernel<D, NT, PAGED>, kvc::Fp8Cfg<D>::kThreads, smem) !=
        cudaSuccess)
      n = 1;
    occ = std::max(1, n);
  });
  return occ;
}

template <int D, bool PAGED>
int fp8_occ_nt(int NT) {
  switch (NT) {
    case 1: return fp8_occupancy<D, 1, PAGED>();
    case 2: return fp8_occupancy<D, 2, PAGED>();
    default: return fp8_occupancy<D, 4, PAGED>();
  }
}

int fp8_occ(int D, int NT, bool paged) {
  if (D == 64) return paged ? fp8_occ_nt<64, true>(NT) : fp8_occ_nt<64, false>(NT);
  return paged ? fp8_occ_nt<128, true>(NT) : fp8_occ_nt<128, false>(NT);
}

int fp8_scratch_floats(int D, int NT) {
  if (D == 64)
    return NT == 1 ? kvc::Fp8Cfg<64>::scratch_floats<1>()
                   : NT == 2 ? kvc::Fp8Cfg<64>::scratch_floats<2>()
                             : kvc::Fp8Cfg<64>::scratch_floats<4>();
  return NT == 1 ? kvc::Fp8Cfg<128>::scratch_floats<1>()
                 : NT == 2 ? kvc::Fp8Cfg<128>::scratch_floats<2>()
                           : kvc::Fp8Cfg<128>::scratch_floats<4>();
}

int mma_scratch_floats(int D, int NT) {
  if (D == 64)
    return NT == 1 ? kvc::MmaCfg<64>::scratch_floats<1>()
                   : NT == 2 ? kvc::MmaCfg<64>::scratch_floats<2>()
                             : kvc::MmaCfg<64>::scratch_floats<4>();
  return NT == 1 ? kvc::MmaCfg<128>::scratch_floats<1>()
                 : NT == 2 ? kvc::MmaCfg<128>::scratch_floats<2>()
                           : kvc::MmaCfg<128>::scratch_floats<4>();
}

// ------------------------------------------------------------ attend plan
struct Plan {
  bool fp8;          // FP8 cache: attend_fp8_kernel (fixed split, NT 8-row n-tiles)
  bool tc;           // tcgen05 kernel, 128 query rows per CTA
  bool mma;          // mma.sync tensor-core kernel (else the CUDA-core kernel)
  bool streamk;      // mma: persistent stream-K kernel (grid = resident CTAs)
  bool combine;      // tcgen05 stream-K: segments merged by a separate combine launch
  int grid;          // streamk: persistent CTAs
  size_t slots;      // streamk: partial-result slots (slot_rows rows x D each) in the workspace
  int slot_rows;     // streamk: rows of a slot
  int NT;            // mma: 8-row n-tiles per CTA
  int R;             // query rows per CTA
  int row_blocks;    // CTAs per KV head along the rows
  int split_tokens;  // tokens per split-K slice
  int num_splits;
  size_t ws_partial_floats;  // partial outputs + lse
  size_t ws_counters;        // slice tickets
  size_t ws_bytes;
};

template <int D, int R, typename T, bool PAGED>
int simt_occupancy() {
  static int occ = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    const size_t smem = kvc::DecodeCfg<D>::template smem_bytes<R>();
    cudaFuncSetAttribute(kvc::attend_decode_kernel<D, R, T, PAGED>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &n, kvc::attend_decode_kernel<D, R, T, PAGED>, kvc::DecodeCfg<D>::kThreads, smem) !=
        cudaSuccess)
      n = 1;
    occ = std::max(1, n);
  });
  return occ;
}

template <int D, typename T, bool PAGED>
int occupancy_for(int R) {
  switch (R) {
    case 1: return simt_occupancy<D, 1, T, PAGED>();
    case 2: return simt_occupancy<D, 2, T, PAGED>();
    default: return simt_occupancy<D, 4, T, PAGED>();
  }
}

template <int D, typename T>
int occupancy_for(int R, bool paged) {
  return paged ? occupancy_for<D, T, true>(R) : occupancy_for<D, T, false>(R);
}

template <typename T>
int occupancy_for(int D, int R, bool paged) {
  switch (D) {
    case 32: return occupancy_for<32, T>(R, paged);
    case 64: return occupancy_for<64, T>(R, paged);
    default: return occupancy_for<128, T>(R, paged);
  }
}

int occupancy(const kvc_cache* c, int R) {
  return c->dtype == KVC_BF16 ? occupancy_for<__nv_bfloat16>(c->D, R, c->paged)
                              : occupancy_for<__half>(c->D, R, c->paged);
}

// window / sink: sliding-window attention (window.cuh); 0 = full attention.
Plan make_plan(const kvc_cache* c, int H_q, int T_new, int max_pages, int window = 0,
               int sink = 0) {
  Plan pl{};
  const int rows = (H_q / c->H_kv) * T_new;
  // Tensor cores from KVC_MMA_MIN_ROWS query rows per K/V row (mma.sync), tcgen05 from
  // KVC_TC_MIN_ROWS (a 128-row block as the MMA's M).
  pl.fp8 = c->fp8;
  pl.tc = !c->fp8 && c->tma && rows >= KVC_TC_MIN_ROWS;
  pl.mma = !c->fp8 && c->tma && rows >= KVC_MMA_MIN_ROWS && !pl.tc;
  int tile, occ, scratch = 1 << 30;
  if (pl.fp8) {
    pl.NT = rows <= 8 ? 1 : (rows <= 16 ? 2 : 4);
    pl.R = pl.NT * 8;
    tile = kvc::Fp8Cfg<64>::kTile;
    occ = fp8_occ(c->D, pl.NT, c->paged);
    scratch = fp8_scratch_floats(c->D, pl.NT);
  } else if (pl.tc) {
    pl.NT = 0;
    pl.R = kvc::TcCfg<64>::kRows;
    tile = kvc::TcCfg<64>::kTile;
    occ = c->dtype == KVC_BF16 ? tc_occ<__nv_bfloat16>(c->D, c->paged)
                               : tc_occ<__half>(c->D, c->paged);
    scratch = c->D == 64 ? kvc::TcCfg<64>::kScratchFloats : kvc::TcCfg<128>::kScratchFloats;
  } else if (pl.mma) {
    pl.NT = rows <= 8 ? 1 : (rows <= 16 ? 2 : 4);
    pl.R = pl.NT * 8;
    tile = 64;
    occ = c->dtype == KVC_BF16 ? mma_occ<__nv_bfloat16>(c->D, pl.NT, c->paged)
                               : mma_occ<__half>(c->D, pl.NT, c->paged);
    scratch = mma_scratch_floats(c->D, pl.NT);
  } else {
    pl.NT = 0;
    pl.R = rows == 1 ? 1 : (rows == 2 ? 2 : 4);
    tile = tile_tokens(c->D);
    occ = occupancy(c, pl.R);
  }
  pl.row_blocks = kvc::ceil_div(rows, pl.R);
  // Persistent stream-K for up to 16 rows per KV head: the per-CTA partial
  // slots need no split size and every CTA streams the same bytes.
  long long cap = c->max_T;
  if (c->paged) cap = std::min<long long>(cap, (long long)max_pages * c->page_size);
  const int tc_max_batch = c->D == 64 ? kvc::TcSkCfg<64>::kMaxBatch
                                      : kvc::TcSkCfg<128>::kMaxBatch;
  if (KVC_TC_STREAMK && pl.tc && c->B <= tc_max_batch && window == 0) {
    pl.streamk = true;
    const int socc = c->dtype == KVC_BF16 ? tc_sk_occ<__nv_bfloat16>(c->D, c->paged)
                                          : tc_sk_occ<__half>(c->D, c->paged);
    // no more CTAs than there can be tiles (penalties included)
    const long long wt_max = (long long)c->B * c->H_kv * pl.row_blocks *
                             ((cap + tile - 1) / tile + KVC_TC_SK_PENALTY);
    pl.grid = (int)std::max<long long>(1, std::min<long long>((long long)c->num_sms * socc,
                                                              wt_max));
    pl.slots = (size_t)pl.grid * 2;
    pl.slot_rows = std::min(pl.R, rows);  // no more rows of a block can be valid
    pl.split_tokens = 1 << 30;
    pl.num_splits = 1;
    pl.ws_partial_floats = pl.slots * pl.slot_rows * (c->D + 1);
    pl.ws_counters = (size_t)c->B * c->H_kv * pl.row_blocks;
    pl.combine = KVC_TC_COMBINE && (double)pl.grid / pl.ws_counters * pl.slot_rows * c->D *
                                           sizeof(float) > (double)KVC_TC_COMBINE_MIN_BYTES;
    // partial outputs, lse, then (combine launch) one descriptor a segment
    pl.ws_bytes = pl.ws_partial_floats * sizeof(float) +
                  (pl.combine ? pl.ws_counters * kvc::kCombineDescInts * sizeof(int) : 0);
    return pl;
  }
  const int fp8_max_batch = c->D == 64 ? kvc::StreamKCfg<64, true>::kMaxBatch
                                       : kvc::StreamKCfg<128, true>::kMaxBatch;
  if (KVC_FP8_STREAMK && pl.fp8 && pl.NT == 1 && c->B <= fp8_max_batch && window == 0) {
    pl.streamk = true;  // the stream-K kernel with E4M3 stages
    pl.grid = c->num_sms * streamk_fp8_occ(c->D, c->paged);
    pl.slots = (size_t)pl.grid * 2;
    pl.slot_rows = pl.R;
    pl.split_tokens = 1 << 30;
    pl.num_splits = 1;
    pl.ws_partial_floats = pl.slots * pl.slot_rows * (c->D + 1);
    pl.ws_counters = (size_t)c->B * c->H_kv * pl.row_blocks;
    pl.ws_bytes = pl.ws_partial_floats * sizeof(float);
    return pl;
  }
  const int max_batch = c->D == 64 ? kvc::StreamKCfg<64>::kMaxBatch
                                   : kvc::StreamKCfg<128>::kMaxBatch;
  if (pl.mma && pl.NT <= 2 && c->B <= max_batch && window == 0) {
    pl.streamk = true;
    const int socc = c->dtype == KVC_BF16 ? streamk_occ<__nv_bfloat16>(c->D, pl.NT, c->paged)
                                          : streamk_occ<__half>(c->D, pl.NT, c->paged);
    pl.grid = c->num_sms * socc;
    pl.slots = (size_t)pl.grid * 2;
    pl.slot_rows = pl.R;
    pl.split_tokens = 1 << 30;  // unused by the stream-K kernel
    pl.num_splits = 1;
    pl.ws_partial_floats = pl.slots * pl.slot_rows * (c->D + 1);
    pl.ws_counters = (size_t)c->B * c->H_kv * pl.row_blocks;
    pl.ws_bytes = pl.ws_partial_floats * sizeof(float);
    return pl;
  }
  if (window > 0)  // a block reads at most its sink tiles and W + T_new positions (+ a tile)
    cap = std::min<long long>(cap, (long long)(sink + tile - 1) / tile * tile + window + T_new +
                                       tile);
  cap = std::max<long long>(cap, 1);
  const long long units = (long long)c->B * c->H_kv * pl.row_blocks;
  const long long target =
      (long long)(pl.fp8 ? KVC_FP8_SPLIT_WAVES : pl.tc ? KVC_TC_SPLIT_WAVES : KVC_SPLIT_WAVES) *
      c->num_sms * occ;
  // the merging CTA keeps one weight per (row, slice) in shared memory
  const long long max_ns = std::min<long long>((cap + tile - 1) / tile, scratch / pl.R);
  long long ns = std::min(std::max((target + units - 1) / units, 1LL), max_ns);
  if (pl.tc)
    ns = std::max(1LL, std::min(ns, cap / ((long long)KVC_TC_MIN_SLICE_TILES * tile)));
  long long S = (cap + ns - 1) / ns;
  S = (S + tile - 1) / tile * tile;
  ns = (cap + S - 1) / S;
  pl.split_tokens = (int)S;
  pl.num_splits = (int)ns;
  pl.ws_partial_floats = ns > 1 ? (size_t)c->B * H_q * T_new * ns * (c->D + 1) : 0;
  pl.ws_counters = ns > 1 ? (size_t)c->B * c->H_kv * pl.row_blocks : 0;
  pl.ws_bytes = pl.ws_partial_floats * sizeof(float);
  return pl;
}

// Grow the tickets to `n` (zero-filled) and the partial workspace to `bytes`.
kvc_status ensure_workspace(kvc_cache* c, size_t bytes, size_t n) {
  if (n > c->n_tickets) {
    if (c->tickets) {
      cudaError_t e = cudaFree(c->tickets);  // synchronises
      c->tickets = nullptr;
      c->n_tickets = 0;
      if (e != cudaSuccess) return cuda_status(e);
    }
    void* t = nullptr;
    if (cudaMalloc(&t, n * sizeof(int)) != cudaSuccess) {
      cudaGetLastError();
      return KVC_ERR_OOM;
    }
    if (cudaMemset(t, 0, n * sizeof(int)) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
      cudaGetLastError();
      cudaFree(t);
      return KVC_ERR_CUDA;
    }
    c->tickets = static_cast<int*>(t);
    c->n_tickets = n;
  }
  if (bytes <= c->ws_bytes) return KVC_OK;
  if (c->ws) {
    cudaError_t e = cudaFree(c->ws);  // synchronises: no launch still reads it
    c->ws = nullptr;
    c->ws_bytes = 0;
    if (e != cudaSuccess) return cuda_status(e);
  }
  void* p = nullptr;
  cudaError_t e = cudaMalloc(&p, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return KVC_ERR_OOM;
  }
  c->ws = static_cast<float*>(p);
  c->ws_bytes = bytes;
  return KVC_OK;
}

// --------------------------------------------------------------- dispatch
template <int D, int NT, typename T, bool PAGED>
kvc_status launch_attend_mma(const kvc::AttendParams& p, const CUtensorMap& tk,
                             const CUtensorMap& tv, cudaStream_t stream) {
  using C = kvc::MmaCfg<D>;
  mma_occupancy<D, NT, T, PAGED>();  // sets the shared-memory attribute once
  const size_t smem = C::template smem_bytes<NT>();
  dim3 grid(p.num_splits * p.row_blocks, p.H_kv, p.B);
  kvc::attend_mma_kernel<D, NT, T, PAGED><<<grid, C::kThreads, smem, stream>>>(p, tk, tv);
  return cuda_status(cudaGetLastError());
}

template <int D, typename T, bool PAGED>
kvc_status dispatch_mma_nt(const kvc::AttendParams& p, int NT, const CUtensorMap& tk,
                           const CUtensorMap& tv, cudaStream_t s) {
  switch (NT) {
    case 1: return launch_attend_mma<D, 1, T, PAGED>(p, tk, tv, s);
    case 2: return launch_attend_mma<D, 2, T, PAGED>(p, tk, tv, s);
    default: return launch_attend_mma<D, 4, T, PAGED>(p, tk, tv, s);
  }
}

template <typename T>
kvc_status dispatch_mma(const kvc::AttendParams& p, int D, int NT, bool paged,
                        const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t s) {
  if (D == 64)
    return paged ? dispatch_mma_nt<64, T, true>(p, NT, tk, tv, s)
                 : dispatch_mma_nt<64, T, false>(p, NT, tk, tv, s);
  return paged ? dispatch_mma_nt<128, T, true>(p, NT, tk, tv, s)
               : dispatch_mma_nt<128, T, false>(p, NT, tk, tv, s);
}

// Dependent launch of the stream-K kernel is on unless KVC_PDL=0 (read once).
static bool dependent_launch_enabled() {
  static const bool on = [] {
    const char* v = getenv("KVC_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

template <int D, int NT, typename T, bool PAGED, bool FP8 = false>
kvc_status launch_attend_streamk(const kvc::AttendParams& p, int grid, bool pdl,
                                 const CUtensorMap& tk, const CUtensorMap& tv,
                                 cudaStream_t stream) {
  using C = kvc::StreamKCfg<D, FP8>;
  streamk_occupancy<D, NT, T, PAGED, FP8>();  // sets the shared-memory attribute once
  const size_t smem = C::template smem_bytes<NT>();
  // Programmatic stream serialization: the kernel may start while the grid
  // ahead of it retires; it waits for that grid (griddepcontrol.wait) before
  // its first read that counts or any write.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cuda_status(
      cudaLaunchKernelEx(&cfg, kvc::attend_streamk_kernel<D, NT, T, PAGED, FP8>, p, tk, tv));
}

kvc_status dispatch_streamk_fp8(const kvc::AttendParams& p, int D, bool paged, int grid,
                                bool pdl, const CUtensorMap& tk, const CUtensorMap& tv,
                                cudaStream_t s) {
  using T = __nv_bfloat16;
  if (D == 64)
    return paged ? launch_attend_streamk<64, 1, T, true, true>(p, grid, pdl, tk, tv, s)
                 : launch_attend_streamk<64, 1, T, false, true>(p, grid, pdl, tk, tv, s);
  return paged ? launch_attend_streamk<128, 1, T, true, true>(p, grid, pdl, tk, tv, s)
               : launch_attend_streamk<128, 1, T, false, true>(p, grid, pdl, tk, tv, s);
}

template <typename T>
kvc_status dispatch_streamk(const kvc::AttendParams& p, int D, int NT, bool paged, int grid,
                            bool pdl, const CUtensorMap& tk, const CUtensorMap& tv,
                            cudaStream_t s) {
  if (D == 64) {
    if (paged)
      return NT == 1 ? launch_attend_streamk<64, 1, T, true>(p, grid, pdl, tk, tv, s)
                     : launch_attend_streamk<64, 2, T, true>(p, grid, pdl, tk, tv, s);
    return NT == 1 ? launch_attend_streamk<64, 1, T, false>(p, grid, pdl, tk, tv, s)
                   : launch_attend_streamk<64, 2, T, false>(p, grid, pdl, tk, tv, s);
  }
  if (paged)
    return NT == 1 ? launch_attend_streamk<128, 1, T, true>(p, grid, pdl, tk, tv, s)
                   : launch_attend_streamk<128, 2, T, true>(p, grid, pdl, tk, tv, s);
  return NT == 1 ? launch_attend_streamk<128, 1, T, false>(p, grid, pdl, tk, tv, s)
                 : launch_attend_streamk<128, 2, T, false>(p, grid, pdl, tk, tv, s);
}

template <int D, int R, typename T, bool PAGED>
kvc_status launch_attend_simt(const kvc::AttendParams& p, cudaStream_t stream) {
  using C = kvc::DecodeCfg<D>;
  simt_occupancy<D, R, T, PAGED>();  // sets the shared-memory attribute once
  const size_t smem = C::template smem_bytes<R>();
  dim3 grid(p.num_splits * p.row_blocks, p.H_kv, p.B);
  kvc::attend_decode_kernel<D, R, T, PAGED><<<grid, C::kThreads, smem, stream>>>(p);
  return cuda_status(cudaGetLastError());
}

template <int D, typename T, bool PAGED>
kvc_status dispatch_r(const kvc::AttendParams& p, int R, cudaStream_t s) {
  switch (R) {
    case 1: return launch_attend_simt<D, 1, T, PAGED>(p, s);
    case 2: return launch_attend_simt<D, 2, T, PAGED>(p, s);
    default: return launch_attend_simt<D, 4, T, PAGED>(p, s);
  }
}

template <int D, typename T>
kvc_status dispatch_paged(const kvc::AttendParams& p, int R, bool paged, cudaStream_t s) {
  return paged ? dispatch_r<D, T, true>(p, R, s) : dispatch_r<D, T, false>(p, R, s);
}

template <typename T>
kvc_status dispatch_d(const kvc::AttendParams& p, int D, int R, bool paged, cudaStream_t s) {
  switch (D) {
    case 32: return dispatch_paged<32, T>(p, R, paged, s);
    case 64: return dispatch_paged<64, T>(p, R, paged, s);
    default: return dispatch_paged<128, T>(p, R, paged, s);
  }
}

template <int D, typename T, bool PAGED>
kvc_status launch_attend_tc(const kvc::AttendParams& p, const CUtensorMap& tk,
                            const CUtensorMap& tv, cudaStream_t stream) {
  using C = kvc::TcCfg<D>;
  tc_occupancy<D, T, PAGED>();  // sets the shared-memory attribute once
  dim3 grid(p.num_splits * p.row_blocks, p.H_kv, p.B);
  kvc::attend_tc_kernel<D, T, PAGED><<<grid, C::kThreads, C::smem_bytes(), stream>>>(p, tk, tv);
  return cuda_status(cudaGetLastError());
}

template <int D, typename T, bool PAGED>
kvc_status launch_attend_tc_streamk(const kvc::AttendParams& p, int grid, bool pdl,
                                    const CUtensorMap& tk, const CUtensorMap& tv,
                                    cudaStream_t stream) {
  tc_sk_occupancy<D, T, PAGED>();  // sets the shared-memory attribute once
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kvc::TcCfg<D>::kThreads);
  cfg.dynamicSmemBytes = kvc::TcSkCfg<D>::smem_bytes();
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cuda_status(
      cudaLaunchKernelEx(&cfg, kvc::attend_tc_streamk_kernel<D, T, PAGED>, p, tk, tv));
}

// The combine launch after a tcgen05 stream-K attend (p.sk_combine != 0): one block
// per (segment, chunk of kCombineRows rows), dependent on the attend grid.
template <int D, typename T>
kvc_status launch_combine(const kvc::AttendParams& p, bool pdl, cudaStream_t stream) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  const int segs = p.B * p.H_kv * p.row_blocks;
  cfg.gridDim = dim3(segs, kvc::ceil_div(p.sk_slot_rows, kvc::kCombineRows));
  cfg.blockDim = dim3(128);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cuda_status(cudaLaunchKernelEx(&cfg, kvc::combine_kernel<T, D>, p));
}

template <typename T>
kvc_status dispatch_tc_streamk(const kvc::AttendParams& p, int D, bool paged, int grid, bool pdl,
                               const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t s) {
  kvc_status st;
  if (D == 64)
    st = paged ? launch_attend_tc_streamk<64, T, true>(p, grid, pdl, tk, tv, s)
               : launch_attend_tc_streamk<64, T, false>(p, grid, pdl, tk, tv, s);
  else
    st = paged ? launch_attend_tc_streamk<128, T, true>(p, grid, pdl, tk, tv, s)
               : launch_attend_tc_streamk<128, T, false>(p, grid, pdl, tk, tv, s);
  if (st != KVC_OK || p.sk_combine == 0) return st;
  return D == 64 ? launch_combine<64, T>(p, pdl, s) : launch_combine<128, T>(p, pdl, s);
}

template <typename T>
kvc_status dispatch_tc(const kvc::AttendParams& p, int D, bool paged, const CUtensorMap& tk,
                       const CUtensorMap& tv, cudaStream_t s) {
  if (D == 64)
    return paged ? launch_attend_tc<64, T, true>(p, tk, tv, s)
                 : launch_attend_tc<64, T, false>(p, tk, tv, s);
  return paged ? launch_attend_tc<128, T, true>(p, tk, tv, s)
               : launch_attend_tc<128, T, false>(p, tk, tv, s);
}

template <int D, int NT, bool PAGED>
kvc_status launch_attend_fp8(const kvc::AttendParams& p, const kvc::Fp8Scales& sc,
                             const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t stream) {
  using C = kvc::Fp8Cfg<D>;
  fp8_occupancy<D, NT, PAGED>();  // sets the shared-memory attribute once
  dim3 grid(p.num_splits * p.row_blocks, p.H_kv, p.B);
  kvc::attend_fp8_kernel<D, NT, PAGED>
      <<<grid, C::kThreads, C::template smem_bytes<NT>(), stream>>>(p, sc, tk, tv);
  return cuda_status(cudaGetLastError());
}

template <int D, bool PAGED>
kvc_status dispatch_fp8_nt(const kvc::AttendParams& p, const kvc::Fp8Scales& sc, int NT,
                           const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t s) {
  switch (NT) {
    case 1: return launch_attend_fp8<D, 1, PAGED>(p, sc, tk, tv, s);
    case 2: return launch_attend_fp8<D, 2, PAGED>(p, sc, tk, tv, s);
    default: return launch_attend_fp8<D, 4, PAGED>(p, sc, tk, tv, s);
  }
}

float* scale_pool(const kvc_cache* c, int layer, int which) {
  return c->scales + (size_t)(2 * layer + which) * c->scale_floats;
}

// The parameter block of an attend call on layer `layer` (no workspace yet).  A pending
// stall (kvc_inject_stall) is taken by this call.
kvc::AttendParams attend_params(kvc_cache* c, int layer, const void* q, int H_q, int T_new,
                                const int32_t* block_table, int max_pages,
                                const int32_t* seq_lens, float scale, void* out,
                                const Plan& pl) {
  kvc::AttendParams p{};
  p.k_pool = c->pool + (size_t)(2 * layer) * c->layer_bytes;
  p.v_pool = c->pool + (size_t)(2 * layer + 1) * c->layer_bytes;
  p.q = q;
  p.out = out;
  p.seq_lens = seq_lens;
  p.block_table = block_table;
  p.max_pages = max_pages;
  p.B = c->B;
  p.H_q = H_q;
  p.H_kv = c->H_kv;
  p.T_new = T_new;
  p.group = H_q / c->H_kv;
  p.rows = p.group * T_new;
  p.max_T = c->max_T;
  p.page_shift = c->page_shift;
  p.num_pages = c->num_pages;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.split_tokens = pl.split_tokens;
  p.num_splits = pl.num_splits;
  p.row_blocks = pl.row_blocks;
  p.err = c->d_err;
  p.wait_limit_ns = c->wait_limit_ns;
  p.sk_penalty = !pl.streamk ? 0
                 : pl.tc      ? KVC_TC_SK_PENALTY
                 : pl.fp8     ? KVC_SK_PENALTY_FP8
                 : c->D == 128 ? KVC_SK_PENALTY_D128
                              : KVC_SK_PENALTY_D64;
  p.sk_blocked = pl.streamk && !pl.tc && !pl.fp8 && c->tma4 ? 1 : 0;
  // tcgen05 stream-K over several row blocks: row-block major when every block spans the
  // same positions (each holds all T_new new-row indices), so a request's K/V tiles are
  // streamed for all blocks at about the same time
  if (KVC_TC_RB_MAJOR && pl.tc && pl.streamk && pl.row_blocks > 1 && T_new <= pl.R) {
    const int last_rows = p.rows - (pl.row_blocks - 1) * pl.R;
    p.sk_rb_major = last_rows >= T_new ? 1 : 0;
  }
  if (pl.fp8) {
    p.k_scales = scale_pool(c, layer, 0);
    p.v_scales = scale_pool(c, layer, 1);
    p.T_pad = c->T_pad;
  }
  p.sk_slot_rows = pl.slot_rows;
  p.stall = c->stall_next ? 1 : 0;
  c->stall_next = false;
  p.replan = c->replan_next ? 1 : 0;
  c->replan_next = false;
  if (pl.combine) {
    // nonzero and new for every call of the process: descriptors left by another call
    // (of any cache: kvc_attend_noalloc shares one scratch) never match
    static std::atomic<int> gen{0};
    int g = gen.fetch_add(1) + 1;
    if (g <= 0) {  // wrapped
      gen.store(1);
      g = 1;
    }
    p.sk_combine = g;
  }
  return p;
}

// Where a plan's partial results start in a workspace of partial outputs then lse.
float* lse_base(const kvc_cache* c, const Plan& pl, float* ws, int H_q, int T_new) {
  if (!ws) return nullptr;
  return pl.streamk ? ws + pl.slots * pl.slot_rows * c->D
                    : ws + (size_t)c->B * H_q * T_new * pl.num_splits * c->D;
}

// Where the combine descriptors start (tcgen05 stream-K): after the slots' lse values.
int* desc_base(const Plan& pl, float* lse) {
  return (lse && pl.combine) ? reinterpret_cast<int*>(lse + pl.slots * pl.slot_rows) : nullptr;
}

// Launch the attend kernel a plan chose for layer `layer`.
kvc_status run_plan(const kvc_cache* c, int layer, const Plan& pl, const kvc::AttendParams& p,
                    cudaStream_t s) {
  if (pl.fp8 && pl.streamk)
    return dispatch_streamk_fp8(p, c->D, c->paged, pl.grid, c->dependent_launch, c->tmk[layer],
                                c->tmv[layer], s);
  if (pl.fp8) {
    const kvc::Fp8Scales sc{scale_pool(c, layer, 0), scale_pool(c, layer, 1), c->T_pad};
    if (c->D == 64)
      return c->paged ? dispatch_fp8_nt<64, true>(p, sc, pl.NT, c->tmk[layer], c->tmv[layer], s)
                      : dispatch_fp8_nt<64, false>(p, sc, pl.NT, c->tmk[layer], c->tmv[layer], s);
    return c->paged ? dispatch_fp8_nt<128, true>(p, sc, pl.NT, c->tmk[layer], c->tmv[layer], s)
                    : dispatch_fp8_nt<128, false>(p, sc, pl.NT, c->tmk[layer], c->tmv[layer], s);
  }
  const bool bf = c->dtype == KVC_BF16;
  if (pl.tc && pl.streamk)
    return bf ? dispatch_tc_streamk<__nv_bfloat16>(p, c->D, c->paged, pl.grid,
                                                   c->dependent_launch, c->tmk[layer],
                                                   c->tmv[layer], s)
              : dispatch_tc_streamk<__half>(p, c->D, c->paged, pl.grid, c->dependent_launch,
                                            c->tmk[layer], c->tmv[layer], s);
  if (pl.tc)
    return bf ? dispatch_tc<__nv_bfloat16>(p, c->D, c->paged, c->tmk[layer], c->tmv[layer], s)
              : dispatch_tc<__half>(p, c->D, c->paged, c->tmk[layer], c->tmv[layer], s);
  if (pl.streamk) {
    const CUtensorMap& tk = p.sk_blocked ? c->tmk4[layer] : c->tmk[layer];
    const CUtensorMap& tv = p.sk_blocked ? c->tmv4[layer] : c->tmv[layer];
    return bf ? dispatch_streamk<__nv_bfloat16>(p, c->D, pl.NT, c->paged, pl.grid,
                                                c->dependent_launch, tk, tv, s)
              : dispatch_streamk<__half>(p, c->D, pl.NT, c->paged, pl.grid,
                                         c->dependent_launch, tk, tv, s);
  }
  if (pl.mma)
    return bf ? dispatch_mma<__nv_bfloat16>(p, c->D, pl.NT, c->paged, c->tmk[layer],
                                            c->tmv[layer], s)
              : dispatch_mma<__half>(p, c->D, pl.NT, c->paged, c->tmk[layer], c->tmv[layer], s);
  return bf ? dispatch_d<__nv_bfloat16>(p, c->D, pl.R, c->paged, s)
            : dispatch_d<__half>(p, c->D, pl.R, c->paged, s);
}

}  // namespace

extern "C" {

const char* kvc_status_string(kvc_status s) {
  switch (s) {
    case KVC_OK: return "KVC_OK";
    case KVC_ERR_INVALID_ARG: return "KVC_ERR_INVALID_ARG";
    case KVC_ERR_UNSUPPORTED: return "KVC_ERR_UNSUPPORTED";
    case KVC_ERR_OOM: return "KVC_ERR_OOM";
    case KVC_ERR_CUDA: return "KVC_ERR_CUDA";
    case KVC_ERR_BOUNDS: return "KVC_ERR_BOUNDS";
    case KVC_ERR_TIMEOUT: return "KVC_ERR_TIMEOUT";
    case KVC_ERR_SCRATCH: return "KVC_ERR_SCRATCH";
  }
  return "KVC_ERR_UNKNOWN";
}

size_t kvc_bytes_formula(int layers, int kv_heads, int head_dim, long long seq_len,
                         int bytes_per_elem, int batch) {
  return (size_t)2 * (size_t)layers * (size_t)kv_heads * (size_t)head_dim * (size_t)seq_len *
         (size_t)bytes_per_elem * (size_t)batch;
}

static kvc_status create_cache(int B, int H_kv, int D, int max_T, kvc_dtype dtype,
                               kvc_kv_format kv_format, int page_size, int num_layers,
                               int num_pages, kvc_cache** out) {
  if (!out) return KVC_ERR_INVALID_ARG;
  *out = nullptr;
  if (B <= 0 || H_kv <= 0 || max_T <= 0 || num_layers <= 0 || page_size < 0 || num_pages < 0)
    return KVC_ERR_INVALID_ARG;
  if (dtype != KVC_FP16 && dtype != KVC_BF16) return KVC_ERR_INVALID_ARG;
  if (kv_format != KVC_KV_NATIVE && kv_format != KVC_KV_FP8_E4M3) return KVC_ERR_INVALID_ARG;
  if (D != 32 && D != 64 && D != 128) return KVC_ERR_UNSUPPORTED;
  const bool fp8 = kv_format == KVC_KV_FP8_E4M3;
  // the FP8 path: bf16 queries, D 64 or 128, pages of 8 or more tokens
  if (fp8 && (dtype != KVC_BF16 || D == 32 || (page_size > 0 && page_size < 8)))
    return KVC_ERR_UNSUPPORTED;
  const bool paged = page_size > 0;
  int shift = 0;
  if (paged) {
    shift = log2_exact(page_size);
    if (shift < 0 || page_size > 1024 || num_pages <= 0) return KVC_ERR_INVALID_ARG;
  } else if (num_pages != 0) {
    return KVC_ERR_INVALID_ARG;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return KVC_ERR_CUDA;
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return KVC_ERR_CUDA;
  }
  const int elt = fp8 ? 1 : kEltBytes;
  const size_t layer_bytes = paged ? (size_t)num_pages * H_kv * page_size * D * elt
                                   : (size_t)B * H_kv * max_T * D * elt;
  kvc_cache* c = new kvc_cache();
  c->B = B;
  c->H_kv = H_kv;
  c->D = D;
  c->max_T = max_T;
  c->page_size = page_size;
  c->page_shift = shift;
  c->num_layers = num_layers;
  c->num_pages = num_pages;
  c->dtype = dtype;
  c->paged = paged;
  c->layer_bytes = layer_bytes;
  c->fp8 = fp8;
  c->T_pad = (max_T + 63) / 64 * 64;
  c->scale_floats = fp8 ? (paged ? (size_t)num_pages * H_kv * page_size
                                 : (size_t)B * H_kv * c->T_pad)
                        : 0;
  c->device = dev;
  c->num_sms = sms;
  c->dependent_launch = dependent_launch_enabled();
  c->wait_limit_ns = 0;
  c->stall_next = false;
  c->replan_next = false;
  void* pool = nullptr;
  if (cudaMalloc(&pool, 2 * layer_bytes * (size_t)num_layers) != cudaSuccess) {
    cudaGetLastError();
    delete c;
    return KVC_ERR_OOM;
  }
  c->pool = static_cast<char*>(pool);
  void* err = nullptr;
  if (cudaMalloc(&err, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    cudaFree(pool);
    delete c;
    return KVC_ERR_OOM;
  }
  c->d_err = static_cast<int*>(err);
  if (fp8) {
    void* sc = nullptr;
    const size_t sbytes = 2 * c->scale_floats * (size_t)num_layers * sizeof(float);
    if (cudaMalloc(&sc, sbytes) != cudaSuccess) {
      cudaGetLastError();
      cudaFree(c->pool);
      cudaFree(c->d_err);
      delete c;
      return KVC_ERR_OOM;
    }
    c->scales = static_cast<float*>(sc);
    if (cudaMemset(sc, 0, sbytes) != cudaSuccess) {  // finite scales everywhere
      cudaGetLastError();
      cudaFree(c->pool);
      cudaFree(c->d_err);
      cudaFree(sc);
      delete c;
      return KVC_ERR_CUDA;
    }
  }
  if (cudaMemset(c->pool, 0, 2 * layer_bytes * (size_t)num_layers) != cudaSuccess ||
      cudaMemset(c->d_err, 0, sizeof(int)) != cudaSuccess ||
      cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    cudaFree(c->pool);
    cudaFree(c->d_err);
    if (c->scales) cudaFree(c->scales);
    delete c;
    return KVC_ERR_CUDA;
  }
  build_tmaps(c);
  if (fp8 && !c->tma) {  // the FP8 attend needs its tensor maps
    kvc_destroy(c);
    return KVC_ERR_UNSUPPORTED;
  }
  *out = c;
  return KVC_OK;
}

kvc_status kvc_create(int B, int H_kv, int D, int max_T, kvc_dtype dtype, int page_size,
                      int num_layers, int num_pages, kvc_cache** out) {
  return create_cache(B, H_kv, D, max_T, dtype, KVC_KV_NATIVE, page_size, num_layers, num_pages,
                      out);
}

kvc_status kvc_create_quantized(int B, int H_kv, int D, int max_T, kvc_dtype dtype,
                                kvc_kv_format kv_format, int page_size, int num_layers,
                                int num_pages, kvc_cache** out) {
  return create_cache(B, H_kv, D, max_T, dtype, kv_format, page_size, num_layers, num_pages,
                      out);
}

kvc_status kvc_destroy(kvc_cache* c) {
  if (!c) return KVC_OK;
  cudaError_t e = cudaDeviceSynchronize();
  cudaFree(c->pool);
  cudaFree(c->d_err);
  if (c->scales) cudaFree(c->scales);
  if (c->ws) cudaFree(c->ws);
  if (c->tickets) cudaFree(c->tickets);
  delete c;
  return cuda_status(e);
}

size_t kvc_bytes(const kvc_cache* c) {
  if (!c) return 0;
  if (c->fp8) {  // one byte a code, plus one fp32 scale a (token, head) for K and for V
    const long long T = c->paged ? (long long)c->num_pages * c->page_size : c->max_T;
    const int batch = c->paged ? 1 : c->B;
    return kvc_bytes_formula(c->num_layers, c->H_kv, c->D, T, 1, batch) +
           kvc_bytes_formula(c->num_layers, c->H_kv, 1, T, (int)sizeof(float), batch);
  }
  if (c->paged)
    return kvc_bytes_formula(c->num_layers, c->H_kv, c->D,
                             (long long)c->num_pages * c->page_size, kEltBytes, 1);
  return kvc_bytes_formula(c->num_layers, c->H_kv, c->D, c->max_T, kEltBytes, c->B);
}

size_t kvc_layer_pool_bytes(const kvc_cache* c) { return c ? c->layer_bytes : 0; }

void* kvc_k_pool(kvc_cache* c, int layer) {
  if (!c || layer < 0 || layer >= c->num_layers) return nullptr;
  return c->pool + (size_t)(2 * layer) * c->layer_bytes;
}

void* kvc_v_pool(kvc_cache* c, int layer) {
  if (!c || layer < 0 || layer >= c->num_layers) return nullptr;
  return c->pool + (size_t)(2 * layer + 1) * c->layer_bytes;
}

float* kvc_k_scales(kvc_cache* c, int layer) {
  if (!c || !c->fp8 || layer < 0 || layer >= c->num_layers) return nullptr;
  return scale_pool(c, layer, 0);
}

float* kvc_v_scales(kvc_cache* c, int layer) {
  if (!c || !c->fp8 || layer < 0 || layer >= c->num_layers) return nullptr;
  return scale_pool(c, layer, 1);
}

size_t kvc_layer_scale_floats(const kvc_cache* c) { return c ? c->scale_floats : 0; }

kvc_status kvc_append(kvc_cache* c, int layer, const void* k_new, const void* v_new, int T_new,
                      const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                      void* stream) {
  if (!c || layer < 0 || layer >= c->num_layers || T_new <= 0) return KVC_ERR_INVALID_ARG;
  if (!k_new || !v_new || !seq_lens || !aligned16(k_new) || !aligned16(v_new) ||
      !aligned4(seq_lens))
    return KVC_ERR_INVALID_ARG;
  if (c->paged && (!block_table || !aligned4(block_table) || max_pages <= 0))
    return KVC_ERR_INVALID_ARG;
  if (!c->paged && block_table) return KVC_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (c->fp8) {
    kvc::AppendFp8Params q{};
    q.k_new = k_new;
    q.v_new = v_new;
    q.k_codes = static_cast<uint8_t*>(kvc_k_pool(c, layer));
    q.v_codes = static_cast<uint8_t*>(kvc_v_pool(c, layer));
    q.k_scales = scale_pool(c, layer, 0);
    q.v_scales = scale_pool(c, layer, 1);
    q.seq_lens = seq_lens;
    q.block_table = block_table;
    q.B = c->B;
    q.H_kv = c->H_kv;
    q.T_new = T_new;
    q.D = c->D;
    q.max_T = c->max_T;
    q.T_pad = c->T_pad;
    q.max_pages = max_pages;
    q.page_shift = c->page_shift;
    q.num_pages = c->num_pages;
    q.err = c->d_err;
    const long long warps = 2LL * c->B * c->H_kv * T_new;
    const unsigned blocks = (unsigned)((warps * 32 + 255) / 256);
    if (c->paged) kvc::append_fp8_kernel<true><<<blocks, 256, 0, st>>>(q);
    else kvc::append_fp8_kernel<false><<<blocks, 256, 0, st>>>(q);
    return cuda_status(cudaGetLastError());
  }
  kvc::AppendParams p{};
  p.k_new = k_new;
  p.v_new = v_new;
  p.k_pool = kvc_k_pool(c, layer);
  p.v_pool = kvc_v_pool(c, layer);
  p.seq_lens = seq_lens;
  p.block_table = block_table;
  p.B = c->B;
  p.H_kv = c->H_kv;
  p.T_new = T_new;
  p.D = c->D;
  p.max_T = c->max_T;
  p.max_pages = max_pages;
  p.page_shift = c->page_shift;
  p.num_pages = c->num_pages;
  p.err = c->d_err;
  const long long vecs = (long long)c->B * c->H_kv * T_new * (c->D / 8);
  const unsigned blocks = (unsigned)((vecs + 255) / 256);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (c->paged) kvc::append_kernel<true><<<blocks, 256, 0, s>>>(p);
  else kvc::append_kernel<false><<<blocks, 256, 0, s>>>(p);
  return cuda_status(cudaGetLastError());
}

kvc_status kvc_commit(kvc_cache* c, int32_t* seq_lens, const int32_t* accepted, int T_new,
                      void* stream) {
  if (!c || !seq_lens || !accepted || T_new <= 0 || !aligned4(seq_lens) || !aligned4(accepted))
    return KVC_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  kvc::commit_kernel<<<(c->B + 127) / 128, 128, 0, s>>>(seq_lens, accepted, c->B, T_new,
                                                          c->max_T, c->d_err);
  return cuda_status(cudaGetLastError());
}

kvc_status kvc_rollback(kvc_cache* c, int32_t* seq_lens, const int32_t* drop, void* stream) {
  if (!c || !seq_lens || !drop || !aligned4(seq_lens) || !aligned4(drop))
    return KVC_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  kvc::rollback_kernel<<<(c->B + 127) / 128, 128, 0, s>>>(seq_lens, drop, c->B, c->d_err);
  return cuda_status(cudaGetLastError());
}

kvc_status kvc_copy_pages(kvc_cache* c, const int32_t* src, const int32_t* dst, int n,
                          void* stream) {
  if (!c || n < 0 || (n > 0 && (!src || !dst || !aligned4(src) || !aligned4(dst))))
    return KVC_ERR_INVALID_ARG;
  if (!c->paged) return KVC_ERR_UNSUPPORTED;
  if (n == 0) return KVC_OK;
  if (2LL * c->num_layers > 65535) return KVC_ERR_UNSUPPORTED;
  const size_t page_bytes = (size_t)c->H_kv * c->page_size * c->D * (c->fp8 ? 1 : kEltBytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  dim3 grid((unsigned)n, (unsigned)(2 * c->num_layers));
  kvc::copy_pages_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<uint4*>(c->pool),
                                               c->layer_bytes / 16, src, dst, n, c->num_layers,
                                               c->num_pages, (int)(page_bytes / 16), c->d_err);
  if (c->fp8) {  // the pages' scales too: H_kv * page_size floats a page
    const size_t scale_page_bytes = (size_t)c->H_kv * c->page_size * sizeof(float);
    kvc::copy_pages_kernel<<<grid, 256, 0, s>>>(
        reinterpret_cast<uint4*>(c->scales), c->scale_floats * sizeof(float) / 16, src, dst, n,
        c->num_layers, c->num_pages, (int)(scale_page_bytes / 16), c->d_err);
  }
  return cuda_status(cudaGetLastError());
}

kvc_status kvc_plan_splits(const kvc_cache* c, int H_q, int T_new, int max_pages,
                           int* num_splits, int* split_tokens) {
  if (!c || H_q <= 0 || T_new <= 0 || H_q % c->H_kv != 0) return KVC_ERR_INVALID_ARG;
  if (c->paged && max_pages <= 0) return KVC_ERR_INVALID_ARG;
  const Plan pl = make_plan(c, H_q, T_new, max_pages);
  if (num_splits) *num_splits = pl.streamk ? pl.grid : pl.num_splits;
  if (split_tokens) *split_tokens = pl.streamk ? 0 : pl.split_tokens;
  return KVC_OK;
}

kvc_status kvc_reserve(kvc_cache* c, int H_q, int T_new, int max_pages) {
  if (!c || H_q <= 0 || T_new <= 0 || H_q % c->H_kv != 0) return KVC_ERR_INVALID_ARG;
  if (c->paged && max_pages <= 0) return KVC_ERR_INVALID_ARG;
  const Plan pl = make_plan(c, H_q, T_new, max_pages);
  return ensure_workspace(c, pl.ws_bytes, pl.ws_counters);
}

kvc_status kvc_attend_window(kvc_cache* c, int layer, const void* q, int H_q, int T_new,
                             const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                             float scale, int window, int sink, void* out, void* stream) {
  if (!c || layer < 0 || layer >= c->num_layers || T_new <= 0 || H_q <= 0 ||
      H_q % c->H_kv != 0)
    return KVC_ERR_INVALID_ARG;
  if (!q || !out || !seq_lens || !aligned16(q) || !aligned16(out) || !aligned4(seq_lens))
    return KVC_ERR_INVALID_ARG;
  if (c->paged && (!block_table || !aligned4(block_table) || max_pages <= 0))
    return KVC_ERR_INVALID_ARG;
  if (!c->paged && block_table) return KVC_ERR_INVALID_ARG;
  if (!(scale == scale) || window < 0 || sink < 0) return KVC_ERR_INVALID_ARG;
  if (window == 0) sink = 0;  // no window: every position is visible anyway
  const Plan pl = make_plan(c, H_q, T_new, max_pages, window, sink);
  kvc_status st = ensure_workspace(c, pl.ws_bytes, pl.ws_counters);
  if (st != KVC_OK) return st;
  kvc::AttendParams p =
      attend_params(c, layer, q, H_q, T_new, block_table, max_pages, seq_lens, scale, out, pl);
  p.window = window;
  p.sink = sink;
  p.ws_o = c->ws;
  p.ws_lse = lse_base(c, pl, c->ws, H_q, T_new);
  p.sk_desc = desc_base(pl, p.ws_lse);
  p.counters = c->tickets;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return run_plan(c, layer, pl, p, s);
}

kvc_status kvc_attend(kvc_cache* c, int layer, const void* q, int H_q, int T_new,
                      const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                      float scale, void* out, void* stream) {
  return kvc_attend_window(c, layer, q, H_q, T_new, block_table, max_pages, seq_lens, scale, 0,
                           0, out, stream);
}

kvc_status kvc_get_error(kvc_cache* c) {
  if (!c) return KVC_ERR_INVALID_ARG;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return KVC_ERR_CUDA;
  int h = 0;
  if (cudaMemcpy(&h, c->d_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return KVC_ERR_CUDA;
  if (h != 0) {
    if (cudaMemset(c->d_err, 0, sizeof(int)) != cudaSuccess) return KVC_ERR_CUDA;
    // A launch that gave up may have left slice tickets behind: clear them all.
    if (c->tickets && cudaMemset(c->tickets, 0, c->n_tickets * sizeof(int)) != cudaSuccess)
      return KVC_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return KVC_ERR_CUDA;
  }
  return static_cast<kvc_status>(h);
}

kvc_status kvc_set_dependent_launch(kvc_cache* c, int on) {
  if (!c) return KVC_ERR_INVALID_ARG;
  c->dependent_launch = on != 0;
  return KVC_OK;
}

kvc_status kvc_set_wait_limit(kvc_cache* c, unsigned long long ns) {
  if (!c) return KVC_ERR_INVALID_ARG;
  c->wait_limit_ns = ns;
  return KVC_OK;
}

kvc_status kvc_inject_stall(kvc_cache* c) {
  if (!c) return KVC_ERR_INVALID_ARG;
  c->stall_next = true;
  return KVC_OK;
}

kvc_status kvc_inject_replan(kvc_cache* c) {
  if (!c) return KVC_ERR_INVALID_ARG;
  c->replan_next = true;
  return KVC_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free attend.
//
// Some callers cannot let a library allocate device memory: code that records
// a decode step inside CUDA stream capture (cudaMalloc is not a capturable
// operation), engines whose caching allocator owns nearly all of the device's
// memory (a side allocation can fail or fragment its pool), and latency-bound
// serving loops that cannot afford the device synchronisation cudaFree implies.
// For them kvc_attend_noalloc runs the same kernels as kvc_attend with the
// split-K scratch (partial results and slice tickets) in the fixed-size device
// array below instead of the cache's growable workspace.
static constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB on every device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

static constexpr int kNoAllocMaxDevices = 64;
static std::mutex g_noalloc_mu;
static void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of the scratch array on the current device: looked up once per
// device (the array's name is only a host-side stand-in in host code).
static kvc_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) {
    cudaGetLastError();
    return KVC_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return KVC_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return KVC_OK;
}

extern "C" kvc_status kvc_attend_noalloc(kvc_cache* c, int layer, const void* q, int H_q,
                                         int T_new, const int32_t* block_table, int max_pages,
                                         const int32_t* seq_lens, float scale, void* out,
                                         void* stream) {
  if (!c || layer < 0 || layer >= c->num_layers || T_new <= 0 || H_q <= 0 ||
      H_q % c->H_kv != 0)
    return KVC_ERR_INVALID_ARG;
  if (!q || !out || !seq_lens || !aligned16(q) || !aligned16(out) || !aligned4(seq_lens))
    return KVC_ERR_INVALID_ARG;
  if (c->paged && (!block_table || !aligned4(block_table) || max_pages <= 0))
    return KVC_ERR_INVALID_ARG;
  if (!c->paged && block_table) return KVC_ERR_INVALID_ARG;
  if (!(scale == scale)) return KVC_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return KVC_ERR_CUDA;
  }
  if (dev != c->device) return KVC_ERR_INVALID_ARG;  // the scratch must be on the cache's GPU
  const Plan pl = make_plan(c, H_q, T_new, max_pages);
  // [tickets, padded to 256 bytes][partial outputs][lse]
  const size_t ticket_bytes = (pl.ws_counters * sizeof(int) + 255) & ~size_t(255);
  if (ticket_bytes + pl.ws_bytes > kNoAllocScratchBytes) return KVC_ERR_SCRATCH;
  void* base = nullptr;
  kvc_status st = noalloc_scratch(&base);
  if (st != KVC_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents; tickets must start at zero.
  if (pl.ws_counters &&
      cudaMemsetAsync(base, 0, pl.ws_counters * sizeof(int), s) != cudaSuccess)
    return cuda_status(cudaGetLastError());
  float* ws = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + ticket_bytes);
  kvc::AttendParams p =
      attend_params(c, layer, q, H_q, T_new, block_table, max_pages, seq_lens, scale, out, pl);
  p.ws_o = ws;
  p.ws_lse = lse_base(c, pl, ws, H_q, T_new);
  p.sk_desc = desc_base(pl, p.ws_lse);
  p.counters = static_cast<int*>(base);
  return run_plan(c, layer, pl, p, s);
}

// ---------------------------------------------------------------------------
// Append and attend in one call.  With the persistent stream-K kernels this is one
// attend launch (plus the combine launch of a tcgen05 plan that uses one): on mma.sync
// the tile holding the new positions takes them from k_new / v_new and the kernel
// writes them into the cache; on tcgen05 the producer warps write them into the cache
// before the copies of those tiles.  The fixed-split kernels run the append kernel and
// then the attend kernel on the same stream.
extern "C" kvc_status kvc_append_attend(kvc_cache* c, int layer, const void* k_new,
                                        const void* v_new, const void* q, int H_q, int T_new,
                                        const int32_t* block_table, int max_pages,
                                        const int32_t* seq_lens, float scale, void* out,
                                        void* stream) {
  if (!c || layer < 0 || layer >= c->num_layers || T_new <= 0 || H_q <= 0 ||
      H_q % c->H_kv != 0)
    return KVC_ERR_INVALID_ARG;
  if (!q || !out || !seq_lens || !k_new || !v_new || !aligned16(q) || !aligned16(out) ||
      !aligned16(k_new) || !aligned16(v_new) || !aligned4(seq_lens))
    return KVC_ERR_INVALID_ARG;
  if (c->paged && (!block_table || !aligned4(block_table) || max_pages <= 0))
    return KVC_ERR_INVALID_ARG;
  if (!c->paged && block_table) return KVC_ERR_INVALID_ARG;
  if (!(scale == scale)) return KVC_ERR_INVALID_ARG;
  const Plan pl = make_plan(c, H_q, T_new, max_pages);
  if (!pl.streamk) {  // the fixed-split kernels do not fuse the append
    kvc_status st = kvc_append(c, layer, k_new, v_new, T_new, block_table, max_pages,
                               seq_lens, stream);
    if (st != KVC_OK) return st;
    return kvc_attend(c, layer, q, H_q, T_new, block_table, max_pages, seq_lens, scale, out,
                      stream);
  }
  kvc_status st = ensure_workspace(c, pl.ws_bytes, pl.ws_counters);
  if (st != KVC_OK) return st;
  kvc::AttendParams p =
      attend_params(c, layer, q, H_q, T_new, block_table, max_pages, seq_lens, scale, out, pl);
  p.ws_o = c->ws;
  p.ws_lse = lse_base(c, pl, c->ws, H_q, T_new);
  p.sk_desc = desc_base(pl, p.ws_lse);
  p.counters = c->tickets;
  p.k_new = k_new;
  p.v_new = v_new;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (pl.fp8)
    return dispatch_streamk_fp8(p, c->D, c->paged, pl.grid, c->dependent_launch, c->tmk[layer],
                                c->tmv[layer], s);
  if (pl.tc)
    return c->dtype == KVC_BF16
               ? dispatch_tc_streamk<__nv_bfloat16>(p, c->D, c->paged, pl.grid,
                                                    c->dependent_launch, c->tmk[layer],
                                                    c->tmv[layer], s)
               : dispatch_tc_streamk<__half>(p, c->D, c->paged, pl.grid, c->dependent_launch,
                                             c->tmk[layer], c->tmv[layer], s);
  const CUtensorMap& tk = p.sk_blocked ? c->tmk4[layer] : c->tmk[layer];
  const CUtensorMap& tv = p.sk_blocked ? c->tmv4[layer] : c->tmv[layer];
  return c->dtype == KVC_BF16
             ? dispatch_streamk<__nv_bfloat16>(p, c->D, pl.NT, c->paged, pl.grid,
                                               c->dependent_launch, tk, tv, s)
             : dispatch_streamk<__half>(p, c->D, pl.NT, c->paged, pl.grid, c->dependent_launch,
                                        tk, tv, s);
}
