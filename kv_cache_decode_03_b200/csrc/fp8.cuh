// fp8.cuh -- N5: an FP8 (E4M3) K/V cache with one fp32 scale per (token, KV head).
//
// The quantised cache is a later item on the pages ("llm-perf-lab" README and "9. 推理"
// 9.3 leave KV quantisation uncovered; it halves the bytes every decode step reads).
// Format: each K (and V) row of D values x is stored as D E4M3 codes and a scale
//     scale = amax / 448   (amax = max_d |x_d|; 448 is E4M3's largest finite value;
//                           an all-zero row takes scale 1)
//     code_d = E4M3(x_d / scale), round to nearest even, saturated to +-448,
// with both divisions in fp32 (IEEE, correctly rounded), so the codes are a pure
// function of the row.  The attend kernel uses code * scale exactly: the K scale
// multiplies the row's score, the V scale the row's softmax weight.
#pragma once

#include <stdint.h>

#include "device_common.cuh"
#include "params.cuh"

namespace kvc {

constexpr float kE4M3Max = 448.f;

// Two E4M3 codes (low byte first) -> two bf16 values (exact: E4M3 has 3 mantissa bits).
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t v) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(v));
  float lo, hi;
  asm("{\n\t.reg .f16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.f32.f16 %0, a;\n\tcvt.f32.f16 %1, b;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(h2));
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two fp32 values -> two E4M3 codes (low byte = lo), nearest even, saturated.
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// 16 E4M3 codes -> 16 bf16 values (two 16-byte chunks, element order kept).
__device__ __forceinline__ void e4m3x16_to_bf16(const uint4& c, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  uint32_t o[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    o[2 * k] = e4m3x2_to_bf16x2((uint16_t)(w[k] & 0xFFFFu));
    o[2 * k + 1] = e4m3x2_to_bf16x2((uint16_t)(w[k] >> 16));
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

struct AppendFp8Params {
  const void* k_new;  // (B, H_kv, T_new, D) bf16
  const void* v_new;
  uint8_t* k_codes;   // this layer's code pools (contiguous (B, H_kv, T_cap, D) or paged)
  uint8_t* v_codes;
  float* k_scales;    // (B, H_kv, T_pad) contiguous, (num_pages, H_kv, P) paged
  float* v_scales;
  const int32_t* seq_lens;
  const int32_t* block_table;
  int B, H_kv, T_new, D;
  int max_T, T_pad;  // capacity; scale row length of the contiguous layout
  int max_pages, page_shift, num_pages;
  int* err;
};

// Quantises one row of D = 32 * PER bf16 values with a warp: lane `lane` holds values
// lane*PER .. lane*PER + PER - 1 of `src`; returns the row's scale (every lane) and the
// lane's PER codes, first value in the low byte.
template <int PER>
__device__ __forceinline__ float quantize_row_warp(const __nv_bfloat16* src, int lane,
                                                   uint32_t& codes) {
  float x[PER];
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    x[k] = __bfloat162float(src[lane * PER + k]);
    amax = fmaxf(amax, fabsf(x[k]));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float scale = amax > 0.f ? amax / kE4M3Max : 1.f;
  codes = 0u;
#pragma unroll
  for (int k = 0; k < PER; k += 2)
    codes |= (uint32_t)f32x2_to_e4m3x2(x[k] / scale, x[k + 1] / scale) << (8 * k);
  return scale;
}

// One warp per new row (b, g, i) and tensor (K or V): lanes own D/32 values each.
template <bool PAGED>
__global__ void append_fp8_kernel(const AppendFp8Params p) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int rows = p.B * p.H_kv * p.T_new;
  if (warp >= 2 * rows) return;
  const bool is_v = warp >= rows;
  const int r = is_v ? warp - rows : warp;
  const int i = r % p.T_new;
  const int g = (r / p.T_new) % p.H_kv;
  const int b = r / (p.T_new * p.H_kv);
  const int L = p.seq_lens[b];
  const int pos = L + i;
  if (L < 0 || pos >= p.max_T) {
    if (lane == 0) flag_error(p.err, KVC_ERR_BOUNDS);
    return;
  }
  size_t row;  // destination row index (codes: row * D bytes; scales: row)
  if (PAGED) {
    const int lp = pos >> p.page_shift;
    const int page = lp < p.max_pages ? p.block_table[(size_t)b * p.max_pages + lp] : -1;
    if (page < 0 || page >= p.num_pages) {
      if (lane == 0) flag_error(p.err, KVC_ERR_BOUNDS);
      return;
    }
    const int P = 1 << p.page_shift;
    row = ((size_t)page * p.H_kv + g) * P + (pos & (P - 1));
  } else {
    row = ((size_t)b * p.H_kv + g) * p.max_T + pos;
  }
  const size_t srow = PAGED ? row : ((size_t)b * p.H_kv + g) * p.T_pad + pos;
  const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(is_v ? p.v_new : p.k_new) +
                             (size_t)r * p.D;
  // D = 64 or 128: each lane holds 2 or 4 consecutive values
  uint32_t codes;
  uint8_t* dst = (is_v ? p.v_codes : p.k_codes) + row * p.D;
  float scale;
  if (p.D == 128) {
    scale = quantize_row_warp<4>(src, lane, codes);
    reinterpret_cast<uint32_t*>(dst)[lane] = codes;
  } else {
    scale = quantize_row_warp<2>(src, lane, codes);
    reinterpret_cast<uint16_t*>(dst)[lane] = (uint16_t)codes;
  }
  if (lane == 0) (is_v ? p.v_scales : p.k_scales)[srow] = scale;
}

}  // namespace kvc
