// append.cuh -- N1: write the new tokens' K and V into the cache.
//
// "9. 推理：从生成到性能优化" section 9.3: the past K/V are never recomputed or
// moved; each step only adds the new token's K/V.  "项目 9-16" project 11 does
// this with a concatenation along T; here the cache is preallocated and the
// rows are written in place (contiguous), or scattered into pages through the
// block table ("9. 推理" section 9.6).
//
// One thread moves one 16-byte vector of K and the matching vector of V, so a
// warp covers 512 contiguous bytes of a row block and every store is a full
// 16-byte store.  The copy is bit-exact.
#pragma once

#include "device_common.cuh"
#include "params.cuh"

namespace kvc {

template <bool PAGED>
__global__ void __launch_bounds__(256) append_kernel(AppendParams p) {
  const int vec_per_row = p.D / 8;  // 16-byte vectors per (token, head) row
  const long long total = (long long)p.B * p.H_kv * p.T_new * vec_per_row;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int c = (int)(idx % vec_per_row);
  long long r = idx / vec_per_row;
  const int i = (int)(r % p.T_new);
  r /= p.T_new;
  const int g = (int)(r % p.H_kv);
  const int b = (int)(r / p.H_kv);

  const int L = p.seq_lens[b];
  const int pos = L + i;
  if (L < 0 || pos >= p.max_T) {
    flag_error(p.err, KVC_ERR_BOUNDS);
    return;
  }
  long long dst_row;
  if (PAGED) {
    const int lp = pos >> p.page_shift;
    if (lp >= p.max_pages) {
      flag_error(p.err, KVC_ERR_BOUNDS);
      return;
    }
    const int page = p.block_table[(long long)b * p.max_pages + lp];
    if (page < 0 || page >= p.num_pages) {
      flag_error(p.err, KVC_ERR_BOUNDS);
      return;
    }
    const int slot = pos & ((1 << p.page_shift) - 1);
    dst_row = ((long long)page * p.H_kv + g) * (1 << p.page_shift) + slot;
  } else {
    dst_row = ((long long)b * p.H_kv + g) * p.max_T + pos;
  }
  const long long src_off = idx * 16;  // (b, g, i, c) row-major == idx order
  const long long dst_off = (dst_row * p.D + c * 8) * 2;
  const uint4 kv = ld_global_nc_v4(static_cast<const char*>(p.k_new) + src_off);
  const uint4 vv = ld_global_nc_v4(static_cast<const char*>(p.v_new) + src_off);
  st_global_v4(static_cast<char*>(p.k_pool) + dst_off, kv);
  st_global_v4(static_cast<char*>(p.v_pool) + dst_off, vv);
}

}  // namespace kvc
