// params.cuh -- launch parameter blocks shared by the host planner and the kernels.
#pragma once

#include <stdint.h>

namespace kvc {

struct AppendParams {
  const void* k_new;  // (B, H_kv, T_new, D)
  const void* v_new;
  void* k_pool;       // this layer's pools
  void* v_pool;
  const int32_t* seq_lens;     // (B)
  const int32_t* block_table;  // (B, max_pages) or null
  int B, H_kv, T_new, D;
  int max_T;       // logical capacity per request
  int max_pages;   // block-table columns
  int page_shift;  // log2(page_size) (paged)
  int num_pages;
  int* err;
};

struct AttendParams {
  const void* k_pool;  // this layer's pools
  const void* v_pool;
  const void* q;       // (B, H_q, T_new, D)
  void* out;           // (B, H_q, T_new, D)
  const int32_t* seq_lens;
  const int32_t* block_table;
  int max_pages;
  int B, H_q, H_kv, T_new, group, rows;  // rows = group * T_new (query rows per KV head)
  int max_T;                             // logical capacity per request
  int page_shift;                        // log2(page_size) (paged)
  int num_pages;
  float scale_log2;   // scale * log2(e): scores are kept in base-2 units
  int window;         // sliding window W (0 = none): row with n positions sees [n - W, n)
  int sink;           // ... and the first `sink` positions (window.cuh)
  int split_tokens;   // tokens per split-K slice (a multiple of the tile; virtual
                      // positions when a window is set, window.cuh)
  int num_splits;     // slices in the grid
  int row_blocks;     // CTAs per KV head along the query rows
  float* ws_o;        // (B, H_q, T_new, num_splits, D) normalised partial outputs
  float* ws_lse;      // (B, H_q, T_new, num_splits) base-2 log-sum-exp of each slice
  int* counters;      // (B, H_kv, row_blocks) slice tickets, zero between launches
  const void* k_new;  // fused append (stream-K kernel): (B, H_kv, T_new, D), else null
  const void* v_new;
  int* err;
  unsigned long long wait_limit_ns;  // bound of every pipeline wait (0: the default, 1 s)
  int sk_penalty;  // stream-K: virtual tiles charged for each segment a CTA enters
  const float* k_scales;  // FP8 cache (stream-K): this layer's K / V scale pools,
  const float* v_scales;  // contiguous (B, H_kv, T_pad) or paged (num_pages, H_kv, P)
  int T_pad;
  int sk_slot_rows;  // stream-K: rows of one partial-result slot (the rows of a row block
                     // that can be valid: min(rows per CTA, query rows per KV head))
  int sk_blocked;  // stream-K, paged, D = 128, pages < 64 tokens: the tensor maps are 4-D
                   // (64 elements, page tokens, 2 halves, page blocks), one box a page
  int sk_rb_major;  // stream-K: segments ordered row block first (every block the same
                   // number of tiles a request)
  int sk_combine;  // tcgen05 stream-K: partial pieces are merged by a separate combine
                   // launch (combine_kernel); the value is this call's generation, which the
                   // segment descriptors in sk_desc carry (0: last-finisher merges)
  int* sk_desc;    // tcgen05 stream-K with sk_combine: kCombineDescInts ints a segment
  int replan;  // dependent-launch test: the stream-K kernel treats its first plan as stale
  int stall;  // failure-detection test: the producers issue no copies, so the first
              // wait runs out (stream-K and tcgen05 kernels)
};

}  // namespace kvc
