/*
 * kvc.h -- C ABI of the B200 (sm_100a) KV-cache attention library (libkvc.so).
 *
 * The library holds a per-layer K/V cache in device memory and runs the two
 * steps of one decode (or speculative-verify) layer-step on it:
 *
 *   kvc_append  writes the new tokens' K and V into the cache, and
 *   kvc_attend  attends the new query rows over every cached position.
 *
 * Sources (web pages, cited by title and section):
 *   "9. 推理：从生成到性能优化" (goclawai.cn/llm/inference):
 *       9.3 "KV Cache" -- past K/V never change; each step projects only the
 *           new token and appends it; the KV-bytes formula;
 *       9.6 -- a paged cache managed in fixed-size blocks;
 *       9.7 -- flash attention is exact attention up to rounding.
 *   "项目 9-16: Decoding、KV Cache、长上下文与推理系统" (sshipanoo.com):
 *       project 11 -- K/V are (B, H, T, D), new K/V go after the past along
 *           T, scores are q.K^T * scale followed by softmax and a product
 *           with V; project 12 -- MQA/GQA query heads share K/V heads.
 *   "llm-perf-lab" README -- a preallocated cache with two-phase
 *       append/commit; speculative decoding verifies gamma drafted tokens in
 *       one pass and rolls the cache back to the accepted prefix.
 *
 * Conventions shared by every call:
 *   - Element type: fp16 or bf16 (kvc_dtype), the same for q, K, V and out.
 *     Arithmetic is fp32 with exact (max-subtracted) softmax.
 *   - All tensor arguments are DEVICE pointers owned by the caller, C-contiguous,
 *     16-byte aligned.  `stream` is a cudaStream_t (NULL = legacy default stream);
 *     every call is asynchronous on it.
 *   - seq_lens: device int32[B]; seq_lens[b] is the committed length L_b of request
 *     b BEFORE the new tokens.  Append and attend never modify it: committing tokens
 *     (append/commit) means raising it after the step, rolling back after a rejected
 *     speculative draft means lowering it -- by the caller, or on the device with
 *     kvc_commit / kvc_rollback.
 *   - GQA: query head h reads KV head h / (H_q / H_kv).  MHA: H_q == H_kv.  MQA: H_kv == 1.
 *   - Causality: new row i (0 <= i < T_new) of request b sees positions 0 .. L_b + i.
 *   - Paged cache: pool[page][H_kv][page_size][D] for K and for V of each layer;
 *     logical position p of request b lives in page block_table[b*max_pages + p/page_size],
 *     slot p % page_size.  block_table is device int32[B][max_pages]; entries that a
 *     call does not reach are never read.  Several requests may list the same physical
 *     page (shared prefix); appends must target pages owned by one request.
 *   - Contiguous cache: per layer K and V are (B, H_kv, max_T, D).
 *   - Host-side argument errors return a status before anything is launched.
 *     Device-side violations (a page id outside [0, num_pages), a position past the
 *     capacity, a pipeline wait that ran out) never trap: the offending write or read
 *     is skipped, a sticky error word in the cache is set, and kvc_get_error reports it.
 *   - A cache handle is not thread-safe; calls on one handle must be serialised.
 */
#ifndef KVC_H
#define KVC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KVC_OK = 0,
    KVC_ERR_INVALID_ARG = 1, /* bad shape, null pointer, misalignment, layer out of range */
    KVC_ERR_UNSUPPORTED = 2, /* a valid request this build does not implement (e.g. D=96) */
    KVC_ERR_OOM = 3,         /* device allocation failed */
    KVC_ERR_CUDA = 4,        /* a CUDA runtime call failed (launch error, no device) */
    KVC_ERR_BOUNDS = 5,      /* device side: page id or position outside the cache */
    KVC_ERR_TIMEOUT = 6,     /* device side: a bounded pipeline wait gave up */
    KVC_ERR_SCRATCH = 7      /* kvc_attend_noalloc: the call needs more than its fixed scratch */
} kvc_status;

typedef enum { KVC_FP16 = 0, KVC_BF16 = 1 } kvc_dtype;

/* How K and V are stored (kvc_create_quantized). */
typedef enum {
    KVC_KV_NATIVE = 0,   /* in the cache's dtype (kvc_create) */
    KVC_KV_FP8_E4M3 = 1  /* FP8 E4M3 codes plus one fp32 scale per (token, KV head) */
} kvc_kv_format;

typedef struct kvc_cache kvc_cache;

/*
 * kvc_create -- allocate a cache of `num_layers` layers on the current device.
 *   B          batch size (requests) the cache serves; every later call uses B requests.
 *   H_kv, D    KV heads and head dim; D must be 32, 64 or 128.
 *   max_T      per-request capacity in tokens (contiguous: allocated; paged: a bound
 *              that appends are checked against).
 *   page_size  0 = contiguous cache; otherwise tokens per page (a power of two, 1..1024).
 *   num_pages  paged pool size in pages (per layer; K and V each); must be 0 if contiguous.
 * The pools are zero-filled.  Returns KVC_ERR_OOM if device memory runs out.
 * Ownership: the handle owns the pools and any workspace; release with kvc_destroy.
 */
kvc_status kvc_create(int B, int H_kv, int D, int max_T, kvc_dtype dtype, int page_size,
                      int num_layers, int num_pages, kvc_cache** out);

/*
 * kvc_create_quantized -- kvc_create with K and V stored in `kv_format`.  The pages
 * leave KV quantisation uncovered ("llm-perf-lab" README; "9. 推理" 9.3 counts the
 * bytes a decode step reads, which FP8 halves); the format is this library's own:
 *   KVC_KV_FP8_E4M3: every appended K (and V) row x of D values becomes
 *       scale = amax / 448       (amax = max_d |x_d|; an all-zero row takes scale 1)
 *       code_d = E4M3(x_d / scale)   (nearest, ties to even, saturated to +-448)
 *     with both divisions in fp32, so codes and scales are a function of the row alone.
 *     Attention then uses code * scale exactly (up to fp32 rounding).  Code pools have
 *     the layouts of kvc_create with 1-byte elements; scale pools hold one fp32 per row:
 *     contiguous (B, H_kv, T_pad) with T_pad = max_T rounded up to a multiple of 64,
 *     paged (num_pages, H_kv, page_size).
 *     Requires dtype KVC_BF16 (q, k_new, v_new and out stay bf16), D 64 or 128, and
 *     page_size 0 or at least 8; otherwise KVC_ERR_UNSUPPORTED.
 * All other calls take the same arguments as for a native cache.  kvc_bytes counts the
 * codes and the scales.
 */
kvc_status kvc_create_quantized(int B, int H_kv, int D, int max_T, kvc_dtype dtype,
                                kvc_kv_format kv_format, int page_size, int num_layers,
                                int num_pages, kvc_cache** out);

/* kvc_destroy -- free the pools, workspace and handle (synchronises the device). NULL is ok. */
kvc_status kvc_destroy(kvc_cache* cache);

/*
 * kvc_bytes -- bytes held by the K and V pools, following the KV-bytes formula of
 * "9. 推理" section 9.3: 2 x layers x kv_heads x head_dim x T x bytes x batch, where
 * T x batch is max_T x B for a contiguous cache and num_pages x page_size for a paged
 * one.  Page tables and workspace are not counted (the page excludes them too).
 */
size_t kvc_bytes(const kvc_cache* cache);

/* kvc_bytes_formula -- the same formula as a pure function (no cache needed). */
size_t kvc_bytes_formula(int layers, int kv_heads, int head_dim, long long seq_len,
                         int bytes_per_elem, int batch);

/*
 * kvc_append -- write the new tokens of one layer into the cache ("9. 推理" 9.3;
 * "项目 9-16" project 11's concatenation, done in place).
 *   k_new, v_new  device (B, H_kv, T_new, D) in the cache dtype.
 *   T_new         tokens per request (>= 1).
 *   block_table   device int32 (B, max_pages) for a paged cache, NULL for a contiguous one.
 *   seq_lens      device int32 (B): new token i of request b goes to position seq_lens[b]+i.
 * Writes are bit-exact copies.  Positions >= max_T, or whose page id is outside the pool,
 * are skipped and flag KVC_ERR_BOUNDS.
 */
kvc_status kvc_append(kvc_cache* cache, int layer, const void* k_new, const void* v_new,
                      int T_new, const int32_t* block_table, int max_pages,
                      const int32_t* seq_lens, void* stream);

/*
 * kvc_attend -- exact-softmax attention of the new query rows of one layer over every
 * cached position ("项目 9-16" projects 11/15; "9. 推理" 9.7).
 *   q      device (B, H_q, T_new, D); H_q must be a multiple of H_kv.
 *   T_new  1 for decode, gamma for a speculative-verify chunk (causal within the chunk).
 *   block_table, max_pages, seq_lens as for kvc_append (the appended rows are visible).
 *   scale  multiplies q.k (callers normally pass 1/sqrt(D)).
 *   out    device (B, H_q, T_new, D), written in the cache dtype.
 * Must follow the kvc_append of the same tokens on the same stream.  Uses a workspace
 * owned by the cache for split-K partial results; it grows on demand (a device
 * allocation, so the first call with a larger shape should precede any stream capture;
 * kvc_reserve sizes it up front).
 * Launch: when the plan picks a persistent kernel (no window; D 64/128; stream-K on
 * mma.sync for 1-16 query rows per KV head, 1-8 on an FP8 cache; stream-K on tcgen05
 * for 17 or more), it is launched with programmatic stream serialization.  It may start
 * while the kernel ahead of it on the stream retires, but reads no input that counts and
 * writes nothing before that kernel has completed (before that it only reads seq_lens
 * and the block table to plan, and prefetches K/V lines into L2; if the lengths changed
 * by then, it plans again).  The environment variable KVC_PDL=0 (read at kvc_create) or
 * kvc_set_dependent_launch turns this into a plain launch.  On the tcgen05 path a
 * segment whose partial results are large is merged by a second, dependent launch on
 * `stream` (the combine); callers see one call either way.
 */
kvc_status kvc_attend(kvc_cache* cache, int layer, const void* q, int H_q, int T_new,
                      const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                      float scale, void* out, void* stream);

/*
 * kvc_attend_window -- kvc_attend restricted to a sliding window with attention sinks
 * ("项目 9-16" roadmap: sliding-window attention over the last W positions, with the
 * first positions kept as attention sinks).  New row i of request b (n = L_b + i + 1
 * positions, causal within the chunk) attends position j iff
 *     j < n  and  (j >= n - window  or  j < sink);
 * window = 0 means no window (exactly kvc_attend; sink is then irrelevant).  Only the
 * positions some row of a block can see are read, so the cost follows W + sink, not n.
 * Other arguments, layouts and errors as kvc_attend; window or sink < 0 is
 * KVC_ERR_INVALID_ARG.
 */
kvc_status kvc_attend_window(kvc_cache* cache, int layer, const void* q, int H_q, int T_new,
                             const int32_t* block_table, int max_pages, const int32_t* seq_lens,
                             float scale, int window, int sink, void* out, void* stream);

/*
 * kvc_append_attend -- kvc_append followed by kvc_attend for the same new tokens, in
 * one launch where the kernel allows it ("9. 推理" 9.3: the new token's K/V join the
 * cache and are attended in the same step).  Arguments are those of the two calls.
 * On the persistent stream-K kernels the attend kernel itself writes the new rows into
 * the cache: on mma.sync (up to 16 query rows per KV head, up to 8 on an FP8 cache; an
 * FP8 cache quantised exactly as kvc_append does) it also uses them straight from
 * k_new / v_new; on tcgen05 (17 or more rows) its copy warps store them into the cache
 * before they load those tiles (the combine launch, where the plan has one, follows).
 * The fixed-split plans (sliding windows, 9+ rows on an FP8 cache, batches beyond the
 * stream-K scan) run the two kernels back to back on `stream`.  Results (cache contents
 * and out) are identical to calling kvc_append then kvc_attend for valid inputs; a
 * request whose new rows would overflow its capacity is flagged KVC_ERR_BOUNDS, and the
 * fused kernels then write none of its rows.
 */
kvc_status kvc_append_attend(kvc_cache* cache, int layer, const void* k_new, const void* v_new,
                             const void* q, int H_q, int T_new, const int32_t* block_table,
                             int max_pages, const int32_t* seq_lens, float scale, void* out,
                             void* stream);

/*
 * kvc_attend_noalloc -- kvc_attend without any device allocation.  The pages have no
 * counterpart of this call: it exists for callers that cannot let a library allocate
 * device memory -- code recording a step inside CUDA stream capture (cudaMalloc cannot
 * be captured), engines whose caching allocator owns almost all device memory (a side
 * allocation can fail or fragment its pool), and latency-bound loops that cannot afford
 * the device synchronisation that cudaFree implies.
 *   Arguments, layouts and results are those of kvc_attend.  The split-K scratch
 *   (partial results and slice tickets) lives in one fixed 16 MiB device array that the
 *   library holds on every GPU that loads it, until the process exits.  A call whose plan
 *   needs more scratch than that returns KVC_ERR_SCRATCH before launching anything
 *   (decode with up to 16 query rows per KV head needs about 2.5 MB on a 148-SM B200).
 *   The first call on a device looks up the array's device address (once per device);
 *   make that first call before any stream capture.  Each call clears the tickets it
 *   uses with an asynchronous memset on `stream`.  Every call shares the one array, so
 *   calls whose executions overlap on the GPU (other streams, other threads, other cache
 *   handles on the same device) race with each other and must be serialised by the caller.
 */
kvc_status kvc_attend_noalloc(kvc_cache* cache, int layer, const void* q, int H_q, int T_new,
                              const int32_t* block_table, int max_pages,
                              const int32_t* seq_lens, float scale, void* out, void* stream);

/*
 * kvc_reserve -- size the attend workspace for up to `H_q` query heads, `T_new` new rows
 * and `max_pages` block-table columns, so that later kvc_attend calls allocate nothing.
 */
kvc_status kvc_reserve(kvc_cache* cache, int H_q, int T_new, int max_pages);

/*
 * kvc_get_error -- synchronise the device, return the sticky device error (KVC_OK,
 * KVC_ERR_BOUNDS or KVC_ERR_TIMEOUT) and clear it.
 */
kvc_status kvc_get_error(kvc_cache* cache);

/*
 * kvc_set_dependent_launch -- launch this cache's persistent attend kernels with
 * programmatic stream serialization (on != 0; the default unless the environment
 * variable KVC_PDL=0) or as a plain launch (on == 0).  Results are the same either way;
 * see kvc_attend.
 */
kvc_status kvc_set_dependent_launch(kvc_cache* cache, int on);

/*
 * kvc_set_wait_limit -- bound, in nanoseconds of %globaltimer, of every pipeline wait in
 * the later attend launches on this cache (0 restores the default of one second).  A wait
 * that runs out never hangs or traps: the kernel records KVC_ERR_TIMEOUT in the sticky
 * error word, finishes without waiting again, and kvc_get_error reports it.
 */
kvc_status kvc_set_wait_limit(kvc_cache* cache, unsigned long long ns);

/*
 * kvc_inject_stall -- failure-detection test hook.  The next attend call on this cache,
 * if it runs the persistent stream-K or the tcgen05 kernel, issues none of its copies,
 * so its first pipeline wait runs out after the wait limit (kvc_set_wait_limit) and
 * kvc_get_error then returns KVC_ERR_TIMEOUT; that call's output is undefined, the
 * cache and the device context stay usable.  Other kernels ignore it; the next call
 * consumes it either way.
 */
kvc_status kvc_inject_stall(kvc_cache* cache);

/*
 * kvc_inject_replan -- test hook for the dependent launch.  The persistent stream-K
 * kernels plan their range from the lengths they read before the dependency wait and
 * read the lengths again after it; if they changed, they plan again.  The mma.sync
 * kernel issues its first copies from the first plan right after the wait, so it also
 * waits for those copies and resets its pipeline first; the tcgen05 kernel issues
 * nothing before the check.  This hook makes the next attend call on this cache
 * (stream-K only) take that path whatever the lengths: its results are the same as
 * without it.  The next call consumes it either way.
 */
kvc_status kvc_inject_replan(kvc_cache* cache);

/* kvc_status_string -- static, human-readable name of a status. */
const char* kvc_status_string(kvc_status status);

/* kvc_k_pool / kvc_v_pool -- device address of a layer's K / V pool (NULL if out of range);
 * for initialising history and for bit-exact inspection. */
void* kvc_k_pool(kvc_cache* cache, int layer);
void* kvc_v_pool(kvc_cache* cache, int layer);

/* kvc_layer_pool_bytes -- bytes of one layer's K (equally V) pool. */
size_t kvc_layer_pool_bytes(const kvc_cache* cache);

/* kvc_k_scales / kvc_v_scales -- device address of a layer's fp32 K / V scale pool of a
 * quantised cache (NULL for a native cache or a layer out of range); kvc_layer_scale_floats
 * -- the number of scales in one of them (0 for a native cache). */
float* kvc_k_scales(kvc_cache* cache, int layer);
float* kvc_v_scales(kvc_cache* cache, int layer);
size_t kvc_layer_scale_floats(const kvc_cache* cache);

/*
 * kvc_commit -- advance every request's committed length by its accepted count
 * ("llm-perf-lab" README: the preallocated cache commits in two phases, append then
 * commit, and speculative decoding keeps only the accepted prefix of the gamma verified
 * tokens).  After an append of T_new tokens at positions L_b .. L_b+T_new-1, the
 * caller accepts accepted[b] of them and this call sets seq_lens[b] = L_b + accepted[b],
 * on the device and in stream order (accepted[] is typically written by the verify
 * step's own kernels, so the host never waits).  Positions past the new length keep the
 * rejected K/V until the next append overwrites them; no attend reads them.
 *   seq_lens   device int32[B], updated in place.
 *   accepted   device int32[B].
 *   T_new      the number of appended tokens the counts refer to.
 * A count outside [0, T_new] or a new length above max_T leaves that request unchanged
 * and sets KVC_ERR_BOUNDS in the sticky error word.
 */
kvc_status kvc_commit(kvc_cache* cache, int32_t* seq_lens, const int32_t* accepted, int T_new,
                      void* stream);

/*
 * kvc_rollback -- lower every request's committed length: seq_lens[b] -= drop[b]
 * ("llm-perf-lab" README: rolling the cache back).  The dropped positions' K/V stay in
 * the pools until an append overwrites them.  A drop outside [0, seq_lens[b]] leaves
 * that request unchanged and sets KVC_ERR_BOUNDS.  seq_lens, drop: device int32[B].
 */
kvc_status kvc_rollback(kvc_cache* cache, int32_t* seq_lens, const int32_t* drop, void* stream);

/*
 * kvc_copy_pages -- make page dst[i] a bit-exact copy of page src[i] (i < n) in every
 * layer, K and V, of a paged cache ("9. 推理" 9.6: a cache managed in fixed-size pages).
 * This is the copy of copy-on-write: before an append would land in a page that other
 * requests also list (a shared prefix whose last page is partly filled), the caller,
 * which owns page reference counts and block tables, takes a free page, copies the
 * shared page into it with this call and points the request's block-table entry at the
 * copy, then appends.
 *   src, dst   device int32[n] page ids in [0, num_pages).  The dst pages must be
 *              distinct and none may also be a src page of the same call.
 * Contiguous caches return KVC_ERR_UNSUPPORTED.  A page id outside the pool skips that
 * pair and sets KVC_ERR_BOUNDS.
 */
kvc_status kvc_copy_pages(kvc_cache* cache, const int32_t* src, const int32_t* dst, int n,
                          void* stream);

/*
 * kvc_plan_splits -- how kvc_attend would divide the work for these arguments (for
 * measurement and tests).  Fixed-size split-K: *num_splits slices of *split_tokens tokens
 * per (request, KV head).  Persistent stream-K (no window, D 64/128, B up to the
 * kernel's scan capacity; any number of query rows per KV head, at most 8 on an FP8
 * cache): *num_splits is the number of persistent CTAs, each streaming an equal share of
 * all K/V tiles, and *split_tokens is 0.
 */
kvc_status kvc_plan_splits(const kvc_cache* cache, int H_q, int T_new, int max_pages,
                           int* num_splits, int* split_tokens);

#ifdef __cplusplus
}
#endif

#endif /* KVC_H */
