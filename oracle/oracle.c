/*
 * oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU statement of the KV-cache attention step of
 * autoregressive decoding.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library; the product path never
 * does, and this file shares no code, header or table with the CUDA path.
 *
 * Sources (web pages, cited by title and section):
 *   [P1] "llm-perf-lab" README (github JingHao-Leon/llm-perf-lab):
 *        the preallocated two-phase append/commit KV cache, the statement
 *        that cached decoding reproduces full-sequence logits, and the
 *        statement that chunked attention equals naive attention for any
 *        chunk size.
 *   [P2] "项目 9-16: Decoding、KV Cache、长上下文与推理系统" (sshipanoo.com
 *        LLM roadmap), project 11 "实现 KV cache" (the CachedSelfAttention
 *        snippet: K/V laid out (B, H, T, D), new K/V concatenated after the
 *        past along T, scores q.K^T / sqrt(head_dim), softmax, times V),
 *        project 12 (MQA/GQA: query heads share K/V heads) and project 15
 *        (naive attention materialises the score matrix; SDPA/FlashAttention
 *        gives the same mathematical result).
 *   [P3] "9. 推理：从生成到性能优化" (goclawai.cn/llm/inference), section 9.3
 *        "KV Cache" (past K/V never change, only the new token is projected
 *        and appended; the KV-bytes formula and its worked 32-layer example),
 *        section 9.6 (paged KV cache managed in blocks), section 9.7 (flash
 *        attention is exact up to floating-point rounding).
 *
 * Readings where the pages are silent:
 *   - causal within the new chunk: new row i of a request with committed
 *     length L sees positions 0 .. L+i (the project-11 snippet applies no
 *     mask, which is only right for one new row);
 *   - GQA head mapping: query head h uses KV head h / (H_q / H_kv);
 *   - paged pool layout: pool[page][kv_head][slot][d], logical position
 *     pos of request b lives in page block_table[b][pos / P], slot pos % P.
 *
 * Every floating-point step is in IEEE double, sums run in index order, and
 * exp() is libm's.  16-bit inputs are decoded exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <omp.h>

#define ORACLE_FP16 0
#define ORACLE_BF16 1

/* ------------------------------------------------------------------ */
/* 16-bit storage formats <-> double (IEEE 754 binary16; bfloat16 is the */
/* top half of an IEEE binary32).                                       */
/* ------------------------------------------------------------------ */

static double decode_fp16(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int mant = h & 0x3ff;
    double v;
    if (expo == 0)
        v = ldexp((double)mant, -24); /* subnormal: mant * 2^-24 */
    else if (expo == 31)
        v = mant ? NAN : INFINITY;
    else
        v = ldexp((double)(mant + 1024), expo - 25); /* 1.mant * 2^(e-15) */
    return sign ? -v : v;
}

static double decode_bf16(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double decode(uint16_t h, int dtype)
{
    return dtype == ORACLE_BF16 ? decode_bf16(h) : decode_fp16(h);
}

/*
 * Round a double to the nearest value with `p` significant bits whose
 * normal exponents run from emin to emax, ties to even, and encode it.
 * fp16: p=11, emin=-14, emax=15, 5 exponent bits, bias 15.
 * bf16: p=8, emin=-126, emax=127, 8 exponent bits, bias 127.
 */
static uint16_t encode_rne(double x, int p, int emin, int emax, int ebits)
{
    uint16_t sign = signbit(x) ? (uint16_t)(1u << 15) : 0;
    int mbits = p - 1;
    uint16_t inf = (uint16_t)(((1u << ebits) - 1) << mbits);
    if (isnan(x))
        return (uint16_t)(inf | (1u << (mbits - 1)));
    double a = fabs(x);
    if (isinf(a))
        return sign | inf;
    if (a == 0.0)
        return sign;
    int e;
    frexp(a, &e);          /* a = f * 2^e, f in [0.5, 1): unbiased exponent e-1 */
    int E = e - 1;
    if (E < emin)
        E = emin;          /* subnormal range shares the smallest quantum */
    double quantum = ldexp(1.0, E - mbits);
    double r = nearbyint(a / quantum); /* exact division; default mode = ties-to-even */
    if (r >= ldexp(1.0, p)) { /* mantissa carried into the next binade */
        r /= 2.0;
        E += 1;
    }
    if (E > emax)
        return sign | inf;
    uint32_t m = (uint32_t)r; /* < 2^p */
    if (m < (1u << mbits))    /* subnormal or zero after rounding */
        return sign | (uint16_t)m;
    uint32_t biased = (uint32_t)(E + (1 << (ebits - 1)) - 1);
    return sign | (uint16_t)((biased << mbits) | (m - (1u << mbits)));
}

int oracle_max_threads(void) { return omp_get_max_threads(); }

void oracle_decode(const uint16_t* src, double* dst, int64_t n, int dtype)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = decode(src[i], dtype);
}

void oracle_round(const double* src, uint16_t* dst, int64_t n, int dtype)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = dtype == ORACLE_BF16 ? encode_rne(src[i], 8, -126, 127, 8)
                                      : encode_rne(src[i], 11, -14, 15, 5);
}

/* ------------------------------------------------------------------ */
/* [P3] section 9.3: KV bytes = 2 x layers x kv_heads x head_dim x      */
/* sequence_length x bytes_per_element x batch (the 2 counts K and V).  */
/* ------------------------------------------------------------------ */
uint64_t oracle_kv_bytes(int64_t layers, int64_t kv_heads, int64_t head_dim,
                         int64_t seq_len, int64_t bytes_per_elem, int64_t batch)
{
    return (uint64_t)2 * (uint64_t)layers * (uint64_t)kv_heads * (uint64_t)head_dim *
           (uint64_t)seq_len * (uint64_t)bytes_per_elem * (uint64_t)batch;
}

/* ------------------------------------------------------------------ */
/* Append ([P1] append/commit cache; [P2] project 11 concatenation      */
/* along T; [P3] 9.3: only the new token's K/V are added, the past is   */
/* never touched).  new_kv: (B, H_kv, T_new, D).  Values are copied as  */
/* raw 16-bit words.                                                    */
/* ------------------------------------------------------------------ */

/* Contiguous cache (B, H_kv, T_cap, D): row L_b + i receives new row i. */
void oracle_append_contig(int B, int H_kv, int T_new, int D, int T_cap,
                          const uint16_t* new_kv, const int32_t* seq_lens,
                          uint16_t* cache)
{
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < H_kv; ++g)
            for (int i = 0; i < T_new; ++i) {
                int64_t pos = (int64_t)seq_lens[b] + i;
                const uint16_t* src = new_kv + (((int64_t)b * H_kv + g) * T_new + i) * D;
                uint16_t* dst = cache + (((int64_t)b * H_kv + g) * T_cap + pos) * D;
                for (int d = 0; d < D; ++d)
                    dst[d] = src[d];
            }
}

/* Paged pool (num_pages, H_kv, P, D): position pos of request b is slot
 * pos % P of page block_table[b * max_pages + pos / P] ([P3] 9.6). */
void oracle_append_paged(int B, int H_kv, int T_new, int D, int P, int max_pages,
                         const uint16_t* new_kv, const int32_t* seq_lens,
                         const int32_t* block_table, uint16_t* pool)
{
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < H_kv; ++g)
            for (int i = 0; i < T_new; ++i) {
                int64_t pos = (int64_t)seq_lens[b] + i;
                int64_t page = block_table[(int64_t)b * max_pages + pos / P];
                int64_t slot = pos % P;
                const uint16_t* src = new_kv + (((int64_t)b * H_kv + g) * T_new + i) * D;
                uint16_t* dst = pool + ((page * H_kv + g) * P + slot) * D;
                for (int d = 0; d < D; ++d)
                    dst[d] = src[d];
            }
}

/* ------------------------------------------------------------------ */
/* FP8 (E4M3) cache.  The pages leave KV quantisation uncovered ([P1];   */
/* [P3] 9.3 counts the bytes a decode step reads); the format is stated  */
/* in full here.  E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa */
/* bits, no infinities, S.1111.111 is NaN, largest finite value 448.     */
/* A row x of D values is stored as                                      */
/*   scale = amax / 448 (fp32; amax = max |x_d|; scale 1 if amax == 0)   */
/*   code_d = E4M3(x_d / scale) (fp32 division; nearest value, ties to   */
/*            the even code, magnitudes at or above 448 give 448).       */
/* ------------------------------------------------------------------ */

static double decode_e4m3(uint8_t c)
{
    int sign = (c >> 7) & 1;
    int e = (c >> 3) & 15;
    int m = c & 7;
    if (e == 15 && m == 7)
        return NAN;
    double v = (e == 0) ? ldexp((double)m, -9)            /* subnormal: m * 2^-9 */
                        : ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
    return sign ? -v : v;
}

/* Nearest finite E4M3 value by search over the 127 non-negative finite codes;
 * a tie takes the code whose last mantissa bit is 0. */
static uint8_t encode_e4m3(float xf)
{
    double x = (double)xf;
    if (x != x)
        return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00; /* -0 keeps its sign */
    double a = fabs(x);
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7E);
    static double value[0x7F]; /* the non-negative finite codes, decoded once */
    static int ready = 0;
    if (!ready) {
        for (int c = 0; c <= 0x7E; ++c)
            value[c] = decode_e4m3((uint8_t)c);
        ready = 1;
    }
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs(value[c] - a);
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    if (best == 0)
        return 0x00 | sign; /* +0 / -0 */
    return (uint8_t)(sign | best);
}

void oracle_decode_e4m3(const uint8_t* src, double* dst, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = decode_e4m3(src[i]);
}

void oracle_encode_e4m3(const float* src, uint8_t* dst, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = encode_e4m3(src[i]);
}

/* One row x of D bf16 words -> D codes and its scale. */
static void quantize_row(const uint16_t* x, int D, uint8_t* code, float* scale_out)
{
    float amax = 0.0f;
    for (int d = 0; d < D; ++d) {
        float v = (float)decode_bf16(x[d]);
        float av = v < 0 ? -v : v;
        if (av > amax)
            amax = av;
    }
    float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
    *scale_out = scale;
    for (int d = 0; d < D; ++d) {
        float v = (float)decode_bf16(x[d]);
        code[d] = encode_e4m3(v / scale);
    }
}

/* rows (n_rows, D) of bf16 words -> codes (n_rows, D) and scales (n_rows) */
void oracle_quantize_fp8(const uint16_t* rows, int64_t n_rows, int D, uint8_t* codes,
                         float* scales)
{
    for (int64_t r = 0; r < n_rows; ++r)
        quantize_row(rows + r * D, D, codes + r * D, &scales[r]);
}

/* FP8 append into a contiguous cache: new row i of (b, g) (bf16 words,
 * new_kv (B, H_kv, T_new, D)) is quantised and lands at position
 * pos = seq_lens[b] + i -- its D codes in codes (B, H_kv, T_cap, D), its
 * scale in scales (B, H_kv, T_pad), the scale rows being T_pad long. */
void oracle_append_fp8_contig(int B, int H_kv, int T_new, int D, int T_cap, int T_pad,
                              const uint16_t* new_kv, const int32_t* seq_lens,
                              uint8_t* codes, float* scales)
{
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < H_kv; ++g)
            for (int i = 0; i < T_new; ++i) {
                int64_t pos = (int64_t)seq_lens[b] + i;
                const uint16_t* src = new_kv + (((int64_t)b * H_kv + g) * T_new + i) * D;
                int64_t code_row = ((int64_t)b * H_kv + g) * T_cap + pos;
                int64_t scale_at = ((int64_t)b * H_kv + g) * T_pad + pos;
                quantize_row(src, D, codes + code_row * D, &scales[scale_at]);
            }
}

/* FP8 append into a paged pool ([P3] 9.6): position pos of request b is slot
 * pos % P of page block_table[b * max_pages + pos / P]; codes are
 * (num_pages, H_kv, P, D), scales (num_pages, H_kv, P). */
void oracle_append_fp8_paged(int B, int H_kv, int T_new, int D, int P, int max_pages,
                             const uint16_t* new_kv, const int32_t* seq_lens,
                             const int32_t* block_table, uint8_t* codes, float* scales)
{
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < H_kv; ++g)
            for (int i = 0; i < T_new; ++i) {
                int64_t pos = (int64_t)seq_lens[b] + i;
                int64_t page = block_table[(int64_t)b * max_pages + pos / P];
                int64_t slot = pos % P;
                const uint16_t* src = new_kv + (((int64_t)b * H_kv + g) * T_new + i) * D;
                int64_t row = (page * H_kv + g) * P + slot;
                quantize_row(src, D, codes + row * D, &scales[row]);
            }
}

/* Logical rows of a paged pool of fixed-size rows (any element type): row pos of
 * (b, g) is row slot = pos % P of page block_table[b][pos / P]. */
void oracle_gather_rows(int B, int H_kv, int row_bytes, int P, int max_pages, int T_cap,
                        const uint8_t* pool, const int32_t* block_table,
                        const int32_t* n_visible, uint8_t* out)
{
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < H_kv; ++g)
            for (int64_t pos = 0; pos < n_visible[b]; ++pos) {
                int64_t page = block_table[(int64_t)b * max_pages + pos / P];
                int64_t slot = pos % P;
                const uint8_t* src = pool + ((page * H_kv + g) * P + slot) * row_bytes;
                uint8_t* dst = out + (((int64_t)b * H_kv + g) * T_cap + pos) * row_bytes;
                for (int k = 0; k < row_bytes; ++k)
                    dst[k] = src[k];
            }
}

/* Attention of bf16 queries over FP8 K/V: K[j] = code * scale exactly, in fp64;
 * the visibility rule of oracle_attend_window (window 0: all positions). */
static void attend_row_fp8(int D, int n, int W, int S, const uint16_t* qrow,
                           const uint8_t* Kc, const float* Ks, const uint8_t* Vc,
                           const float* Vs, double scale, double* orow)
{
    double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    char* seen = (char*)malloc((size_t)(n > 0 ? n : 1));
    double* qd = (double*)malloc(sizeof(double) * (size_t)D);
    for (int d = 0; d < D; ++d)
        qd[d] = decode_bf16(qrow[d]);
    for (int j = 0; j < n; ++j) {
        seen[j] = (W == 0 || j >= n - W || j < S);
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += qd[d] * (decode_e4m3(Kc[(int64_t)j * D + d]) * (double)Ks[j]);
        s[j] = scale * dot;
    }
    double mx = -INFINITY;
    for (int j = 0; j < n; ++j)
        if (seen[j] && s[j] > mx)
            mx = s[j];
    double denom = 0.0;
    for (int j = 0; j < n; ++j) {
        s[j] = seen[j] ? exp(s[j] - mx) : 0.0;
        denom += s[j];
    }
    for (int d = 0; d < D; ++d)
        orow[d] = 0.0;
    for (int j = 0; j < n; ++j) {
        if (!seen[j])
            continue;
        double pj = s[j] / denom;
        for (int d = 0; d < D; ++d)
            orow[d] += pj * (decode_e4m3(Vc[(int64_t)j * D + d]) * (double)Vs[j]);
    }
    free(qd);
    free(seen);
    free(s);
}

/* q: (B, H_q, T_new, D) bf16 words; Kc, Vc: (B, H_kv, T_cap, D) codes;
 * Ks, Vs: (B, H_kv, T_cap) scales. */
void oracle_attend_fp8(int B, int H_q, int H_kv, int T_new, int D, int T_cap,
                       const uint16_t* q, const uint8_t* Kc, const float* Ks,
                       const uint8_t* Vc, const float* Vs, const int32_t* seq_lens,
                       double scale, int window, int sink, double* out, int nthreads)
{
    int group = H_q / H_kv;
    int64_t nrows = (int64_t)B * H_q * T_new;
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int64_t r = 0; r < nrows; ++r) {
        int i = (int)(r % T_new);
        int h = (int)((r / T_new) % H_q);
        int b = (int)(r / ((int64_t)T_new * H_q));
        int g = h / group;
        int n = seq_lens[b] + i + 1;
        int64_t base = ((int64_t)b * H_kv + g) * T_cap;
        attend_row_fp8(D, n, window, sink, q + r * D, Kc + base * D, Ks + base, Vc + base * D,
                       Vs + base, scale, out + r * D);
    }
}

/* ------------------------------------------------------------------ */
/* Commit, rollback and page copy ([P1]: a two-phase append/commit      */
/* cache; speculative decoding keeps the accepted prefix of the         */
/* verified tokens and rolls the rest back; [P3] 9.6: fixed-size pages).*/
/* A request (or page pair) whose values are out of range is left as it */
/* is; the number of those is returned.                                 */
/* ------------------------------------------------------------------ */

/* seq_lens[b] becomes seq_lens[b] + accepted[b] when 0 <= accepted[b] <= T_new
 * and the result stays within the capacity max_T. */
int oracle_commit(int B, int32_t* seq_lens, const int32_t* accepted, int T_new, int max_T)
{
    int rejected = 0;
    for (int b = 0; b < B; ++b) {
        int64_t grown = (int64_t)seq_lens[b] + accepted[b];
        if (accepted[b] < 0 || accepted[b] > T_new || seq_lens[b] < 0 || grown > max_T) {
            ++rejected;
            continue;
        }
        seq_lens[b] = (int32_t)grown;
    }
    return rejected;
}

/* seq_lens[b] becomes seq_lens[b] - drop[b] when 0 <= drop[b] <= seq_lens[b]. */
int oracle_rollback(int B, int32_t* seq_lens, const int32_t* drop)
{
    int rejected = 0;
    for (int b = 0; b < B; ++b) {
        if (drop[b] < 0 || drop[b] > seq_lens[b]) {
            ++rejected;
            continue;
        }
        seq_lens[b] -= drop[b];
    }
    return rejected;
}

/* One pool of num_pages pages of page_elems elements: page dst[i] receives a
 * copy of page src[i] for every i < n whose two ids lie in [0, num_pages). */
int oracle_copy_pages(int num_pages, int64_t page_elems, const int32_t* src,
                      const int32_t* dst, int n, uint16_t* pool)
{
    int rejected = 0;
    for (int i = 0; i < n; ++i) {
        if (src[i] < 0 || src[i] >= num_pages || dst[i] < 0 || dst[i] >= num_pages) {
            ++rejected;
            continue;
        }
        const uint16_t* from = pool + (int64_t)src[i] * page_elems;
        uint16_t* to = pool + (int64_t)dst[i] * page_elems;
        for (int64_t e = 0; e < page_elems; ++e)
            to[e] = from[e];
    }
    return rejected;
}

/* Logical view of request b's first n_b positions from the paged pool:
 * out (B, H_kv, T_cap, D), rows >= n_b left untouched. */
void oracle_gather_paged(int B, int H_kv, int D, int P, int max_pages, int T_cap,
                         const uint16_t* pool, const int32_t* block_table,
                         const int32_t* n_visible, uint16_t* out)
{
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < H_kv; ++g)
            for (int64_t pos = 0; pos < n_visible[b]; ++pos) {
                int64_t page = block_table[(int64_t)b * max_pages + pos / P];
                int64_t slot = pos % P;
                const uint16_t* src = pool + ((page * H_kv + g) * P + slot) * D;
                uint16_t* dst = out + (((int64_t)b * H_kv + g) * T_cap + pos) * D;
                for (int d = 0; d < D; ++d)
                    dst[d] = src[d];
            }
}

/* ------------------------------------------------------------------ */
/* Attend: the naive definition ([P2] projects 11 and 15; exact        */
/* softmax).  q: (B, H_q, T_new, D).  K, V: logical caches             */
/* (B, H_kv, T_cap, D) that already hold the T_new appended rows at    */
/* positions L_b .. L_b+T_new-1.  out: (B, H_q, T_new, D) doubles.     */
/*                                                                      */
/* For request b, query head h, new row i:                              */
/*   g = h / (H_q / H_kv),  n = L_b + i + 1 visible positions,          */
/*   s_j = scale * sum_d q[b,h,i,d] K[b,g,j,d]          (j < n)          */
/*   p_j = exp(s_j - max_k s_k) / sum_k exp(s_k - max_k s_k)             */
/*   out[b,h,i,:] = sum_j p_j V[b,g,j,:]                                 */
/* The whole score row is materialised, as in the naive form.          */
/* ------------------------------------------------------------------ */

static void attend_row(int D, int n, const uint16_t* qrow, const uint16_t* Kbase,
                       const uint16_t* Vbase, int dtype, double scale, double* orow)
{
    double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double* qd = (double*)malloc(sizeof(double) * (size_t)D);
    for (int d = 0; d < D; ++d)
        qd[d] = decode(qrow[d], dtype);
    for (int j = 0; j < n; ++j) {
        double dot = 0.0;
        const uint16_t* krow = Kbase + (int64_t)j * D;
        for (int d = 0; d < D; ++d)
            dot += qd[d] * decode(krow[d], dtype);
        s[j] = scale * dot;
    }
    double mx = -INFINITY;
    for (int j = 0; j < n; ++j)
        if (s[j] > mx)
            mx = s[j];
    double denom = 0.0;
    for (int j = 0; j < n; ++j) {
        s[j] = exp(s[j] - mx);
        denom += s[j];
    }
    for (int d = 0; d < D; ++d)
        orow[d] = 0.0;
    for (int j = 0; j < n; ++j) {
        double pj = s[j] / denom;
        const uint16_t* vrow = Vbase + (int64_t)j * D;
        for (int d = 0; d < D; ++d)
            orow[d] += pj * decode(vrow[d], dtype);
    }
    free(qd);
    free(s);
}

void oracle_attend(int B, int H_q, int H_kv, int T_new, int D, int T_cap,
                   const uint16_t* q, const uint16_t* K, const uint16_t* V, int dtype,
                   const int32_t* seq_lens, double scale, double* out, int nthreads)
{
    int group = H_q / H_kv;
    int64_t nrows = (int64_t)B * H_q * T_new;
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int64_t r = 0; r < nrows; ++r) {
        int i = (int)(r % T_new);
        int h = (int)((r / T_new) % H_q);
        int b = (int)(r / ((int64_t)T_new * H_q));
        int g = h / group;
        int n = seq_lens[b] + i + 1;
        const uint16_t* Kb = K + ((int64_t)b * H_kv + g) * T_cap * D;
        const uint16_t* Vb = V + ((int64_t)b * H_kv + g) * T_cap * D;
        attend_row(D, n, q + r * D, Kb, Vb, dtype, scale, out + r * D);
    }
}

/*
 * Sliding-window attention with attention sinks ([P2] roadmap: sliding-window
 * attention keeps each query's last W positions; attention sinks keep the first
 * S positions as well).  The row with n positions attends position j iff
 *   j < n  and  (W == 0  or  j >= n - W  or  j < S);
 * W == 0 is full attention.  Otherwise the naive definition: every score is
 * materialised, invisible ones are excluded from the max, the sum and the
 * weighted V sum.
 */
static void attend_row_window(int D, int n, int W, int S, const uint16_t* qrow,
                              const uint16_t* Kbase, const uint16_t* Vbase, int dtype,
                              double scale, double* orow)
{
    double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    char* seen = (char*)malloc((size_t)(n > 0 ? n : 1));
    double* qd = (double*)malloc(sizeof(double) * (size_t)D);
    for (int d = 0; d < D; ++d)
        qd[d] = decode(qrow[d], dtype);
    for (int j = 0; j < n; ++j) {
        seen[j] = (W == 0 || j >= n - W || j < S);
        double dot = 0.0;
        const uint16_t* krow = Kbase + (int64_t)j * D;
        for (int d = 0; d < D; ++d)
            dot += qd[d] * decode(krow[d], dtype);
        s[j] = scale * dot;
    }
    double mx = -INFINITY;
    for (int j = 0; j < n; ++j)
        if (seen[j] && s[j] > mx)
            mx = s[j];
    double denom = 0.0;
    for (int j = 0; j < n; ++j) {
        s[j] = seen[j] ? exp(s[j] - mx) : 0.0;
        denom += s[j];
    }
    for (int d = 0; d < D; ++d)
        orow[d] = 0.0;
    for (int j = 0; j < n; ++j) {
        if (!seen[j])
            continue;
        double pj = s[j] / denom;
        const uint16_t* vrow = Vbase + (int64_t)j * D;
        for (int d = 0; d < D; ++d)
            orow[d] += pj * decode(vrow[d], dtype);
    }
    free(qd);
    free(seen);
    free(s);
}

void oracle_attend_window(int B, int H_q, int H_kv, int T_new, int D, int T_cap,
                          const uint16_t* q, const uint16_t* K, const uint16_t* V, int dtype,
                          const int32_t* seq_lens, double scale, int window, int sink,
                          double* out, int nthreads)
{
    int group = H_q / H_kv;
    int64_t nrows = (int64_t)B * H_q * T_new;
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int64_t r = 0; r < nrows; ++r) {
        int i = (int)(r % T_new);
        int h = (int)((r / T_new) % H_q);
        int b = (int)(r / ((int64_t)T_new * H_q));
        int g = h / group;
        int n = seq_lens[b] + i + 1;
        const uint16_t* Kb = K + ((int64_t)b * H_kv + g) * T_cap * D;
        const uint16_t* Vb = V + ((int64_t)b * H_kv + g) * T_cap * D;
        attend_row_window(D, n, window, sink, q + r * D, Kb, Vb, dtype, scale, out + r * D);
    }
}

/*
 * Chunked attention ([P1]: blocking the computation over the keys only
 * reorders it; the result equals naive attention for any chunk size).
 * Keys are taken `chunk` at a time; a running maximum m, running sum l
 * and running weighted sum acc are rescaled by exp(m_old - m_new) each
 * time the maximum grows, and out = acc / l at the end.
 */
void oracle_attend_chunked(int B, int H_q, int H_kv, int T_new, int D, int T_cap,
                           const uint16_t* q, const uint16_t* K, const uint16_t* V,
                           int dtype, const int32_t* seq_lens, double scale, int chunk,
                           double* out, int nthreads)
{
    int group = H_q / H_kv;
    int64_t nrows = (int64_t)B * H_q * T_new;
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int64_t r = 0; r < nrows; ++r) {
        int i = (int)(r % T_new);
        int h = (int)((r / T_new) % H_q);
        int b = (int)(r / ((int64_t)T_new * H_q));
        int g = h / group;
        int n = seq_lens[b] + i + 1;
        const uint16_t* Kb = K + ((int64_t)b * H_kv + g) * T_cap * D;
        const uint16_t* Vb = V + ((int64_t)b * H_kv + g) * T_cap * D;
        double* qd = (double*)malloc(sizeof(double) * (size_t)D);
        double* acc = out + r * D;
        double* s = (double*)malloc(sizeof(double) * (size_t)chunk);
        for (int d = 0; d < D; ++d) {
            qd[d] = decode(q[r * D + d], dtype);
            acc[d] = 0.0;
        }
        double m = -INFINITY, l = 0.0;
        for (int c0 = 0; c0 < n; c0 += chunk) {
            int c1 = c0 + chunk < n ? c0 + chunk : n;
            double mc = -INFINITY;
            for (int j = c0; j < c1; ++j) {
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += qd[d] * decode(Kb[(int64_t)j * D + d], dtype);
                s[j - c0] = scale * dot;
                if (s[j - c0] > mc)
                    mc = s[j - c0];
            }
            double m_new = mc > m ? mc : m;
            double alpha = exp(m - m_new); /* m = -inf on the first chunk: alpha = 0 */
            l *= alpha;
            for (int d = 0; d < D; ++d)
                acc[d] *= alpha;
            for (int j = c0; j < c1; ++j) {
                double pj = exp(s[j - c0] - m_new);
                l += pj;
                for (int d = 0; d < D; ++d)
                    acc[d] += pj * decode(Vb[(int64_t)j * D + d], dtype);
            }
            m = m_new;
        }
        for (int d = 0; d < D; ++d)
            acc[d] /= l;
        free(s);
        free(qd);
    }
}
