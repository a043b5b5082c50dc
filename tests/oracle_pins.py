"""Checks that pin the oracle to things other than itself.

Each ``check_*`` takes an ``oracle.Oracle`` and raises AssertionError on a
mismatch.  ``tests/test_oracle_pins.py`` runs them against the real oracle;
``tests/test_oracle_mutants.py`` runs them against copies of the oracle with
planted mistakes and requires every mutant to fail at least one of them.

What pins what:

* storage formats -- numpy's float16 conversion and torch's bfloat16 over all
  65536 words; rounding against numpy (fp16) and a brute-force nearest-value
  search over every finite bfloat16 (bf16);
* the KV-bytes formula -- the worked example on the inference chapter
  ("9. 推理：从生成到性能优化", section 9.3), stored in tests/golden/kv_bytes.txt;
* attention -- torch's fp64 ``scaled_dot_product_attention`` (a library
  routine) with an explicit causal-within-chunk mask and its own GQA
  expansion; closed forms (equal keys give the mean of the visible values,
  equal values give that value, one visible position gives V_0, a zero query
  gives the mean, one dominant key gives its value row); a 50-digit
  ``decimal`` evaluation on tiny shapes;
* the pages' invariants -- token-by-token cached decoding equals the last
  rows of full causal attention ("llm-perf-lab" README; inference chapter
  9.3 and 9.10), chunked equals naive for any chunk size ("llm-perf-lab"
  README), GQA equals MHA over repeated K/V heads ("项目 9-16" roadmap,
  project 12), a request's result does not depend on its batch mates
  (inference chapter 9.10: test batch 1 and batch 2);
* the paged layout -- a shuffled pool read through its block table gives the
  same logical rows as the contiguous cache ("9. 推理" section 9.6);
* commit / rollback / page copy ("llm-perf-lab" README: two-phase
  append/commit, speculative decoding keeps the accepted prefix) -- a
  speculative round (append gamma drafts, commit the accepted ones, append the
  next token) attends exactly like plain cached decoding of the accepted
  prefix; commit then rollback of the same counts is the identity; out-of-range
  counts change nothing; copy-on-write of a shared, partly filled page leaves
  every request's logical cache equal to an unshared contiguous cache;
* sliding window with attention sinks ("项目 9-16" roadmap) -- a window longer
  than the context is full attention, a window of one gives the row's own value
  (a sink covering everything gives full attention again), and every row equals
  plain attention over a contiguous cache holding only its visible positions;
* the FP8 (E4M3) cache -- decoding against torch's float8_e4m3fn over all 256
  codes, encoding against torch's round-to-nearest-even below 448 (plus exact
  ties between neighbours and saturation above), row quantisation against the
  format's half-step error bound and its amax -> 448 property, attention
  over the dequantised values against torch's fp64 SDPA (causal and windowed),
  the any-width paged gather against a loop written in the test and against
  the 16-bit gather, and the FP8 append's placement of codes and scales by
  hand (contiguous) and through a shuffled block table (paged).
"""
from __future__ import annotations

import decimal
import math
from pathlib import Path

import numpy as np
import torch

import oracle as oracle_mod
from workloads import normal_bits

GOLDEN = Path(__file__).resolve().parent / "golden"
FP16, BF16 = oracle_mod.FP16, oracle_mod.BF16
DT = {FP16: "fp16", BF16: "bf16"}


# ---------------------------------------------------------------------------
# independent decoders (numpy / torch), used only on the test side
# ---------------------------------------------------------------------------

def np_decode(bits: np.ndarray, dtype: int) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if dtype == FP16:
        return bits.view(np.float16).astype(np.float64)
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(
        torch.float64).numpy()


def fp_bits(x: np.ndarray, dtype: int) -> np.ndarray:
    """Exactly representable test values -> storage words (values must be exact)."""
    x = np.asarray(x, dtype=np.float64)
    if dtype == FP16:
        b = x.astype(np.float16)
        assert np.array_equal(b.astype(np.float64), x), "value not exact in fp16"
        return b.view(np.uint16)
    t = torch.from_numpy(x).to(torch.bfloat16)
    assert np.array_equal(t.to(torch.float64).numpy(), x), "value not exact in bf16"
    return t.view(torch.int16).numpy().view(np.uint16)


def sdpa_reference(q, K, V, seq_lens, scale, dtype):
    """torch fp64 SDPA per request with the causal-within-chunk boolean mask."""
    qd, Kd, Vd = np_decode(q, dtype), np_decode(K, dtype), np_decode(V, dtype)
    B, H_q, T_new, D = q.shape
    H_kv = K.shape[1]
    out = np.empty((B, H_q, T_new, D))
    for b in range(B):
        n = int(seq_lens[b]) + T_new
        qt = torch.from_numpy(qd[b:b + 1])
        kt = torch.from_numpy(np.ascontiguousarray(Kd[b:b + 1, :, :n]))
        vt = torch.from_numpy(np.ascontiguousarray(Vd[b:b + 1, :, :n]))
        j = torch.arange(n)[None, :]
        i = torch.arange(T_new)[:, None]
        mask = j <= int(seq_lens[b]) + i  # True = attend
        o = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, attn_mask=mask, scale=float(scale), enable_gqa=(H_q != H_kv))
        out[b] = o[0].numpy()
    return out


def random_case(B, H_q, H_kv, T_new, D, L, dtype, seed, T_cap=None, std=1.0):
    L = np.broadcast_to(np.asarray(L, dtype=np.int32), (B,)).copy()
    T_cap = T_cap or int(L.max()) + T_new
    q = normal_bits((B, H_q, T_new, D), DT[dtype], seed, "pin_q")
    K = normal_bits((B, H_kv, T_cap, D), DT[dtype], seed, "pin_k", std=std)
    V = normal_bits((B, H_kv, T_cap, D), DT[dtype], seed, "pin_v", std=std)
    return q, K, V, L


def assert_close(a, b, atol, rtol=0.0, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    bad = ~(np.abs(a - b) <= atol + rtol * np.abs(b))
    assert not bad.any(), f"{what}: {bad.sum()} mismatches, max |diff| " \
                          f"{np.nanmax(np.abs(a - b)) if np.isfinite(a).all() else 'nan'}"


# ---------------------------------------------------------------------------
# storage formats
# ---------------------------------------------------------------------------

ALL_WORDS = np.arange(65536, dtype=np.uint32).astype(np.uint16)


def check_decode_fp16_exhaustive(o):
    got = o.decode(ALL_WORDS, FP16)
    ref = np_decode(ALL_WORDS, FP16)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def check_decode_bf16_exhaustive(o):
    got = o.decode(ALL_WORDS, BF16)
    ref = np_decode(ALL_WORDS, BF16)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def _round_probe_values(dtype: int) -> np.ndarray:
    g = np.random.default_rng(1234 + dtype)
    finite = np_decode(ALL_WORDS, dtype)
    finite = np.unique(finite[np.isfinite(finite)])
    mids = (finite[:-1] + finite[1:]) / 2.0               # exact ties
    near = np.concatenate([np.nextafter(mids, np.inf), np.nextafter(mids, -np.inf)])
    rnd = g.standard_normal(20000) * np.exp(g.uniform(-30, 30, 20000))
    big = np.array([65504.0, 65519.9, 65520.0, 1e6, 3.4e38, 3.39e38, 1e300, 0.0, -0.0])
    return np.concatenate([finite, mids, near, rnd, -rnd, big, -big])


def check_round_fp16(o):
    x = _round_probe_values(FP16)
    got = o.round(x, FP16)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)  # numpy: nearest, ties to even
    assert np.array_equal(got, ref), f"{np.sum(got != ref)} fp16 rounding mismatches"


def check_round_bf16_bruteforce(o):
    x = _round_probe_values(BF16)
    x = x[np.abs(x) < 3.0e38]
    got = o.round(x, BF16)
    # brute force: nearest finite bf16 by search over the sorted value table,
    # ties to the even word
    words = ALL_WORDS[np.isfinite(np_decode(ALL_WORDS, BF16))]
    vals = np_decode(words, BF16)
    order = np.lexsort((words, vals))
    vals, words = vals[order], words[order]
    keep = np.concatenate([[True], vals[1:] != vals[:-1]])  # drop -0 duplicate of +0
    vals, words = vals[keep], words[keep]
    hi = np.clip(np.searchsorted(vals, x), 1, len(vals) - 1)
    lo = hi - 1
    dlo, dhi = np.abs(x - vals[lo]), np.abs(vals[hi] - x)
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (words[hi] % 2 == 0))
    ref = np.where(pick_hi, words[hi], words[lo])
    ref_v = np_decode(ref, BF16)
    got_v = np_decode(got, BF16)
    assert np.array_equal(got_v, ref_v), f"{np.sum(got_v != ref_v)} bf16 rounding mismatches"


# ---------------------------------------------------------------------------
# KV bytes
# ---------------------------------------------------------------------------

def golden_kv_bytes():
    rows = []
    for line in (GOLDEN / "kv_bytes.txt").read_text().splitlines():
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append(tuple(int(v) for v in line.split()))
    assert len(rows) == 2
    return rows


def check_kv_bytes_golden(o):
    for layers, heads, dim, T, e, batch, want in golden_kv_bytes():
        assert o.kv_bytes(layers, heads, dim, T, e, batch) == want
    assert o.kv_bytes(32, 32, 128, 4096, 2, 1) == 2 * 1024 ** 3
    # linear in every factor (context x4 -> cache x4, the page's first consequence)
    assert o.kv_bytes(32, 8, 128, 4 * 4096, 2, 1) == 4 * o.kv_bytes(32, 8, 128, 4096, 2, 1)
    assert o.kv_bytes(1, 1, 1, 1, 1, 1) == 2


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

SDPA_SHAPES = [
    # B, H_q, H_kv, T_new, D, L, dtype
    (2, 4, 4, 1, 32, [37, 64], FP16),        # MHA decode
    (2, 8, 2, 1, 64, [100, 3], BF16),        # GQA decode
    (1, 8, 1, 3, 128, [50], BF16),           # MQA verify chunk
    (2, 6, 3, 5, 64, [0, 17], FP16),         # causal chunk from an empty past
    (1, 4, 2, 8, 32, [9], BF16),
]


def check_attend_vs_sdpa(o):
    for idx, (B, H_q, H_kv, T_new, D, L, dtype) in enumerate(SDPA_SHAPES):
        q, K, V, L = random_case(B, H_q, H_kv, T_new, D, L, dtype, seed=100 + idx)
        scale = float(np.float32(1 / math.sqrt(D)))
        got = o.attend(q, K, V, L, scale, dtype, nthreads=2)
        ref = sdpa_reference(q, K, V, L, scale, dtype)
        assert_close(got, ref, atol=1e-12, rtol=1e-12, what=f"sdpa shape {idx}")


def check_closed_forms(o):
    D, T_cap = 8, 24
    g = np.random.default_rng(7)
    vals = (g.integers(-64, 64, size=(1, 2, T_cap, D)) / 16.0)
    qv = (g.integers(-64, 64, size=(1, 4, 3, D)) / 16.0)
    for dtype in (FP16, BF16):
        q, V = fp_bits(qv, dtype), fp_bits(vals, dtype)
        Vd = np_decode(V, dtype)
        L = np.array([11], dtype=np.int32)
        # (i) all keys equal -> uniform weights -> mean of the visible values
        Keq = fp_bits(np.broadcast_to(vals[:, :, :1, :], vals.shape).copy(), dtype)
        out = o.attend(q, Keq, V, L, 0.25, dtype, nthreads=1)
        for h in range(4):
            for i in range(3):
                n = 11 + i + 1
                assert_close(out[0, h, i], Vd[0, h // 2, :n].mean(0), 1e-13,
                             what="equal keys")
        # (ii) all value rows equal c -> out = c exactly (weights sum to one)
        c = vals[:, :, :1, :]
        Vc = fp_bits(np.broadcast_to(c, vals.shape).copy(), dtype)
        Kr = fp_bits(g.integers(-64, 64, size=vals.shape) / 16.0, dtype)
        out = o.attend(q, Kr, Vc, L, 0.5, dtype, nthreads=1)
        for h in range(4):
            assert_close(out[0, h], np.broadcast_to(c[0, h // 2], (3, D)), 1e-13,
                         what="equal values")
        # (iii) empty past, first new row sees only position 0 -> V_0
        out = o.attend(q, Kr, V, np.array([0], np.int32), 0.5, dtype, nthreads=1)
        for h in range(4):
            assert_close(out[0, h, 0], Vd[0, h // 2, 0], 0.0, what="one visible")
        # (iv) zero query -> all scores 0 -> mean of the visible values
        q0 = fp_bits(np.zeros((1, 4, 3, D)), dtype)
        out = o.attend(q0, Kr, V, L, 0.5, dtype, nthreads=1)
        for h in range(4):
            for i in range(3):
                assert_close(out[0, h, i], Vd[0, h // 2, :12 + i].mean(0), 1e-13,
                             what="zero query")
        # (v) one dominant key -> its value row
        qd = np.zeros((1, 4, 3, D))
        qd[..., 0] = 1.0
        Kd = np.zeros(vals.shape)
        Kd[:, :, 5, 0] = 64.0  # score 64*scale*... vs 0 elsewhere
        out = o.attend(fp_bits(qd, dtype), fp_bits(Kd, dtype), V, L, 1.0, dtype,
                       nthreads=1)
        for h in range(4):
            for i in range(3):
                n = 12 + i
                w_other = (n - 1) * math.exp(-64.0)
                assert_close(out[0, h, i], Vd[0, h // 2, 5], 1e-25 + 8 * w_other,
                             what="dominant key")


def check_decimal_bruteforce(o):
    decimal.getcontext().prec = 50
    Dd = decimal.Decimal
    for dtype in (FP16, BF16):
        B, H_q, H_kv, T_new, D = 1, 2, 1, 2, 4
        q, K, V, L = random_case(B, H_q, H_kv, T_new, D, [5], dtype, seed=55 + dtype)
        scale = 0.5
        got = o.attend(q, K, V, L, scale, dtype, nthreads=1)
        qd, Kd, Vd = np_decode(q, dtype), np_decode(K, dtype), np_decode(V, dtype)
        for h in range(H_q):
            for i in range(T_new):
                n = int(L[0]) + i + 1
                s = [Dd(scale) * sum(Dd(float(qd[0, h, i, d])) * Dd(float(Kd[0, 0, j, d]))
                                     for d in range(D)) for j in range(n)]
                w = [x.exp() for x in s]  # no max subtraction: exact arithmetic here
                tot = sum(w)
                for d in range(D):
                    ref = sum(w[j] * Dd(float(Vd[0, 0, j, d])) for j in range(n)) / tot
                    assert abs(got[0, h, i, d] - float(ref)) <= 1e-14 * max(1.0, abs(float(ref)))


# ---------------------------------------------------------------------------
# invariants stated by the pages
# ---------------------------------------------------------------------------

def check_cached_equals_full_causal(o):
    """Token-by-token append + decode equals the rows of one full causal pass."""
    B, H, D, T = 2, 4, 32, 24
    for dtype in (FP16, BF16):
        q, K, V, _ = random_case(B, H, H, T, D, [0, 0], dtype, seed=77 + dtype)
        scale = float(np.float32(1 / math.sqrt(D)))
        full = o.attend(q, K, V, np.zeros(B, np.int32), scale, dtype, nthreads=2)
        # two slack rows: a planted off-by-one writes there instead of past the array
        Kc = np.zeros(K.shape[:2] + (T + 2, D), K.dtype)
        Vc = np.zeros(V.shape[:2] + (T + 2, D), V.dtype)
        for t in range(T):
            L = np.full(B, t, np.int32)
            o.append_contig(Kc, np.ascontiguousarray(K[:, :, t:t + 1]), L)
            o.append_contig(Vc, np.ascontiguousarray(V[:, :, t:t + 1]), L)
            step = o.attend(np.ascontiguousarray(q[:, :, t:t + 1]), Kc, Vc, L, scale, dtype,
                            nthreads=2)
            assert np.array_equal(step[:, :, 0], full[:, :, t]), f"step {t}"
        assert np.array_equal(Kc[:, :, :T], K) and np.array_equal(Vc[:, :, :T], V)
        assert not Kc[:, :, T:].any() and not Vc[:, :, T:].any()


def check_chunked_equals_naive(o):
    B, H_q, H_kv, T_new, D = 2, 4, 2, 4, 64
    for dtype in (FP16, BF16):
        q, K, V, L = random_case(B, H_q, H_kv, T_new, D, [130, 61], dtype, seed=88 + dtype)
        naive = o.attend(q, K, V, L, 0.125, dtype, nthreads=2)
        for chunk in (1, 2, 7, 64, 128, 1000):
            ch = o.attend_chunked(q, K, V, L, 0.125, dtype, chunk, nthreads=2)
            assert_close(ch, naive, 1e-13, 1e-12, what=f"chunk {chunk}")


def check_gqa_equals_expanded_mha(o):
    B, H_q, T_new, D = 2, 8, 2, 32
    for H_kv in (1, 2, 4, 8):
        q, K, V, L = random_case(B, H_q, H_kv, T_new, D, [20, 33], BF16, seed=99 + H_kv)
        g = H_q // H_kv
        Ke = np.ascontiguousarray(np.repeat(K, g, axis=1))
        Ve = np.ascontiguousarray(np.repeat(V, g, axis=1))
        a = o.attend(q, K, V, L, 0.2, BF16, nthreads=2)
        b = o.attend(q, Ke, Ve, L, 0.2, BF16, nthreads=2)
        assert np.array_equal(a, b), f"H_kv={H_kv}"


def check_batch_invariance(o):
    B, H_q, H_kv, T_new, D = 3, 4, 2, 3, 32
    q, K, V, L = random_case(B, H_q, H_kv, T_new, D, [5, 40, 0], FP16, seed=111)
    full = o.attend(q, K, V, L, 0.3, FP16, nthreads=3)
    for b in range(B):
        one = o.attend(np.ascontiguousarray(q[b:b + 1]), np.ascontiguousarray(K[b:b + 1]),
                       np.ascontiguousarray(V[b:b + 1]), L[b:b + 1], 0.3, FP16, nthreads=1)
        assert np.array_equal(one[0], full[b])


def check_paged_equals_contig(o):
    """Appending through a shuffled block table and reading back through it gives the
    same logical rows as the contiguous cache; untouched slots keep their words."""
    B, H_kv, D, P, T_new = 3, 2, 16, 4, 3
    L = np.array([0, 9, 14], np.int32)
    T_cap = 20
    need = -(-(L + T_new) // P)
    max_pages = int(-(-T_cap // P))
    num_pages = int(need.sum()) + 2
    perm = np.random.default_rng(5).permutation(num_pages).astype(np.int32)
    # entries the pages never reach name the spare page past the pool (see pool_mem):
    # a planted mistake that reads them writes into memory the test owns
    bt = np.full((B, max_pages), num_pages, np.int32)
    cur = 0
    for b in range(B):
        bt[b, :need[b]] = perm[cur:cur + need[b]]
        cur += need[b]
    hist = normal_bits((B, H_kv, T_cap, D), "bf16", 3, "hist")
    new = normal_bits((B, H_kv, T_new, D), "bf16", 3, "new")
    # contiguous reference: history then append
    contig = hist.copy()
    o.append_contig(contig, new, L)
    for b in range(B):  # independent check of the contiguous append
        assert np.array_equal(contig[b, :, L[b]:L[b] + T_new], new[b])
        assert np.array_equal(contig[b, :, :L[b]], hist[b, :, :L[b]])
        assert np.array_equal(contig[b, :, L[b] + T_new:], hist[b, :, L[b] + T_new:])
    # paged: place the history rows by hand (page = table[pos // P], slot = pos % P)
    canary = np.uint16(0x7E01)
    # the pool is a view of one page more, so a planted mistake that writes past the
    # pool lands in memory the test owns
    pool_mem = np.full((num_pages + 1, H_kv, P, D), canary, np.uint16)
    pool = pool_mem[:num_pages]
    for b in range(B):
        for pos in range(int(L[b])):
            pool[bt[b, pos // P], :, pos % P] = hist[b, :, pos]
    before = pool.copy()
    o.append_paged(pool, new, L, bt)
    for b in range(B):
        for i in range(T_new):
            pos = int(L[b]) + i
            assert np.array_equal(pool[bt[b, pos // P], :, pos % P], new[b, :, i])
    changed = np.any(pool != before, axis=-1)
    assert changed.sum() == B * H_kv * T_new  # nothing else written
    logical = o.gather_paged(pool, bt, L + T_new, T_cap)
    for b in range(B):
        n = int(L[b]) + T_new
        assert np.array_equal(logical[b, :, :n], contig[b, :, :n])


def check_speculative_round_equals_plain_decode(o):
    """Verify gamma drafts, keep the first a_b, append the next token: the next step's
    output equals cached decoding that only ever appended the accepted tokens."""
    B, H_q, H_kv, D, gamma = 3, 4, 2, 32, 4
    L0 = np.array([5, 0, 11], np.int32)
    acc = np.array([2, 0, 4], np.int32)
    T_cap = int(L0.max()) + gamma + 3   # slack rows: a planted off-by-one stays in bounds
    scale = 0.25
    for dtype in (FP16, BF16):
        dt = DT[dtype]
        hist_k = normal_bits((B, H_kv, T_cap, D), dt, 21, "spec_hk")
        hist_v = normal_bits((B, H_kv, T_cap, D), dt, 21, "spec_hv")
        draft_k = normal_bits((B, H_kv, gamma, D), dt, 21, "spec_dk")
        draft_v = normal_bits((B, H_kv, gamma, D), dt, 21, "spec_dv")
        nxt_k = normal_bits((B, H_kv, 1, D), dt, 21, "spec_nk")
        nxt_v = normal_bits((B, H_kv, 1, D), dt, 21, "spec_nv")
        q = normal_bits((B, H_q, 1, D), dt, 21, "spec_q")
        # speculative: append gamma drafts, commit acc, append the next token
        Ks, Vs = hist_k.copy(), hist_v.copy()
        o.append_contig(Ks, draft_k, L0)
        o.append_contig(Vs, draft_v, L0)
        L1, bad = o.commit(L0, acc, gamma, T_cap)
        assert bad == 0
        o.append_contig(Ks, nxt_k, L1)
        o.append_contig(Vs, nxt_v, L1)
        spec = o.attend(q, Ks, Vs, L1, scale, dtype, nthreads=2)
        # plain: per request, the history, then only the accepted drafts, then the token
        Kp, Vp = hist_k.copy(), hist_v.copy()
        for b in range(B):
            a, l0 = int(acc[b]), int(L0[b])
            Kp[b, :, l0:l0 + a] = draft_k[b, :, :a]
            Vp[b, :, l0:l0 + a] = draft_v[b, :, :a]
            Kp[b, :, l0 + a] = nxt_k[b, :, 0]
            Vp[b, :, l0 + a] = nxt_v[b, :, 0]
        plain = o.attend(q, Kp, Vp, L0 + acc, scale, dtype, nthreads=2)
        assert np.array_equal(spec, plain)


def check_commit_rollback(o):
    L = np.array([0, 7, 100, 3], np.int32)
    a = np.array([3, 0, 2, 1], np.int32)
    L1, bad = o.commit(L, a, 3, 1000)
    assert bad == 0 and np.array_equal(L1 - L, a)
    L2, bad = o.rollback(L1, a)
    assert bad == 0 and np.array_equal(L2, L)
    # out-of-range counts and capacity overflow leave a request as it is
    L3, bad = o.commit(L, np.array([4, -1, 2, 0], np.int32), 3, 101)
    assert bad == 3 and np.array_equal(L3, np.array([0, 7, 100, 3]))
    L4, bad = o.rollback(L, np.array([1, 8, 100, -2], np.int32))
    assert bad == 3 and np.array_equal(L4, np.array([0, 7, 0, 3]))


def check_copy_on_write(o):
    """Two requests share prefix pages, the last one partly filled; request 1 copies
    that page, re-points its table and both append: every request's logical cache
    equals its own unshared contiguous cache, and the skipped pairs change nothing."""
    H_kv, D, P = 2, 8, 4
    prefix = 6                       # pages 0 (full) and 1 (half) shared
    T_cap = prefix + 3               # slack rows: a planted off-by-one stays in bounds
    shared = normal_bits((1, H_kv, prefix, D), "fp16", 31, "cow_prefix")[0]
    new = normal_bits((2, H_kv, 1, D), "fp16", 31, "cow_new")
    num_pages = 5
    pool = np.full((num_pages, H_kv, P, D), np.uint16(0x3C00), np.uint16)
    for pos in range(prefix):
        pool[pos // P, :, pos % P] = shared[:, pos]
    bt = np.array([[0, 1, 4, 4], [0, 1, 4, 4]], np.int32)   # spare columns: a valid page
    before = pool.copy()
    assert o.copy_pages(pool, [1, 9, -1], [3, 2, 4]) == 2      # one valid pair
    assert np.array_equal(pool[3], before[1])
    assert np.array_equal(np.delete(pool, 3, axis=0), np.delete(before, 3, axis=0))
    bt[1, 1] = 3                                               # request 1 owns its copy
    L = np.array([prefix, prefix], np.int32)
    o.append_paged(pool, new, L, bt)
    logical = o.gather_paged(pool, bt, L + 1, T_cap)
    for b in range(2):
        contig = np.zeros((1, H_kv, T_cap, D), np.uint16)
        contig[0, :, :prefix] = shared
        o.append_contig(contig, np.ascontiguousarray(new[b:b + 1]), L[b:b + 1])
        assert np.array_equal(logical[b, :, :prefix + 1], contig[0, :, :prefix + 1]), \
            f"request {b}"


def check_window_special_cases(o):
    B, H_q, H_kv, T_new, D = 2, 4, 2, 3, 32
    for dtype in (FP16, BF16):
        q, K, V, L = random_case(B, H_q, H_kv, T_new, D, [37, 5], dtype, seed=131 + dtype)
        full = o.attend(q, K, V, L, 0.3, dtype, nthreads=2)
        assert np.array_equal(o.attend_window(q, K, V, L, 0.3, dtype, 10 ** 6, 0), full)
        assert np.array_equal(o.attend_window(q, K, V, L, 0.3, dtype, 1, 10 ** 6), full)
        own = o.attend_window(q, K, V, L, 0.3, dtype, 1, 0)
        Vd = o.decode(V, dtype)
        for b in range(B):
            for h in range(H_q):
                for i in range(T_new):
                    n = int(L[b]) + i + 1
                    assert np.array_equal(own[b, h, i], Vd[b, h // (H_q // H_kv), n - 1])


def check_window_equals_gathered(o):
    """Each row's windowed output equals plain attention over a contiguous cache that
    holds exactly its visible positions (sinks first, then the window), in order."""
    B, H_q, H_kv, T_new, D = 2, 6, 3, 4, 16
    cases = [(8, 0), (8, 3), (3, 5), (20, 2), (1, 1)]
    for dtype in (FP16, BF16):
        q, K, V, L = random_case(B, H_q, H_kv, T_new, D, [30, 9], dtype, seed=141 + dtype)
        g = H_q // H_kv
        for W, S in cases:
            win = o.attend_window(q, K, V, L, 0.25, dtype, W, S, nthreads=2)
            for b in range(B):
                for h in range(H_q):
                    for i in range(T_new):
                        n = int(L[b]) + i + 1
                        keep = [j for j in range(n) if j >= n - W or j < S]
                        Kg = np.ascontiguousarray(K[b:b + 1, h // g:h // g + 1, keep])
                        Vg = np.ascontiguousarray(V[b:b + 1, h // g:h // g + 1, keep])
                        qr = np.ascontiguousarray(q[b:b + 1, h:h + 1, i:i + 1])
                        ref = o.attend(qr, Kg, Vg, np.array([len(keep) - 1], np.int32), 0.25,
                                       dtype, nthreads=1)
                        assert_close(win[b, h, i], ref[0, 0, 0], 1e-15, 1e-13,
                                     what=f"W={W} S={S} b={b} h={h} i={i}")


def bf16_words(x) -> np.ndarray:
    """float64 values rounded to bf16 (torch, nearest even), as storage words."""
    t = torch.from_numpy(np.asarray(x, np.float64)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def check_e4m3_decode_exhaustive(o):
    codes = np.arange(256, dtype=np.uint8)
    got = o.decode_e4m3(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all(), np.nonzero(~same)


def check_e4m3_encode(o):
    finite = o.decode_e4m3(np.arange(0x7F, dtype=np.uint8))          # 0 .. 448
    mids = ((finite[:-1] + finite[1:]) / 2).astype(np.float32)      # exact ties
    r = np.random.default_rng(7)
    probe = np.concatenate([mids, -mids, r.standard_normal(20000).astype(np.float32) * 30,
                            np.float32([0.0, -0.0, 1e-9, 2.0 ** -10, 2.0 ** -9, 447.9,
                                        -447.9])])
    got = o.encode_e4m3(probe)
    ref = torch.from_numpy(probe).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    small = np.abs(probe) < 448
    assert np.array_equal(got[small], ref[small])
    # ties go to the even code
    tie = o.encode_e4m3(mids)
    assert np.all((tie & 1) == 0)
    # saturation and NaN
    big = np.float32([448.0, 460.0, 1e6, -500.0, np.inf])
    assert np.array_equal(o.encode_e4m3(big), np.uint8([0x7E, 0x7E, 0x7E, 0xFE, 0x7E]))
    assert o.encode_e4m3(np.float32([np.nan]))[0] & 0x7F == 0x7F


def check_quantize_fp8(o):
    r = np.random.default_rng(11)
    x = r.standard_normal((64, 128)) * np.exp(r.uniform(-8, 8, size=(64, 1)))
    x[3] = 0.0                                            # an all-zero row
    x[5, :] = 1e-30                                       # below bf16's normal range
    bits = bf16_words(x)
    codes, scales = o.quantize_fp8(bits)
    xd = np_decode(bits, BF16)
    assert scales[3] == 1.0 and not codes[3].any()
    deq = o.decode_e4m3(codes) * scales[:, None].astype(np.float64)
    y = np.abs(xd) / scales[:, None]                     # the row in code units
    half_step = np.where(y >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(y, 1e-300))) - 4),
                         2.0 ** -10)
    assert np.all(np.abs(deq - xd) <= half_step * scales[:, None] * (1 + 1e-6) + 1e-300)
    for i in range(64):
        if scales[i] != 1.0 or codes[i].any():
            j = int(np.argmax(np.abs(xd[i])))
            assert codes[i, j] & 0x7F == 0x7E, i          # amax lands on +-448 ...
            assert abs(deq[i, j] - xd[i, j]) <= 2.0 ** -22 * abs(xd[i, j]), i  # ... exactly


def check_attend_fp8_vs_sdpa(o):
    B, H_q, H_kv, T_new, D = 2, 4, 2, 3, 32
    L = np.array([40, 9], np.int32)
    T_cap = int(L.max()) + T_new
    r = np.random.default_rng(13)
    q = bf16_words(r.standard_normal((B, H_q, T_new, D)))
    Kc = r.integers(0, 256, size=(B, H_kv, T_cap, D)).astype(np.uint8)
    Vc = r.integers(0, 256, size=(B, H_kv, T_cap, D)).astype(np.uint8)
    Kc[(Kc & 0x7F) == 0x7F] = 0x01                       # no NaN codes
    Vc[(Vc & 0x7F) == 0x7F] = 0x02
    Ks = np.float32(r.uniform(1e-3, 2e-2, size=(B, H_kv, T_cap)))
    Vs = np.float32(r.uniform(1e-2, 1.0, size=(B, H_kv, T_cap)))
    to64 = lambda c: torch.from_numpy(c).view(torch.float8_e4m3fn).to(torch.float64)
    K = (to64(Kc) * torch.from_numpy(Ks.astype(np.float64))[..., None])
    V = (to64(Vc) * torch.from_numpy(Vs.astype(np.float64))[..., None])
    qd = torch.from_numpy(np_decode(q, BF16))
    g = H_q // H_kv
    for W, S in ((0, 0), (5, 2), (1, 0)):
        got = o.attend_fp8(q, Kc, Ks, Vc, Vs, L, 0.3, W, S, nthreads=2)
        for b in range(B):
            n = np.arange(T_new)[:, None] + int(L[b]) + 1          # visible counts per row
            j = np.arange(T_cap)[None, :]
            keep = (j < n) & ((W == 0) | (j >= n - W) | (j < S))
            mask = torch.from_numpy(np.where(keep, 0.0, -np.inf))
            ref = torch.nn.functional.scaled_dot_product_attention(
                qd[b:b + 1], K[b:b + 1].repeat_interleave(g, 1), V[b:b + 1].repeat_interleave(g, 1),
                attn_mask=mask, scale=0.3)
            assert_close(got[b], ref[0].numpy(), 1e-13, 1e-11, what=f"W={W} S={S} b={b}")



def _shuffled_table(L, T_new, P, T_cap, seed):
    """A block table over a shuffled pool: request b's first ceil((L_b + T_new) / P)
    entries name distinct pages; every other entry names the spare page num_pages."""
    need = -(-(L + T_new) // P)
    max_pages = int(-(-T_cap // P))
    num_pages = int(need.sum()) + 2
    perm = np.random.default_rng(seed).permutation(num_pages).astype(np.int32)
    bt = np.full((len(L), max_pages), num_pages, np.int32)
    cur = 0
    for b in range(len(L)):
        bt[b, :need[b]] = perm[cur:cur + need[b]]
        cur += need[b]
    return bt, num_pages


def check_gather_rows(o):
    """gather_rows (any row width) reads position pos of (b, g) from slot pos % P of page
    table[b][pos // P]: against a loop written here over 1-byte and 4-byte rows, and
    byte for byte against gather_paged on a 16-bit pool ("9. 推理" section 9.6)."""
    B, H_kv, D, P, T_new, T_cap = 3, 2, 8, 4, 3, 20
    L = np.array([0, 9, 14], np.int32)
    bt, num_pages = _shuffled_table(L, T_new, P, T_cap, 21)
    n = L + T_new
    r = np.random.default_rng(22)
    # spare pages past the pool: a planted mistake that reads past it stays in test memory
    codes_mem = r.integers(0, 256, size=(num_pages + 4, H_kv, P, D)).astype(np.uint8)
    scales_mem = np.float32(r.uniform(-5, 5, size=(num_pages + 4, H_kv, P)))
    words_mem = r.integers(0, 1 << 16, size=(num_pages + 4, H_kv, P, D)).astype(np.uint16)
    for pool_mem in (codes_mem, scales_mem, words_mem):
        pool = pool_mem[:num_pages]
        got = o.gather_rows(pool, bt, n, T_cap)
        ref = np.zeros((B, H_kv, T_cap) + pool.shape[3:], pool.dtype)
        for b in range(B):
            for g in range(H_kv):
                for pos in range(int(n[b])):
                    ref[b, g, pos] = pool[bt[b, pos // P], g, pos % P]
        assert got.dtype == pool.dtype and got.shape == ref.shape
        assert np.array_equal(got.view(np.uint8), ref.view(np.uint8))
    words = words_mem[:num_pages]
    assert np.array_equal(o.gather_rows(words, bt, n, T_cap), o.gather_paged(words, bt, n, T_cap))


def check_append_fp8_placement(o):
    """FP8 append: new row i of (b, g), quantised, lands at position L_b + i -- codes and
    scale together -- in a contiguous cache (checked by hand, with scale rows padded past
    the capacity), and through a shuffled block table the paged pool reads back (with
    gather_rows) exactly as the contiguous cache; nothing else is written."""
    B, H_kv, D, P, T_new, T_cap, T_pad = 3, 2, 16, 4, 3, 20, 64
    L = np.array([0, 9, 14], np.int32)
    r = np.random.default_rng(31)
    x = r.standard_normal((B, H_kv, T_new, D)) * np.exp(r.uniform(-3, 3, (B, H_kv, T_new, 1)))
    new = bf16_words(x)
    qc, qs = o.quantize_fp8(new)
    # history: arbitrary codes and scales at every slot
    hist_c = r.integers(0, 256, size=(B, H_kv, T_cap, D)).astype(np.uint8)
    hist_s = np.float32(r.uniform(1, 2, size=(B, H_kv, T_pad)))
    codes, scales = hist_c.copy(), hist_s.copy()
    o.append_fp8(codes, scales, new, L)
    for b in range(B):
        for i in range(T_new):
            assert np.array_equal(codes[b, :, L[b] + i], qc[b, :, i]), (b, i)
            assert np.array_equal(scales[b, :, L[b] + i], qs[b, :, i]), (b, i)
    assert np.any(codes != hist_c, axis=-1).sum() <= B * H_kv * T_new
    assert (scales != hist_s).sum() == B * H_kv * T_new
    # paged: the same history placed by hand, then the append through the table
    bt, num_pages = _shuffled_table(L, T_new, P, T_cap, 32)
    pc_mem = np.full((num_pages + 4, H_kv, P, D), 0xA5, np.uint8)
    ps_mem = np.full((num_pages + 4, H_kv, P), -7.0, np.float32)
    pc, ps = pc_mem[:num_pages], ps_mem[:num_pages]
    for b in range(B):
        for pos in range(int(L[b])):
            pc[bt[b, pos // P], :, pos % P] = hist_c[b, :, pos]
            ps[bt[b, pos // P], :, pos % P] = hist_s[b, :, pos]
    before_c, before_s = pc_mem.copy(), ps_mem.copy()
    o.append_fp8(pc, ps, new, L, bt)
    n = L + T_new
    got_c = o.gather_rows(pc, bt, n, T_cap)
    got_s = o.gather_rows(ps, bt, n, T_cap)
    for b in range(B):
        assert np.array_equal(got_c[b, :, :n[b]], codes[b, :, :n[b]]), b
        assert np.array_equal(got_s[b, :, :n[b]], scales[b, :, :n[b]]), b
    assert (ps_mem != before_s).sum() == B * H_kv * T_new
    assert np.any(pc_mem != before_c, axis=-1).sum() <= B * H_kv * T_new
    assert np.array_equal(pc_mem[num_pages:], before_c[num_pages:])


ALL_CHECKS = [
    check_decode_fp16_exhaustive,
    check_decode_bf16_exhaustive,
    check_round_fp16,
    check_round_bf16_bruteforce,
    check_kv_bytes_golden,
    check_attend_vs_sdpa,
    check_closed_forms,
    check_decimal_bruteforce,
    check_cached_equals_full_causal,
    check_chunked_equals_naive,
    check_gqa_equals_expanded_mha,
    check_batch_invariance,
    check_paged_equals_contig,
    check_speculative_round_equals_plain_decode,
    check_commit_rollback,
    check_copy_on_write,
    check_window_special_cases,
    check_window_equals_gathered,
    check_e4m3_decode_exhaustive,
    check_e4m3_encode,
    check_quantize_fp8,
    check_gather_rows,
    check_append_fp8_placement,
    check_attend_fp8_vs_sdpa,
]
