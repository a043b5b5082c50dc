"""CUDA path (through the C ABI) against the fp64 oracle, on identical seeded inputs.

Bars: cache contents bit-exact after every append (the whole pool is compared,
so slots the append must not touch are checked too); attention output within
|gpu - oracle| <= 2e-3 + 1e-2 |oracle| per element (fp32 accumulation,
bf16/fp16 output), with max_abs_err reported.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import kv_cache_decode_03_b200 as kvc
import workloads as W
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU, skipped there
    pytest.skip("needs a CUDA device", allow_module_level=True)


def run_case(case: W.Case, layer: int = 0, requests=None, check_pools: bool = True,
             nthreads: int = 0, twice: bool = False, fused: bool = False):
    """Append + attend on the GPU (two calls, or kvc_append_attend when fused); compare
    pools bit-exactly and outputs within tolerance."""
    g = H.DeviceCase(case, layers=layer + 1)
    try:
        kp0, vp0 = case.k_pool(layer), case.v_pool(layer)
        g.load_pools(layer, kp0, vp0)
        q = case.q(layer)
        if fused:
            out = g.cache.append_attend(layer, H.to_device(case.k_new(layer), case.dtype),
                                        H.to_device(case.v_new(layer), case.dtype),
                                        H.to_device(q, case.dtype), g.seq_lens, g.block_table,
                                        scale=case.scale)
        else:
            g.append(layer, case.k_new(layer), case.v_new(layer))
            out = g.attend(layer, q)
        if twice:
            out2 = g.attend(layer, q)
            torch.cuda.synchronize()
            assert torch.equal(out.view(torch.int16), out2.view(torch.int16)), "nondeterministic"
        assert g.cache.get_error() == kvc.KVC_OK
        kref, vref = H.oracle_pools_after_append(case, layer, kp0, vp0)
        if check_pools:
            kg, vg = g.pools(layer)
            assert np.array_equal(kg, kref), "K pool differs from the oracle's image"
            assert np.array_equal(vg, vref), "V pool differs from the oracle's image"
        sel, ref = H.oracle_attend(case, kref, vref, q, requests, nthreads)
        got = H.out_to_f64(out)[sel]
        return H.compare(got, ref, case.name)
    finally:
        g.close()


# ---------------------------------------------------------------------------
# small grid: every head dim, dtype, layout and row grouping; ragged lengths
# that span several tiles and slices
# ---------------------------------------------------------------------------

HEADS = [(4, 4, 1), (8, 2, 1), (8, 1, 3), (6, 2, 2), (3, 3, 5), (8, 8, 4)]


@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("heads", HEADS, ids=lambda h: f"hq{h[0]}_hkv{h[1]}_t{h[2]}")
def test_small_grid(D, dtype, paged, heads):
    H_q, H_kv, T_new = heads
    seed = 1000 + D + 7 * H_q + 13 * T_new + (1 if dtype == "bf16" else 0)
    if paged:
        case = W.paged_case("grid", 3, H_q, H_kv, D, dtype, T_new, 0, 700, 16, seed=seed,
                            pool_seed=seed + 1)
    else:
        L = W.rng(seed, "L").integers(0, 700, size=3, endpoint=True)
        case = W.contig_case("grid", 3, H_q, H_kv, D, dtype, T_new, L, seed=seed,
                             max_T=int(L.max()) + T_new + 5)
    run_case(case)


@pytest.mark.parametrize("P", [1, 8, 64, 256])
def test_page_sizes(P):
    case = W.paged_case(f"pages{P}", 4, 8, 2, 64, "bf16", 2, 0, 900, P, seed=50 + P,
                        pool_seed=60 + P, share_frac=0.5, share_tokens=4 * P)
    run_case(case)


# ---------------------------------------------------------------------------
# 17 or more query rows per KV head (the 128-row tcgen05 blocks): MQA decode,
# verify chunks, prefill chunks; row counts that leave a ragged last block and
# blocks that cut one head's chunk in two.  At these lengths the partial pieces of a
# segment are merged by the combine launch in 4-row chunks; 18 rows (4 x 4 + 2) and a
# last block of 7 rows (135 = 128 + 4 + 3) leave a short chunk.
# ---------------------------------------------------------------------------

TC_HEADS = [(64, 1, 1), (16, 2, 8), (8, 1, 25), (32, 1, 9), (12, 12, 128), (6, 1, 3),
            (3, 1, 45)]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("heads", TC_HEADS, ids=lambda h: f"hq{h[0]}_hkv{h[1]}_t{h[2]}")
def test_many_rows_grid(D, dtype, paged, heads):
    H_q, H_kv, T_new = heads
    seed = 3000 + D + 7 * H_q + 13 * T_new + (1 if dtype == "bf16" else 0)
    if paged:
        case = W.paged_case("rows", 3, H_q, H_kv, D, dtype, T_new, 0, 700, 16, seed=seed,
                            pool_seed=seed + 1)
    else:
        L = W.rng(seed, "L").integers(0, 700, size=3, endpoint=True)
        L[0] = 0
        case = W.contig_case("rows", 3, H_q, H_kv, D, dtype, T_new, L, seed=seed,
                             max_T=int(L.max()) + T_new + 5)
    run_case(case)


@pytest.mark.parametrize("P", [8, 64, 256])
def test_many_rows_page_sizes(P):
    case = W.paged_case(f"rows_pages{P}", 3, 32, 1, 128, "bf16", 4, 0, 900, P, seed=70 + P,
                        pool_seed=80 + P, share_frac=0.5, share_tokens=4 * P)
    run_case(case)


def test_many_rows_long_context_many_slices():
    """One request, one KV head, 100K positions: about a hundred slices of one row block,
    merged by one CTA."""
    case = W.contig_case("rows_long", 1, 64, 1, 128, "bf16", 2, [100000], seed=90,
                         max_T=100002)
    run_case(case)


def test_many_rows_deterministic():
    case = W.paged_case("rows_det", 2, 32, 1, 128, "bf16", 8, 500, 5000, 16, seed=91,
                        pool_seed=92)
    run_case(case, twice=True)


# ---------------------------------------------------------------------------
# edge cases
# ---------------------------------------------------------------------------

def test_empty_past_single_position():
    case = W.contig_case("empty", 2, 4, 2, 128, "bf16", 1, 0, seed=5, max_T=1)
    run_case(case)


def test_empty_past_chunk():
    case = W.contig_case("empty_chunk", 2, 8, 2, 64, "fp16", 7, [0, 3], seed=6, max_T=16)
    run_case(case)


def test_full_capacity():
    """Append fills the very last slot of the capacity."""
    case = W.contig_case("full", 2, 8, 8, 64, "bf16", 3, [997, 1], seed=7, max_T=1000)
    run_case(case)


def test_long_context_many_splits():
    case = W.paged_case("long", 2, 16, 2, 128, "bf16", 4, 20000, 40000, 16, seed=8,
                        pool_seed=9)
    run_case(case)


def test_mqa_wide_group():
    case = W.paged_case("mqa", 2, 32, 1, 128, "bf16", 8, 100, 3000, 16, seed=10, pool_seed=11)
    run_case(case)


def test_deterministic():
    case = W.paged_case("det", 4, 32, 8, 128, "bf16", 1, 500, 5000, 16, seed=12, pool_seed=13)
    run_case(case, twice=True)


# ---------------------------------------------------------------------------
# the named workloads
# ---------------------------------------------------------------------------

def test_mha_b1_h16_d32_decode():
    run_case(W.mha_small(512), twice=True)


def test_mha_b1_token_by_token_matches_full_causal():
    """64 appends of one token into an empty cache, each followed by a decode attend,
    equal the rows of one full causal attention over the 64 tokens."""
    import oracle
    base = W.mha_small(512)
    T = 64
    case = W.contig_case("tbt", 1, 16, 16, 32, "fp16", 1, 0, seed=base.seed, max_T=T)
    K = W.normal_bits((1, 16, T, 32), "fp16", case.seed, "tbt_k")
    V = W.normal_bits((1, 16, T, 32), "fp16", case.seed, "tbt_v")
    Q = W.normal_bits((1, 16, T, 32), "fp16", case.seed, "tbt_q")
    g = H.DeviceCase(case)
    try:
        rows = []
        for t in range(T):
            sl = torch.full((1,), t, dtype=torch.int32, device="cuda")
            g.append(0, np.ascontiguousarray(K[:, :, t:t + 1]),
                     np.ascontiguousarray(V[:, :, t:t + 1]), seq_lens=sl)
            rows.append(H.out_to_f64(g.attend(0, np.ascontiguousarray(Q[:, :, t:t + 1]),
                                              seq_lens=sl)))
        assert g.cache.get_error() == kvc.KVC_OK
        kg, vg = g.pools(0)
        assert np.array_equal(kg, K) and np.array_equal(vg, V)
    finally:
        g.close()
    full = oracle.get().attend(Q, K, V, np.zeros(1, np.int32), case.scale, oracle.FP16)
    H.compare(np.concatenate(rows, axis=2), full, "token-by-token")


@pytest.mark.parametrize("T_past", W.MHA_SWEEP_T)
def test_mha_b4_h12_d64_decode(T_past):
    run_case(W.mha_sweep(T_past))


@pytest.mark.parametrize("chunk", W.PREFILL_CHUNKS)
@pytest.mark.parametrize("T", W.MHA_SWEEP_T)
def test_mha_b4_h12_d64_chunked_prefill(T, chunk):
    """Build the cache chunk by chunk (append + causal attend of each chunk); every
    emitted row equals full causal attention (all rows up to 1024 tokens, sampled
    rows beyond)."""
    import oracle
    B, Hh, D = 4, 12, 64
    case = W.contig_case("prefill", B, Hh, Hh, D, "fp16", 1, 0, seed=2, max_T=T)
    K = W.normal_bits((B, Hh, T, D), "fp16", 2, "prefill_k", T)
    V = W.normal_bits((B, Hh, T, D), "fp16", 2, "prefill_v", T)
    Q = W.normal_bits((B, Hh, T, D), "fp16", 2, "prefill_q", T)
    g = H.DeviceCase(case)
    out = np.empty((B, Hh, T, D))
    try:
        for s0 in range(0, T, chunk):
            n = min(chunk, T - s0)
            sl = torch.full((B,), s0, dtype=torch.int32, device="cuda")
            g.append(0, np.ascontiguousarray(K[:, :, s0:s0 + n]),
                     np.ascontiguousarray(V[:, :, s0:s0 + n]), seq_lens=sl)
            o = g.cache.attend(0, H.to_device(np.ascontiguousarray(Q[:, :, s0:s0 + n]), "fp16"),
                               sl, scale=case.scale)
            out[:, :, s0:s0 + n] = H.out_to_f64(o)
        assert g.cache.get_error() == kvc.KVC_OK
        kg, vg = g.pools(0)
        assert np.array_equal(kg, K) and np.array_equal(vg, V)
    finally:
        g.close()
    o = oracle.get()
    if T <= 1024:
        ref = o.attend(Q, K, V, np.zeros(B, np.int32), case.scale, oracle.FP16)
        H.compare(out, ref, f"prefill T={T} chunk={chunk}")
        return
    picks = sorted(set([0, 1, chunk - 1, chunk, T - 1] +
                       list(W.rng(T, chunk, "rows").integers(0, T, size=12))))
    for t in picks:
        ref = o.attend(np.ascontiguousarray(Q[:, :, t:t + 1]), K, V,
                       np.full(B, t, np.int32), case.scale, oracle.FP16)
        H.compare(out[:, :, t:t + 1], ref, f"prefill T={T} chunk={chunk} row={t}")


def test_gqa_b16_l4096_one_layer_full():
    """One layer of the 32-layer GQA decode at full size, every request checked."""
    run_case(W.gqa_32layer(layers=1))


def test_gqa_b16_l4096_one_layer_full_fused():
    """The bench's launch at full size: kvc_append_attend (append fused into the persistent
    kernel, dependent launch), pools bit-exact and every request checked."""
    run_case(W.gqa_32layer(layers=1), fused=True)


@pytest.mark.parametrize("L", [4096, 8192])
def test_mha_b4_h12_d64_fused_full(L):
    """MHA decode at full size through the bench's launch (kvc_append_attend)."""
    run_case(W.mha_sweep(L), fused=True)


def test_gqa_b16_l4096_layer_offsets():
    """Layers are independent pools: layer 3 of a 4-layer cache gives the same check."""
    case = W.gqa_32layer(layers=4)
    run_case(case, layer=3, requests=[0, 7, 15])


def test_paged_gqa_b64_full():
    """Paged GQA decode at full size (64 requests, 16 sharing the prefix pages);
    pools bit-exact, 16 requests (all sharers among them) checked against the oracle."""
    case = W.paged_gqa()
    sh = list(case.shared_requests[:8])
    others = [b for b in range(case.B) if b not in case.shared_requests][:8]
    run_case(case, requests=sorted(sh + others))


def test_paged_gqa_b64_full_fused():
    """Paged GQA decode at full size through the bench's launch (kvc_append_attend)."""
    case = W.paged_gqa()
    sh = list(case.shared_requests[:8])
    others = [b for b in range(case.B) if b not in case.shared_requests][-8:]
    run_case(case, requests=sorted(sh + others), fused=True)


@pytest.mark.parametrize("gamma", [2, 4, 8])
@pytest.mark.parametrize("H_kv", [8, 1])
def test_spec_verify_full(gamma, H_kv):
    """Speculative-verify chunks over 8K-32K paged contexts, causal within the chunk."""
    case = W.spec_verify(gamma, H_kv)
    run_case(case, requests=[0, 13, 31])


# ---------------------------------------------------------------------------
# errors: host-side rejections and device-side bounds flags (no fault, no trap)
# ---------------------------------------------------------------------------

def test_host_rejections():
    c = kvc.KVCache(2, 2, 64, 64, "bf16")
    try:
        q = torch.zeros(2, 3, 1, 64, dtype=torch.bfloat16, device="cuda")  # 3 % 2 != 0
        sl = torch.zeros(2, dtype=torch.int32, device="cuda")
        with pytest.raises(kvc.KvcError) as e:
            c.attend(0, q, sl)
        assert e.value.status == kvc.KVC_ERR_INVALID_ARG
        buf = torch.zeros(2 * 2 * 1 * 64 + 1, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(kvc.KvcError) as e:  # misaligned by 2 bytes
            kvc.kvc_append(c.handle, 0, buf.data_ptr() + 2, buf.data_ptr(), 1, 0, 0,
                           sl.data_ptr(), 0)
        assert e.value.status == kvc.KVC_ERR_INVALID_ARG
        with pytest.raises(kvc.KvcError) as e:
            kvc.kvc_attend(c.handle, 5, q.data_ptr(), 2, 1, 0, 0, sl.data_ptr(), 1.0,
                           q.data_ptr(), 0)
        assert e.value.status == kvc.KVC_ERR_INVALID_ARG
    finally:
        c.close()


def test_device_bounds_flag_on_bad_page_id():
    case = W.paged_case("badpage", 2, 8, 2, 64, "bf16", 1, 40, 60, 16, seed=20, pool_seed=21)
    good = case.block_table.copy()
    bt = case.block_table.copy()
    bt[1, 1] = case.num_pages + 5  # outside the pool
    case.block_table = bt
    g = H.DeviceCase(case)
    try:
        g.load_pools(0)
        g.attend(0, case.q(0))
        assert g.cache.get_error() == kvc.KVC_ERR_BOUNDS
        assert g.cache.get_error() == kvc.KVC_OK  # cleared
        bt[1, 1] = -1
        g.block_table = torch.from_numpy(bt).cuda()
        g.append(0, case.k_new(0), case.v_new(0))
        assert g.cache.get_error() == kvc.KVC_OK  # append never reaches logical page 1
        g.attend(0, case.q(0))
        assert g.cache.get_error() == kvc.KVC_ERR_BOUNDS  # attend does
        # the rejected page left the slice tickets clean: a valid table works again
        g.block_table = torch.from_numpy(good).cuda()
        g.attend(0, case.q(0))
        assert g.cache.get_error() == kvc.KVC_OK
    finally:
        g.close()


def test_device_bounds_flag_on_capacity_overflow():
    case = W.contig_case("overflow", 2, 4, 4, 32, "fp16", 2, [10, 15], seed=22, max_T=16)
    g = H.DeviceCase(case)
    try:
        g.load_pools(0)
        before = g.pools(0)
        g.append(0, case.k_new(0), case.v_new(0))  # request 1 would write slot 16
        assert g.cache.get_error() == kvc.KVC_ERR_BOUNDS
        after = g.pools(0)
        # request 0's rows landed, request 1's overflow row did not, nothing else moved
        kref = before[0].copy()
        kref[0, :, 10:12] = case.k_new(0)[0]
        kref[1, :, 15] = case.k_new(0)[1, :, 0]
        assert np.array_equal(after[0], kref)
        g.attend(0, case.q(0))
        assert g.cache.get_error() == kvc.KVC_ERR_BOUNDS
    finally:
        g.close()


def test_kv_bytes_of_a_cache_follows_the_formula():
    c = kvc.KVCache(1, 32, 128, 4096, "fp16", num_layers=32)
    try:
        assert c.nbytes == 2 * 1024 ** 3
    finally:
        c.close()
    c = kvc.KVCache(1, 8, 128, 4096, "fp16", num_layers=32)
    try:
        assert c.nbytes == 512 * 1024 ** 2
    finally:
        c.close()
    c = kvc.KVCache(16, 8, 128, 4097, "bf16", num_layers=2)
    try:
        assert c.nbytes == kvc.kvc_bytes_formula(2, 8, 128, 4097, 2, 16)
    finally:
        c.close()
    c = kvc.KVCache(4, 8, 128, 8208, "bf16", page_size=16, num_layers=1, num_pages=1000)
    try:
        assert c.nbytes == kvc.kvc_bytes_formula(1, 8, 128, 16 * 1000, 2, 1)
    finally:
        c.close()


def test_alternating_plans_share_one_cache():
    """Decode (persistent stream-K), a 32-row verify chunk (fixed split-K) and decode
    again on the same cache: each kernel's slice tickets must be left clean for the next."""
    import oracle
    base = W.paged_case("alt", 6, 32, 8, 128, "bf16", 8, 300, 6000, 16, seed=31, pool_seed=32)
    g = H.DeviceCase(base)
    try:
        kp, vp = base.k_pool(0), base.v_pool(0)
        g.load_pools(0, kp, vp)
        o = oracle.get()
        vis = base.seq_lens.astype(np.int64) + base.T_new
        K = o.gather_paged(kp, base.block_table, vis, int(vis.max()))
        V = o.gather_paged(vp, base.block_table, vis, int(vis.max()))
        for T_new in (1, 8, 1, 4, 1):
            q = W.normal_bits((base.B, base.H_q, T_new, base.D), "bf16", 31, "alt_q", T_new)
            out = g.cache.attend(0, H.to_device(q, "bf16"), g.seq_lens, g.block_table,
                                 scale=base.scale)
            assert g.cache.get_error() == kvc.KVC_OK
            ref = o.attend(q, K, V, base.seq_lens, base.scale, oracle.BF16)
            H.compare(H.out_to_f64(out), ref, f"T_new={T_new}")
    finally:
        g.close()


FUSED = {
    # stream-K (fused in one launch): decode, contiguous and paged with shared prefixes
    "gqa_contig_decode": lambda: W.contig_case("fz1", 5, 32, 8, 128, "bf16", 1,
                                               [4095, 64, 127, 0, 3000], seed=41, max_T=4100),
    "gqa_paged_shared": lambda: W.paged_case("fz2", 8, 32, 8, 128, "bf16", 1, 100, 3000, 16,
                                             seed=42, pool_seed=43, share_frac=0.25,
                                             share_tokens=512),
    # a verify chunk whose new rows straddle a 64-token tile boundary
    "gqa_verify_straddle": lambda: W.contig_case("fz3", 3, 16, 8, 128, "bf16", 4,
                                                 [62, 125, 1021], seed=44, max_T=1100),
    "d64_fp16_paged": lambda: W.paged_case("fz4", 4, 16, 4, 64, "fp16", 2, 0, 900, 16,
                                           seed=45, pool_seed=46),
    # one and two query rows per KV head (MHA decode, MHA verify) on the same kernel
    "mha_d64_decode": lambda: W.contig_case("fz7", 4, 12, 12, 64, "fp16", 1,
                                            [4095, 0, 63, 1500], seed=50, max_T=4100),
    "mha_d128_paged_t2": lambda: W.paged_case("fz8", 3, 8, 8, 128, "bf16", 2, 0, 1200, 16,
                                              seed=51, pool_seed=52),
    "gqa2_d64_paged": lambda: W.paged_case("fz9", 3, 8, 4, 64, "bf16", 1, 0, 900, 8,
                                           seed=53, pool_seed=54),
    # tcgen05 stream-K (17+ rows): the copy warps store the new rows before loading their
    # tiles; MQA verify (then the combine launch), new rows straddling tile boundaries in
    # two row blocks, 8-token pages, and a prefill chunk whose later positions only the
    # second row block sees
    "mqa_tc_paged": lambda: W.paged_case("fz6", 2, 32, 1, 128, "bf16", 4, 100, 2000, 16,
                                         seed=48, pool_seed=49),
    "mqa_tc_straddle_two_blocks": lambda: W.contig_case("fz10", 3, 32, 1, 128, "bf16", 8,
                                                        [60, 125, 1021], seed=55,
                                                        max_T=1100),
    "gqa_tc_d64_fp16_pages8": lambda: W.paged_case("fz11", 3, 16, 2, 64, "fp16", 8, 0, 900,
                                                   8, seed=56, pool_seed=57),
    "mha_tc_prefill_chunk": lambda: W.contig_case("fz12", 2, 2, 2, 64, "bf16", 200,
                                                  [0, 300], seed=58, max_T=520),
    # other kernels: append then attend, two launches
    "mha_simt_d32": lambda: W.contig_case("fz5", 2, 8, 8, 32, "fp16", 1, [700, 33], seed=47),
}


@pytest.mark.parametrize("name", list(FUSED))
def test_append_attend_fused(name):
    run_case(FUSED[name](), fused=True, twice=False)
