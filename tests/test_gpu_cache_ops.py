"""Commit, rollback and copy-on-write page copies on the GPU, against the oracle.

Bars: lengths and pools bit-exact; attention after a speculative round or a
copy-on-write within the attention tolerance of tests/gpu_harness.py.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import kv_cache_decode_03_b200 as kvc
import oracle
import workloads as W
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU, skipped there
    pytest.skip("needs a CUDA device", allow_module_level=True)


def i32(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, np.int32)).cuda()


def test_commit_and_rollback_match_oracle():
    B, gamma, max_T = 64, 8, 5000
    r = W.rng(1, "commit")
    L = r.integers(0, 4990, size=B).astype(np.int32)
    acc = r.integers(0, gamma + 1, size=B).astype(np.int32)
    acc[:3] = [0, gamma, gamma]
    L[2] = max_T - gamma                      # lands exactly on the capacity
    o = oracle.get()
    c = kvc.KVCache(B, 2, 64, max_T, "bf16")
    try:
        sl = i32(L)
        c.commit(sl, i32(acc), gamma)
        ref, bad = o.commit(L, acc, gamma, max_T)
        assert bad == 0 and c.get_error() == kvc.KVC_OK
        assert np.array_equal(sl.cpu().numpy(), ref)
        drop = np.minimum(r.integers(0, 50, size=B), ref).astype(np.int32)
        c.rollback(sl, i32(drop))
        ref2, bad = o.rollback(ref, drop)
        assert bad == 0 and c.get_error() == kvc.KVC_OK
        assert np.array_equal(sl.cpu().numpy(), ref2)
        # out-of-range counts: those requests keep their lengths, the error is flagged
        bad_acc = acc.copy()
        bad_acc[[5, 9, 11]] = [-1, gamma + 1, 10 ** 6]
        before = sl.cpu().numpy()
        c.commit(sl, i32(bad_acc), gamma)
        ref3, nbad = o.commit(before, bad_acc, gamma, max_T)
        assert nbad >= 3 and c.get_error() == kvc.KVC_ERR_BOUNDS
        assert np.array_equal(sl.cpu().numpy(), ref3)
        bad_drop = np.zeros(B, np.int32)
        bad_drop[[0, 1]] = [-3, int(ref3[1]) + 1]
        before = sl.cpu().numpy()
        c.rollback(sl, i32(bad_drop))
        assert c.get_error() == kvc.KVC_ERR_BOUNDS
        assert np.array_equal(sl.cpu().numpy(), before)
    finally:
        c.close()


def test_copy_pages_bit_exact_all_layers():
    B, H_kv, D, P, layers = 4, 2, 128, 16, 3
    case = W.paged_case("copy", B, 8, H_kv, D, "bf16", 1, 100, 600, P, seed=41, pool_seed=42)
    g = H.DeviceCase(case, layers=layers)
    o = oracle.get()
    try:
        pools = []
        for layer in range(layers):
            kp, vp = case.k_pool(layer), case.v_pool(layer)
            g.load_pools(layer, kp, vp)
            pools.append((kp.copy(), vp.copy()))
        r = W.rng(43, "pairs")
        perm = r.permutation(case.num_pages).astype(np.int32)
        src, dst = perm[:7].copy(), perm[7:14].copy()
        g.cache.copy_pages(i32(src), i32(dst))
        assert g.cache.get_error() == kvc.KVC_OK
        for layer in range(layers):
            for which, img in zip("kv", pools[layer]):
                assert o.copy_pages(img, src, dst) == 0
            kg, vg = g.pools(layer)
            assert np.array_equal(kg, pools[layer][0]) and np.array_equal(vg, pools[layer][1])
        # a pair with an id outside the pool is skipped and flagged; the others copy
        src2 = np.array([perm[20], case.num_pages, perm[21]], np.int32)
        dst2 = np.array([perm[22], perm[23], -1], np.int32)
        g.cache.copy_pages(i32(src2), i32(dst2))
        assert g.cache.get_error() == kvc.KVC_ERR_BOUNDS
        for layer in range(layers):
            for img in pools[layer]:
                assert o.copy_pages(img, src2, dst2) == 2
            kg, vg = g.pools(layer)
            assert np.array_equal(kg, pools[layer][0]) and np.array_equal(vg, pools[layer][1])
    finally:
        g.close()


def test_copy_pages_rejects_contiguous_cache():
    c = kvc.KVCache(2, 2, 64, 64, "bf16")
    try:
        with pytest.raises(kvc.KvcError) as e:
            c.copy_pages(i32([0]), i32([1]))
        assert e.value.status == kvc.KVC_ERR_UNSUPPORTED
    finally:
        c.close()


@pytest.mark.parametrize("H_q,H_kv", [(8, 2), (32, 1)], ids=["gqa", "mqa"])
def test_speculative_round_end_to_end(H_q, H_kv):
    """Verify gamma drafts (append + attend), commit the accepted counts on the device,
    decode the next token: both outputs match the oracle, which keeps its own image."""
    B, D, P, gamma, dtype = 6, 128, 16, 4, "bf16"
    # pages for L + gamma + 1 positions, so that a fully accepted chunk still has room
    case = W.paged_case("spec", B, H_q, H_kv, D, dtype, gamma + 1, 30, 900, P, seed=51,
                        pool_seed=52)
    o = oracle.get()
    odt = H.ORACLE_DT[dtype]
    L0 = case.seq_lens.astype(np.int32)
    acc = W.rng(53, "acc").integers(0, gamma + 1, size=B).astype(np.int32)
    acc[:2] = [0, gamma]
    dk = W.normal_bits((B, H_kv, gamma, D), dtype, 54, "dk")
    dv = W.normal_bits((B, H_kv, gamma, D), dtype, 54, "dv")
    dq = W.normal_bits((B, H_q, gamma, D), dtype, 54, "dq")
    nk = W.normal_bits((B, H_kv, 1, D), dtype, 55, "nk")
    nv = W.normal_bits((B, H_kv, 1, D), dtype, 55, "nv")
    nq = W.normal_bits((B, H_q, 1, D), dtype, 55, "nq")
    g = H.DeviceCase(case)
    try:
        kp, vp = case.k_pool(0), case.v_pool(0)
        g.load_pools(0, kp, vp)
        out1 = g.cache.append_attend(0, H.to_device(dk, dtype), H.to_device(dv, dtype),
                                     H.to_device(dq, dtype), g.seq_lens, g.block_table,
                                     scale=case.scale)
        g.cache.commit(g.seq_lens, i32(acc), gamma)
        out2 = g.cache.append_attend(0, H.to_device(nk, dtype), H.to_device(nv, dtype),
                                     H.to_device(nq, dtype), g.seq_lens, g.block_table,
                                     scale=case.scale)
        assert g.cache.get_error() == kvc.KVC_OK
        L1_gpu = g.seq_lens.cpu().numpy()
        kg, vg = g.pools(0)
        got1, got2 = H.out_to_f64(out1), H.out_to_f64(out2)
    finally:
        g.close()
    # oracle: its own pool image through the same steps
    ko, vo = kp.copy(), vp.copy()
    o.append_paged(ko, dk, L0, case.block_table)
    o.append_paged(vo, dv, L0, case.block_table)
    vis = L0 + gamma
    K = o.gather_paged(ko, case.block_table, vis, int(vis.max()))
    V = o.gather_paged(vo, case.block_table, vis, int(vis.max()))
    H.compare(got1, o.attend(dq, K, V, L0, case.scale, odt), "verify chunk")
    L1, bad = o.commit(L0, acc, gamma, case.max_T)
    assert bad == 0 and np.array_equal(L1_gpu, L1)
    o.append_paged(ko, nk, L1, case.block_table)
    o.append_paged(vo, nv, L1, case.block_table)
    assert np.array_equal(kg, ko) and np.array_equal(vg, vo)
    vis = L1 + 1
    K = o.gather_paged(ko, case.block_table, vis, int(vis.max()))
    V = o.gather_paged(vo, case.block_table, vis, int(vis.max()))
    H.compare(got2, o.attend(nq, K, V, L1, case.scale, odt), "decode after commit")


def test_copy_on_write_then_append():
    """Eight requests share 40 prefix tokens (page 2 of 16 tokens is partly filled).
    Every sharer but the first takes a private copy of page 2 (kvc_copy_pages) and
    re-points its table; all append one token at position 40 and attend."""
    B, H_q, H_kv, D, P, prefix, dtype = 8, 8, 2, 64, 16, 40, "fp16"
    n_shared = prefix // P + 1             # pages 0, 1 full; page 2 holds 8 of 16
    num_pages = n_shared + (B - 1) + 4
    bt = np.full((B, 4), -1, np.int32)
    bt[:, :n_shared] = np.arange(n_shared)
    cow_dst = np.arange(n_shared, n_shared + B - 1, dtype=np.int32)
    L = np.full(B, prefix, np.int32)
    case = W.Case(name="cow", B=B, H_q=H_q, H_kv=H_kv, D=D, dtype=dtype, T_new=1, seq_lens=L,
                  seed=61, layers=1, max_T=4 * P, page_size=P, block_table=bt,
                  num_pages=num_pages)
    o = oracle.get()
    odt = H.ORACLE_DT[dtype]
    pool_k = W.normal_bits((num_pages, H_kv, P, D), dtype, 62, "cow_k")
    pool_v = W.normal_bits((num_pages, H_kv, P, D), dtype, 62, "cow_v")
    nk = W.normal_bits((B, H_kv, 1, D), dtype, 63, "nk")
    nv = W.normal_bits((B, H_kv, 1, D), dtype, 63, "nv")
    q = W.normal_bits((B, H_q, 1, D), dtype, 63, "q")
    g = H.DeviceCase(case)
    try:
        g.load_pools(0, pool_k, pool_v)
        src = np.full(B - 1, n_shared - 1, np.int32)
        g.cache.copy_pages(i32(src), i32(cow_dst))
        bt2 = bt.copy()
        bt2[1:, n_shared - 1] = cow_dst
        g.block_table.copy_(torch.from_numpy(bt2))
        out = g.cache.append_attend(0, H.to_device(nk, dtype), H.to_device(nv, dtype),
                                    H.to_device(q, dtype), g.seq_lens, g.block_table,
                                    scale=case.scale)
        assert g.cache.get_error() == kvc.KVC_OK
        kg, vg = g.pools(0)
        got = H.out_to_f64(out)
    finally:
        g.close()
    ko, vo = pool_k.copy(), pool_v.copy()
    for img in (ko, vo):
        assert o.copy_pages(img, src, cow_dst) == 0
    o.append_paged(ko, nk, L, bt2)
    o.append_paged(vo, nv, L, bt2)
    assert np.array_equal(kg, ko) and np.array_equal(vg, vo)
    # the shared pages keep the prefix; each request sees the prefix plus its own token
    K = o.gather_paged(ko, bt2, L + 1, prefix + 1)
    V = o.gather_paged(vo, bt2, L + 1, prefix + 1)
    for b in range(B):
        assert np.array_equal(K[b, :, prefix], nk[b, :, 0])
        assert np.array_equal(K[b, :, :prefix], K[0, :, :prefix])
    H.compare(got, o.attend(q, K, V, L, case.scale, odt), "attend after copy-on-write")
