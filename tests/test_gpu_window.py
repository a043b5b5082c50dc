"""Sliding-window attention with attention sinks on the GPU, against the oracle.

Every kernel route is covered: CUDA cores (1-2 rows per KV head), mma.sync
(3-63 rows) and tcgen05 (64+ rows); contiguous and paged caches; windows shorter
than a tile, spanning several slices, and longer than the context; sinks that end
inside a tile.  Bar: the attention tolerance of tests/gpu_harness.py.
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


def run_window(case: W.Case, window: int, sink: int, requests=None):
    g = H.DeviceCase(case)
    try:
        kp0, vp0 = case.k_pool(0), case.v_pool(0)
        g.load_pools(0, kp0, vp0)
        q = case.q(0)
        g.append(0, case.k_new(0), case.v_new(0))
        out = g.cache.attend_window(0, H.to_device(q, case.dtype), g.seq_lens, window, sink,
                                    g.block_table, scale=case.scale)
        assert g.cache.get_error() == kvc.KVC_OK
        got = H.out_to_f64(out)
    finally:
        g.close()
    o = oracle.get()
    kref, vref = H.oracle_pools_after_append(case, 0, kp0, vp0)
    sel = np.arange(case.B) if requests is None else np.asarray(requests)
    L = case.seq_lens[sel]
    vis = L.astype(np.int64) + case.T_new
    if case.paged:
        bt = case.block_table[sel]
        K = o.gather_paged(kref, bt, vis, int(vis.max()))
        V = o.gather_paged(vref, bt, vis, int(vis.max()))
    else:
        K, V = np.ascontiguousarray(kref[sel]), np.ascontiguousarray(vref[sel])
    ref = o.attend_window(np.ascontiguousarray(q[sel]), K, V, L, case.scale,
                          H.ORACLE_DT[case.dtype], window, sink)
    return H.compare(got[sel], ref, f"{case.name} W={window} S={sink}")


WINDOWS = [(1, 0), (7, 0), (64, 0), (100, 4), (300, 16), (1000, 1), (100000, 0)]
ROUTES = [  # (H_q, H_kv, T_new, D): rows per KV head -> kernel
    (4, 4, 1, 32),     # 1 row: CUDA cores
    (6, 3, 1, 64),     # 2 rows: CUDA cores
    (8, 2, 1, 128),    # 4 rows: mma.sync (fixed split with a window)
    (8, 2, 4, 128),    # 16 rows: mma.sync
    (16, 2, 4, 64),    # 32 rows: mma.sync
    (32, 1, 4, 128),   # 128 rows: tcgen05
    (16, 1, 5, 64),    # 80 rows: tcgen05, a ragged row block
]


@pytest.mark.parametrize("ws", WINDOWS, ids=lambda w: f"W{w[0]}_S{w[1]}")
@pytest.mark.parametrize("route", ROUTES, ids=lambda r: f"hq{r[0]}_hkv{r[1]}_t{r[2]}_d{r[3]}")
@pytest.mark.parametrize("paged", [False, True])
def test_window_routes(route, ws, paged):
    H_q, H_kv, T_new, D = route
    window, sink = ws
    seed = 5000 + 7 * H_q + 11 * T_new + D
    if paged:
        case = W.paged_case("win", 3, H_q, H_kv, D, "bf16", T_new, 0, 2500, 16, seed=seed,
                            pool_seed=seed + 1)
    else:
        L = W.rng(seed, "L").integers(0, 2500, size=3, endpoint=True)
        L[0] = 3
        case = W.contig_case("win", 3, H_q, H_kv, D, "fp16", T_new, L, seed=seed,
                             max_T=int(L.max()) + T_new + 5)
    run_window(case, window, sink)


@pytest.mark.parametrize("route", [(8, 2, 1, 128), (32, 1, 4, 128), (8, 8, 1, 64)],
                         ids=["mma", "tcgen05", "cudacore"])
def test_window_long_context(route):
    """24K-40K positions, a 512-position window and 4 sinks: the slices of the window
    part start far from the sinks, and a row's earliest slices can hold nothing it sees."""
    H_q, H_kv, T_new, D = route
    case = W.paged_case("win_long", 2, H_q, H_kv, D, "bf16", T_new, 24000, 40000, 16,
                        seed=71, pool_seed=72)
    run_window(case, 512, 4)


def test_window_zero_is_full_attention():
    case = W.paged_case("win0", 2, 8, 2, 128, "bf16", 2, 100, 900, 16, seed=73, pool_seed=74)
    g = H.DeviceCase(case)
    try:
        g.load_pools(0)
        g.append(0, case.k_new(0), case.v_new(0))
        q = H.to_device(case.q(0), case.dtype)
        a = g.cache.attend(0, q, g.seq_lens, g.block_table, scale=case.scale)
        b = g.cache.attend_window(0, q, g.seq_lens, 0, 7, g.block_table, scale=case.scale)
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
        with pytest.raises(kvc.KvcError) as e:
            g.cache.attend_window(0, q, g.seq_lens, -1, 0, g.block_table, scale=case.scale)
        assert e.value.status == kvc.KVC_ERR_INVALID_ARG
        assert g.cache.get_error() == kvc.KVC_OK
    finally:
        g.close()
