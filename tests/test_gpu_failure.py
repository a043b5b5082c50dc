"""Failure detection on the GPU without a fault: a pipeline wait that runs out.

kvc_inject_stall makes the next attend's producers issue no copies, so the first
mbarrier wait of every CTA can never complete.  With a short wait limit the kernel
must give up within the limit, record KVC_ERR_TIMEOUT in the cache's sticky error
word, release what it holds (the tcgen05 kernel its TMEM) and return; the host reads
the status with kvc_get_error, and the next call on the same cache and context is
correct again.  Nothing here traps, faults or waits without a bound.
"""
from __future__ import annotations

import time

import numpy as np
import pytest
import torch

import kv_cache_decode_03_b200 as kvc
import workloads as W
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU, skipped there
    pytest.skip("needs a CUDA device", allow_module_level=True)

LIMIT_NS = 2_000_000  # 2 ms

CASES = {
    # 4 query rows per KV head: the persistent stream-K kernel
    "streamk": lambda: W.contig_case("stall_streamk", 3, 16, 4, 128, "bf16", 1, 700, seed=91),
    # paged, 2 rows per KV head: stream-K with per-box page lookups
    "streamk_paged": lambda: W.paged_case("stall_paged", 4, 8, 4, 64, "fp16", 1, 100, 900, 16,
                                          seed=92, pool_seed=93),
    # MQA verify chunk, 128 rows per KV head: the tcgen05 kernel
    "tcgen05": lambda: W.contig_case("stall_tc", 2, 32, 1, 128, "bf16", 4, 1500, seed=94),
}


@pytest.mark.parametrize("kind", sorted(CASES))
def test_wait_that_runs_out_reports_timeout(kind):
    case = CASES[kind]()
    ns, split_tokens = None, None
    g = H.DeviceCase(case)
    try:
        mp = case.max_pages if case.paged else 0
        ns, split_tokens = g.cache.plan(case.H_q, case.T_new, mp)
        rows = case.H_q // case.H_kv * case.T_new
        if kind.startswith("streamk"):
            assert split_tokens == 0, "expected the persistent stream-K plan"
        else:
            assert rows >= 64, "expected the tcgen05 plan"
        g.load_pools()
        g.append(0, case.k_new(0), case.v_new(0))
        q = case.q(0)
        assert g.cache.get_error() == kvc.KVC_OK
        g.cache.set_wait_limit(LIMIT_NS)
        g.cache.inject_stall()
        t0 = time.perf_counter()
        g.attend(0, q)
        status = g.cache.get_error()  # synchronises
        elapsed = time.perf_counter() - t0
        assert status == kvc.KVC_ERR_TIMEOUT, kvc.kvc_status_string(status)
        assert elapsed < 2.0, f"the bounded wait took {elapsed:.3f} s"
        assert g.cache.get_error() == kvc.KVC_OK  # the error word was cleared
        # the same cache and context still compute correct results
        g.cache.set_wait_limit(0)
        out = g.attend(0, q)
        assert g.cache.get_error() == kvc.KVC_OK
        kref, vref = H.oracle_pools_after_append(case)
        sel, ref = H.oracle_attend(case, kref, vref, q)
        H.compare(H.out_to_f64(out)[sel], ref, f"{case.name} after a timeout")
    finally:
        g.close()


def test_stall_is_consumed_by_one_call():
    """A stall affects only the next attend: a second call is unaffected."""
    case = CASES["streamk"]()
    g = H.DeviceCase(case)
    try:
        g.load_pools()
        g.append(0, case.k_new(0), case.v_new(0))
        q = case.q(0)
        g.cache.set_wait_limit(LIMIT_NS)
        g.cache.inject_stall()
        g.attend(0, q)
        assert g.cache.get_error() == kvc.KVC_ERR_TIMEOUT
        out = g.attend(0, q)
        assert g.cache.get_error() == kvc.KVC_OK
        kref, vref = H.oracle_pools_after_append(case)
        sel, ref = H.oracle_attend(case, kref, vref, q)
        H.compare(H.out_to_f64(out)[sel], ref, case.name)
    finally:
        g.close()


def test_dependent_launch_switch_gives_identical_results():
    """kvc_set_dependent_launch changes how the stream-K kernel is launched, not what it
    computes: outputs are bit-identical with and without programmatic serialization."""
    case = W.contig_case("pdl_switch", 4, 12, 12, 64, "fp16", 1, 3000, seed=95)
    g = H.DeviceCase(case)
    try:
        g.load_pools()
        g.append(0, case.k_new(0), case.v_new(0))
        q = case.q(0)
        outs = []
        for on in (True, False, True):
            g.cache.set_dependent_launch(on)
            outs.append(g.attend(0, q))
        assert g.cache.get_error() == kvc.KVC_OK
        for o in outs[1:]:
            assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
        kref, vref = H.oracle_pools_after_append(case)
        sel, ref = H.oracle_attend(case, kref, vref, q)
        H.compare(H.out_to_f64(outs[0])[sel], ref, case.name)
    finally:
        g.close()
