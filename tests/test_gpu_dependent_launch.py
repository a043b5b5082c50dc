"""Kernels that follow one another on one stream with no host sync between them.

The stream-K attend kernel is launched with programmatic stream serialization:
it may start while the kernel ahead of it retires, prefetches into L2 from the
lengths it sees then, and waits for that kernel before the pass that counts.
These chains check that the pass that counts still sees what the kernel ahead
wrote: lengths that a commit or rollback kernel just changed (the kernel ahead
is a plain launch), and a query that the previous attend just produced (the
kernel ahead is itself a stream-K attend that lets its successor start early).
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

GAMMA = 4


def i32(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, np.int32)).cuda()


def make_case(paged: bool, seed: int) -> W.Case:
    """GQA decode (4 query rows per KV head: the stream-K route), room for GAMMA + 1 more."""
    if paged:
        return W.paged_case("pdl_paged", 5, 8, 2, 64, "fp16", GAMMA + 1, 40, 3000, 16,
                            seed=seed, pool_seed=seed + 1)
    L = W.rng(seed, "L").integers(40, 3000, size=5, endpoint=True)
    return W.contig_case("pdl_contig", 5, 8, 2, 128, "bf16", 1, L, seed=seed,
                         max_T=int(L.max()) + GAMMA + 2)


def assert_stream_k(run: H.DeviceCase, case: W.Case) -> None:
    """The plan of a one-token step is the persistent stream-K kernel (the one launched
    dependently): no fixed split, a grid of at least one CTA per SM."""
    ns, split_tokens = run.cache.plan(case.H_q, 1, case.max_pages if case.paged else 0)
    assert split_tokens == 0 and ns >= torch.cuda.get_device_properties(0).multi_processor_count


def oracle_step(case: W.Case, kp, vp, L, nk, nv, nq):
    """The oracle's append of one token at L and attention over L + 1 positions."""
    o = oracle.get()
    ko, vo = kp.copy(), vp.copy()
    if case.paged:
        o.append_paged(ko, nk, L, case.block_table)
        o.append_paged(vo, nv, L, case.block_table)
        vis = L + 1
        ko = o.gather_paged(ko, case.block_table, vis, int(vis.max()))
        vo = o.gather_paged(vo, case.block_table, vis, int(vis.max()))
    else:
        o.append_contig(ko, nk, L)
        o.append_contig(vo, nv, L)
    return o.attend(nq, ko, vo, L, case.scale, H.ORACLE_DT[case.dtype])


@pytest.mark.parametrize("paged", [False, True], ids=["contig", "paged"])
@pytest.mark.parametrize("op", ["commit", "rollback"])
def test_length_kernel_then_attend(op, paged):
    case = make_case(paged, 700 + paged + (op == "rollback") * 10)
    o = oracle.get()
    B, dt = case.B, case.dtype
    L0 = case.seq_lens.astype(np.int32)
    g = W.rng(case.seed, "delta")
    if op == "commit":
        delta = g.integers(1, GAMMA + 1, size=B).astype(np.int32)
        L1, bad = o.commit(L0, delta, GAMMA, case.max_T)
    else:
        delta = g.integers(1, 30, size=B).astype(np.int32)
        L1, bad = o.rollback(L0, delta)
    assert bad == 0 and not np.array_equal(L1, L0)
    nk = W.normal_bits((B, case.H_kv, 1, case.D), dt, case.seed + 2, "nk")
    nv = W.normal_bits((B, case.H_kv, 1, case.D), dt, case.seed + 2, "nv")
    nq = W.normal_bits((B, case.H_q, 1, case.D), dt, case.seed + 2, "nq")
    kp, vp = case.k_pool(0), case.v_pool(0)
    run = H.DeviceCase(case)
    try:
        run.load_pools(0, kp, vp)
        assert_stream_k(run, case)
        d_delta = i32(delta)
        k_d, v_d, q_d = (H.to_device(a, dt) for a in (nk, nv, nq))
        out = torch.empty_like(q_d)
        torch.cuda.synchronize()
        # the chain: a kernel that changes the lengths, then the attend that reads them
        if op == "commit":
            run.cache.commit(run.seq_lens, d_delta, GAMMA)
        else:
            run.cache.rollback(run.seq_lens, d_delta)
        run.cache.append_attend(0, k_d, v_d, q_d, run.seq_lens, run.block_table,
                                scale=case.scale, out=out)
        torch.cuda.synchronize()
        assert run.cache.get_error() == kvc.KVC_OK
        assert np.array_equal(run.seq_lens.cpu().numpy(), L1)
        got = H.out_to_f64(out)
    finally:
        run.close()
    H.compare(got, oracle_step(case, kp, vp, L1, nk, nv, nq), f"{op} then attend")


@pytest.mark.parametrize("paged", [False, True], ids=["contig", "paged"])
def test_attend_chain_reads_the_previous_output(paged):
    """q of each attend is the output of the one before; the first output buffer starts
    as NaN, so a read ahead of the previous kernel's writes would show."""
    case = make_case(paged, 720 + paged)
    if not paged:  # long rows: every segment splits into pieces that share the workspace
        L = W.rng(case.seed, "long").integers(6000, 9000, size=case.B, endpoint=True)
        case = W.contig_case("pdl_chain", case.B, case.H_q, case.H_kv, case.D, case.dtype, 1,
                             L, seed=case.seed)
    q = W.normal_bits((case.B, case.H_q, 1, case.D), case.dtype, case.seed + 3, "q")
    kp, vp = case.k_pool(0), case.v_pool(0)
    links = 3
    run = H.DeviceCase(case)
    try:
        run.load_pools(0, kp, vp)
        assert_stream_k(run, case)
        q_d = H.to_device(q, case.dtype)
        outs = [torch.full_like(q_d, float("nan")) for _ in range(links)]
        torch.cuda.synchronize()
        src = q_d
        for out in outs:  # no sync between the links
            run.cache.attend(0, src, run.seq_lens, run.block_table, scale=case.scale, out=out)
            src = out
        torch.cuda.synchronize()
        assert run.cache.get_error() == kvc.KVC_OK
        # each link again, alone, from the settled input of the chain
        for i in range(1, links):
            again = torch.empty_like(q_d)
            run.cache.attend(0, outs[i - 1], run.seq_lens, run.block_table, scale=case.scale,
                             out=again)
            torch.cuda.synchronize()
            assert not torch.isnan(outs[i]).any()
            assert torch.equal(outs[i].view(torch.int16), again.view(torch.int16)), i
        first = H.out_to_f64(outs[0])
    finally:
        run.close()
    o = oracle.get()
    L = case.seq_lens.astype(np.int32)
    if paged:
        vis = L + 1
        K = o.gather_paged(kp, case.block_table, vis, int(vis.max()))
        V = o.gather_paged(vp, case.block_table, vis, int(vis.max()))
    else:
        K, V = kp, vp
    H.compare(first, o.attend(q, K, V, L, case.scale, H.ORACLE_DT[case.dtype]), "first link")


REPLAN = {
    # 4 rows per KV head, contiguous bf16 D 128
    "gqa_contig": lambda: W.contig_case("rp1", 5, 32, 8, 128, "bf16", 1,
                                        [4000, 63, 0, 1300, 64], seed=801, max_T=4100),
    # 2 rows per KV head, paged fp16 D 64, pages of 16 (one box a page) and a verify chunk
    "paged_d64_t2": lambda: W.paged_case("rp2", 4, 8, 8, 64, "fp16", 2, 0, 1500, 16,
                                         seed=802, pool_seed=803),
    # MHA decode, one row per KV head
    "mha_d64": lambda: W.contig_case("rp3", 4, 12, 12, 64, "fp16", 1, [2047, 1, 900, 4095],
                                     seed=804, max_T=4100),
    # tcgen05 stream-K (17+ rows): MQA verify (then the combine launch), and paged GQA
    # verify with 64 rows per KV head
    "mqa_tc_t4": lambda: W.contig_case("rp4", 4, 32, 1, 128, "bf16", 4, [4000, 2100, 0, 2500],
                                       seed=805, max_T=4100),
    "gqa_tc_paged_t8": lambda: W.paged_case("rp5", 3, 16, 2, 128, "bf16", 8, 1500, 3000, 16,
                                            seed=806, pool_seed=807),
}


@pytest.mark.parametrize("kind", sorted(REPLAN))
def test_replan_after_the_wait_gives_identical_results(kind):
    """kvc_inject_replan makes the stream-K kernel treat the plan it made before its
    dependency wait as stale: on mma.sync the copies it issued from that plan are
    drained, the pipeline barriers reset and the range planned again; on tcgen05 (which
    issues nothing before the check) the range is planned again.  Outputs (attend, and
    the fused append + attend with the cache it writes) are bit-identical to the ordinary
    path's."""
    case = REPLAN[kind]()
    run = H.DeviceCase(case)
    try:
        run.load_pools(0, case.k_pool(0), case.v_pool(0))
        assert_stream_k(run, case)
        dt = case.dtype
        q_d = H.to_device(case.q(0), dt)
        k_d, v_d = H.to_device(case.k_new(0), dt), H.to_device(case.v_new(0), dt)
        outs, pools = [], []
        for replan in (False, True, False):
            if replan:
                run.cache.inject_replan()
            out = run.cache.append_attend(0, k_d, v_d, q_d, run.seq_lens, run.block_table,
                                          scale=case.scale)
            torch.cuda.synchronize()
            assert run.cache.get_error() == kvc.KVC_OK
            outs.append(out)
            pools.append(run.pools(0))
        for replan in (True, False):
            if replan:
                run.cache.inject_replan()
            outs.append(run.cache.attend(0, q_d, run.seq_lens, run.block_table,
                                         scale=case.scale))
            torch.cuda.synchronize()
            assert run.cache.get_error() == kvc.KVC_OK
        for o in outs[1:]:
            assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
        for kp, vp in pools[1:]:
            assert np.array_equal(kp, pools[0][0]) and np.array_equal(vp, pools[0][1])
        kref, vref = H.oracle_pools_after_append(case)
        sel, ref = H.oracle_attend(case, kref, vref, case.q(0))
        H.compare(H.out_to_f64(outs[1])[sel], ref, f"{kind} after a replan")
    finally:
        run.close()
