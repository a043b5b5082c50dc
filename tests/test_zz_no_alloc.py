"""kvc_attend_noalloc against kvc_attend and against the oracle, through the C ABI (GPU).

kvc_attend_noalloc serves callers that cannot let the library allocate device
memory: a decode step recorded inside CUDA stream capture (cudaMalloc cannot be
captured), an engine whose caching allocator owns the device's memory (a side
allocation can fail or fragment its pool), a latency-bound loop that cannot take
the synchronisation a free implies.  It runs the same plan and the same kernels as
kvc_attend with its split-K scratch in a fixed 16 MiB device array of the library.

Here every kernel family an unwindowed attend can take -- persistent stream-K on
mma.sync (bf16/fp16 and E4M3 stages) and on tcgen05, the CUDA-core kernel and the
fixed-split FP8 kernel (the fixed-split mma.sync and tcgen05 kernels serve only
windowed calls) -- is called twice in a row
through the new entry point.  Each case first checks that the plan takes
the intended kernel with more than one slice (so the scratch is really used).  The
two outputs must be byte-identical to kvc_attend's (same plan, same kernels,
deterministic merge order), and within the parity tolerance of the fp64 oracle.  The
caching allocator's counters and the device's free memory must not move across the
calls.  A plan that needs more than the fixed scratch is rejected before anything
launches.

This file is collected last and needs nothing from the other test files, so it runs
the same alone in a fresh process or after the whole suite.
"""
from __future__ import annotations

import gc

import numpy as np
import pytest
import torch

import kv_cache_decode_03_b200 as kvc
import oracle
import workloads as W
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _call(fn, cache, case, q, seq, bt, out):
    fn(cache.handle, 0, q.data_ptr(), case.H_q, case.T_new,
       0 if bt is None else bt.data_ptr(), case.max_pages if case.paged else 0,
       seq.data_ptr(), case.scale, out.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _device_memory():
    torch.cuda.synchronize()
    return (torch.cuda.memory_allocated(), torch.cuda.memory_reserved(),
            torch.cuda.mem_get_info()[0])


# (case, kv_format, route): route is checked against kvc_plan_splits
CASES = {
    # persistent stream-K: 4 query rows per KV head, paged, shared prefix pages
    "streamk_paged_gqa": (lambda: W.paged_case("na_sk", 8, 32, 8, 128, "bf16", 1, 300, 5000,
                                               16, seed=91, pool_seed=92, share_frac=0.25,
                                               share_tokens=256), "native", "streamk"),
    # persistent stream-K on tcgen05 with a quarter of the 128-row block used: 32 rows per
    # KV head (a GQA verify chunk), paged
    "streamk_tcgen05_gqa": (lambda: W.paged_case("na_gqa", 4, 16, 2, 128, "bf16", 4, 1000,
                                                 4000, 16, seed=93, pool_seed=94), "native",
                            "streamk"),
    # persistent stream-K on tcgen05: MQA verify, 128 rows per KV head, about 2K tokens
    "streamk_tcgen05_mqa": (lambda: W.contig_case("na_tc", 2, 32, 1, 128, "bf16", 4, 2100,
                                                  seed=97), "native", "streamk"),
    # CUDA-core kernel (D = 32 has no tensor maps), several slices per head
    "splitk_simt_d32": (lambda: W.contig_case("na_simt", 2, 16, 16, 32, "fp16", 1, 6000,
                                              seed=95), "native", "split"),
    # FP8 cache, 4 rows per KV head: the stream-K kernel with E4M3 stages
    "streamk_fp8_gqa": (lambda: W.contig_case("na_fp8sk", 4, 16, 4, 128, "bf16", 1, 3000,
                                              seed=98), "fp8", "streamk"),
    # FP8 cache, 12 rows per KV head: the fixed-split FP8 kernel
    "splitk_fp8_gqa": (lambda: W.contig_case("na_fp8", 4, 16, 4, 128, "bf16", 3, 3000,
                                             seed=96), "fp8", "split"),
}


def _load(case: W.Case, kv_format: str):
    """A one-layer cache holding the case's history (FP8: the oracle's quantisation of it),
    and the oracle's fp64 attention for the case after its append."""
    o = oracle.get()
    cache = kvc.KVCache(case.B, case.H_kv, case.D, case.max_T, case.dtype, case.page_size, 1,
                        case.num_pages, kv_format=kv_format)
    seq = torch.from_numpy(case.seq_lens.astype(np.int32)).cuda()
    bt = torch.from_numpy(case.block_table).cuda() if case.paged else None
    kp, vp = case.k_pool(0), case.v_pool(0)
    if kv_format == "native":
        for which, arr in (("k", kp), ("v", vp)):
            view = cache.pool(0, which)
            view.view(torch.int16).copy_(torch.from_numpy(arr.view(np.int16)).reshape(view.shape))
        cache.append(0, H.to_device(case.k_new(0), case.dtype),
                     H.to_device(case.v_new(0), case.dtype), seq, bt)
        kref, vref = H.oracle_pools_after_append(case)
        _, ref = H.oracle_attend(case, kref, vref, case.q(0))
        return cache, seq, bt, ref
    assert not case.paged
    img = {}
    for which, arr in (("k", kp), ("v", vp)):
        codes, scales = o.quantize_fp8(arr)
        pad = cache.scales(0, which).shape[-1] - scales.shape[-1]
        scales = np.concatenate([scales, np.zeros(scales.shape[:-1] + (pad,), np.float32)], -1)
        cache.pool(0, which).copy_(torch.from_numpy(codes))
        cache.scales(0, which).copy_(torch.from_numpy(scales))
        new = case.k_new(0) if which == "k" else case.v_new(0)
        o.append_fp8(codes, scales, new, case.seq_lens)
        img[which] = (codes, scales)
    cache.append(0, H.to_device(case.k_new(0), case.dtype),
                 H.to_device(case.v_new(0), case.dtype), seq, bt)
    T_cap = int(case.seq_lens.max()) + case.T_new
    (kc, ks), (vc, vs) = img["k"], img["v"]
    ref = o.attend_fp8(case.q(0), kc[:, :, :T_cap], ks[:, :, :T_cap], vc[:, :, :T_cap],
                       vs[:, :, :T_cap], case.seq_lens, case.scale)
    return cache, seq, bt, ref


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_attend_twice_in_a_row(name):
    make, kv_format, route = CASES[name]
    case = make()
    cache, seq, bt, ref = _load(case, kv_format)
    try:
        ns, split_tokens = cache.plan(case.H_q, case.T_new, case.max_pages if case.paged else 0)
        if route == "streamk":
            assert split_tokens == 0, "expected the persistent stream-K plan"
        else:
            assert split_tokens > 0 and ns > 1, f"expected a split plan, got {ns} x {split_tokens}"
        q = H.to_device(case.q(0), case.dtype)
        base = torch.empty_like(q)
        _call(kvc.kvc_attend, cache, case, q, seq, bt, base)
        outs = [torch.full_like(q, float("nan")), torch.full_like(q, float("nan"))]
        # no collection inside the window: a tensor of an earlier case freed there would
        # move the counters without any allocation by the calls
        gc.collect()
        gc.disable()
        try:
            before = _device_memory()
            for out in outs:  # two calls in a row share (and reuse) the static scratch
                _call(kvc.kvc_attend_noalloc, cache, case, q, seq, bt, out)
            after = _device_memory()
        finally:
            gc.enable()
        assert cache.get_error() == kvc.KVC_OK
        assert after[:2] == before[:2], "the caching allocator's counters moved"
        # device-wide free memory can also move under other processes: it must not drop
        # by more than a page-granular fluctuation in every one of a few readings
        if after[2] < before[2]:
            assert any(_device_memory()[2] >= before[2] for _ in range(5)), \
                "kvc_attend_noalloc took device memory"
        for k, out in enumerate(outs):
            assert torch.equal(out.view(torch.int16), base.view(torch.int16)), \
                f"{name} call {k}: differs from kvc_attend"
            H.compare(H.out_to_f64(out), ref, f"{name} call {k} vs the oracle")
    finally:
        cache.close()


def test_noalloc_rejects_plans_beyond_its_scratch():
    """MQA verify of 64 requests over 32K-token page tables needs about 39 MB of partial
    slots (two 128-row slots for each of the 296 persistent CTAs): rejected with
    KVC_ERR_SCRATCH on the host, before any launch."""
    B, H_q, T_new, max_pages = 64, 32, 8, 2049
    cache = kvc.KVCache(B, 1, 128, max_pages * 16, "bf16", page_size=16, num_layers=1,
                        num_pages=64)
    try:
        q = torch.zeros((B, H_q, T_new, 128), dtype=torch.bfloat16, device="cuda")
        out = torch.empty_like(q)
        seq = torch.zeros(B, dtype=torch.int32, device="cuda")
        bt = torch.zeros((B, max_pages), dtype=torch.int32, device="cuda")
        with pytest.raises(kvc.KvcError) as e:
            kvc.kvc_attend_noalloc(cache.handle, 0, q.data_ptr(), H_q, T_new, bt.data_ptr(),
                                   max_pages, seq.data_ptr(), 0.088, out.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
        assert e.value.status == kvc.KVC_ERR_SCRATCH
        assert cache.get_error() == kvc.KVC_OK
    finally:
        cache.close()
