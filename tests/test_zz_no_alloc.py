"""kvc_attend_noalloc against kvc_attend, through the C ABI (GPU).

kvc_attend_noalloc serves callers that cannot let the library allocate device
memory: a decode step recorded inside CUDA stream capture, an engine whose
caching allocator owns the device's memory, a latency-bound loop that cannot
take the synchronisation a free implies.  It runs the same kernels as
kvc_attend with its split-K scratch in a fixed 16 MiB device array of the
library.  Here each kernel family (persistent stream-K, fixed split-K on
tensor cores, the CUDA-core kernel) is called twice in a row through the new
entry point and compared with the existing one within the parity tolerance,
device free memory is checked to stay put across those calls, and a plan that
needs more than the fixed scratch is rejected before anything launches.

This file is collected last and needs nothing from the other test files, so
it runs the same alone in a fresh process or after the whole suite.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import kv_cache_decode_03_b200 as kvc
import workloads as W

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

ATOL, RTOL = 2e-3, 1e-2  # the parity tolerance used by every attention test
TDT = {"fp16": torch.float16, "bf16": torch.bfloat16}


def _dev(bits: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(TDT[dtype])


def _setup(case: W.Case):
    cache = kvc.KVCache(case.B, case.H_kv, case.D, case.max_T, case.dtype, case.page_size, 1,
                        case.num_pages)
    for which, arr in (("k", case.k_pool(0)), ("v", case.v_pool(0))):
        view = cache.pool(0, which)
        view.view(torch.int16).copy_(torch.from_numpy(arr.view(np.int16)).reshape(view.shape))
    seq = torch.from_numpy(case.seq_lens.astype(np.int32)).cuda()
    bt = torch.from_numpy(case.block_table).cuda() if case.paged else None
    return cache, seq, bt


def _call(fn, cache, case, q, seq, bt, out):
    fn(cache.handle, 0, q.data_ptr(), case.H_q, case.T_new,
       0 if bt is None else bt.data_ptr(), case.max_pages, seq.data_ptr(), case.scale,
       out.data_ptr(), torch.cuda.current_stream().cuda_stream)


CASES = {
    # persistent stream-K: 4 query rows per KV head, paged, shared prefix pages
    "streamk_paged_gqa": lambda: W.paged_case("na_sk", 8, 32, 8, 128, "bf16", 1, 300, 5000, 16,
                                              seed=91, pool_seed=92, share_frac=0.25,
                                              share_tokens=256),
    # fixed split-K on tensor cores: 32 rows per KV head (an MQA-style verify chunk);
    # contexts up to 4K tokens keep its scratch near 8 MB
    "splitk_mma_verify": lambda: W.paged_case("na_mma", 4, 16, 2, 128, "bf16", 4, 1000, 4000,
                                              16, seed=93, pool_seed=94),
    # CUDA-core kernel with several slices: MHA decode, contiguous fp16
    "splitk_simt_mha": lambda: W.contig_case("na_simt", 4, 12, 12, 64, "fp16", 1, 6000, seed=95,
                                             max_T=8193),
}


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_attend_twice_in_a_row(name):
    case = CASES[name]()
    cache, seq, bt = _setup(case)
    try:
        q = _dev(case.q(0), case.dtype)
        ref = torch.empty_like(q)
        _call(kvc.kvc_attend, cache, case, q, seq, bt, ref)
        outs = [torch.empty_like(q), torch.empty_like(q)]
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        for out in outs:  # two calls in a row share (and reuse) the static scratch
            _call(kvc.kvc_attend_noalloc, cache, case, q, seq, bt, out)
        torch.cuda.synchronize()
        free_after = torch.cuda.mem_get_info()[0]
        assert cache.get_error() == kvc.KVC_OK
        assert free_after == free_before, "kvc_attend_noalloc changed device free memory"
        r = ref.float().cpu().numpy().astype(np.float64)
        for k, out in enumerate(outs):
            o = out.float().cpu().numpy().astype(np.float64)
            assert np.isfinite(o).all()
            err = np.abs(o - r)
            assert np.all(err <= ATOL + RTOL * np.abs(r)), \
                f"{name} call {k}: max_abs_err {err.max():.3e}"
    finally:
        cache.close()


def test_noalloc_rejects_plans_beyond_its_scratch():
    """MQA verify of 64 requests over 32K-token page tables needs 17-25 MB of split-K
    scratch (by occupancy): rejected with KVC_ERR_SCRATCH on the host, before any launch."""
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
