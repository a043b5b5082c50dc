"""The FP8 (E4M3) cache on the GPU, against the oracle.

Bars: codes and scales written by the append bit-exact; attention over the cache
within the attention tolerance of tests/gpu_harness.py against the oracle's fp64
attention over code * scale.
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


class Fp8Run:
    """An FP8 cache whose history is the oracle's quantisation of seeded bf16 rows."""

    def __init__(self, case: W.Case, random_history: bool = False):
        self.case = c = case
        self.o = oracle.get()
        self.cache = kvc.KVCache(c.B, c.H_kv, c.D, c.max_T, "bf16", c.page_size, 1,
                                 c.num_pages, kv_format="fp8")
        self.seq_lens = i32(c.seq_lens)
        self.bt = torch.from_numpy(c.block_table).cuda() if c.paged else None
        if random_history:  # any finite codes and positive scales
            g = W.rng(c.seed, "fp8_history")
            shape = c.pool_shape()
            kc, vc = (g.integers(0, 256, size=shape).astype(np.uint8) for _ in range(2))
            for a in (kc, vc):
                a[(a & 0x7F) == 0x7F] = 0x3C
            ks, vs = (np.float32(g.uniform(1e-3, 1e-2, size=shape[:3])) for _ in range(2))
        else:
            kc, ks = self.o.quantize_fp8(c.k_pool(0))
            vc, vs = self.o.quantize_fp8(c.v_pool(0))
        sk = self.cache.scales(0, "k")
        if not c.paged:  # scale rows are padded to whole 64-token tiles
            pad = sk.shape[-1] - ks.shape[-1]
            ks = np.concatenate([ks, np.zeros(ks.shape[:-1] + (pad,), np.float32)], -1)
            vs = np.concatenate([vs, np.zeros(vs.shape[:-1] + (pad,), np.float32)], -1)
        self.img = {"kc": kc, "ks": ks, "vc": vc, "vs": vs}
        self.cache.pool(0, "k").copy_(torch.from_numpy(kc))
        self.cache.pool(0, "v").copy_(torch.from_numpy(vc))
        sk.copy_(torch.from_numpy(ks))
        self.cache.scales(0, "v").copy_(torch.from_numpy(vs))

    def append(self):
        c = self.case
        self.cache.append(0, H.to_device(c.k_new(0), "bf16"), H.to_device(c.v_new(0), "bf16"),
                          self.seq_lens, self.bt)
        bt = c.block_table if c.paged else None
        self.o.append_fp8(self.img["kc"], self.img["ks"], c.k_new(0), c.seq_lens, bt)
        self.o.append_fp8(self.img["vc"], self.img["vs"], c.v_new(0), c.seq_lens, bt)

    def check_pools(self):
        torch.cuda.synchronize()
        got = {"kc": self.cache.pool(0, "k"), "vc": self.cache.pool(0, "v"),
               "ks": self.cache.scales(0, "k"), "vs": self.cache.scales(0, "v")}
        for key, t in got.items():
            a = t.cpu().numpy()
            b = self.img[key]
            assert a.dtype == b.dtype and np.array_equal(a.view(np.uint8), b.view(np.uint8)), key

    def reference(self, q, window=0, sink=0, requests=None):
        c, o = self.case, self.o
        sel = np.arange(c.B) if requests is None else np.asarray(requests)
        L = c.seq_lens[sel]
        vis = L.astype(np.int64) + c.T_new
        T_cap = int(vis.max())
        if c.paged:
            bt = c.block_table[sel]
            parts = [o.gather_rows(self.img[k], bt, vis, T_cap) for k in ("kc", "ks", "vc", "vs")]
        else:
            parts = [self.img[k][sel][:, :, :T_cap] for k in ("kc", "ks", "vc", "vs")]
        return sel, o.attend_fp8(np.ascontiguousarray(q[sel]), *parts, L, c.scale, window, sink)

    def close(self):
        self.cache.close()


def run(case: W.Case, window: int = 0, sink: int = 0, requests=None, check_pools=True):
    r = Fp8Run(case)
    try:
        r.append()
        q = case.q(0)
        qd = H.to_device(q, "bf16")
        if window:
            out = r.cache.attend_window(0, qd, r.seq_lens, window, sink, r.bt, scale=case.scale)
        else:
            out = r.cache.attend(0, qd, r.seq_lens, r.bt, scale=case.scale)
        assert r.cache.get_error() == kvc.KVC_OK
        if check_pools:
            r.check_pools()
        sel, ref = r.reference(q, window, sink, requests)
        return H.compare(H.out_to_f64(out)[sel], ref, f"{case.name} fp8 W={window} S={sink}")
    finally:
        r.close()


ROUTES = [(4, 4, 1), (8, 4, 1), (8, 2, 1), (8, 2, 4), (16, 2, 4), (32, 1, 2), (32, 1, 4),
          (6, 2, 5)]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("heads", ROUTES, ids=lambda h: f"hq{h[0]}_hkv{h[1]}_t{h[2]}")
def test_fp8_append_and_attend(D, paged, heads):
    H_q, H_kv, T_new = heads
    seed = 9000 + D + 7 * H_q + 13 * T_new + paged
    if paged:
        case = W.paged_case("fp8", 3, H_q, H_kv, D, "bf16", T_new, 0, 1500, 16, seed=seed,
                            pool_seed=seed + 1)
    else:
        L = W.rng(seed, "L").integers(0, 1500, size=3, endpoint=True)
        L[0] = 2
        case = W.contig_case("fp8", 3, H_q, H_kv, D, "bf16", T_new, L, seed=seed,
                             max_T=int(L.max()) + T_new + 5)
    run(case)


@pytest.mark.parametrize("ws", [(7, 0), (300, 4), (100000, 0)], ids=lambda w: f"W{w[0]}_S{w[1]}")
@pytest.mark.parametrize("heads", [(8, 2, 1), (32, 1, 4)], ids=["gqa", "mqa_verify"])
def test_fp8_window(heads, ws):
    H_q, H_kv, T_new = heads
    case = W.paged_case("fp8w", 3, H_q, H_kv, 128, "bf16", T_new, 0, 2000, 16, seed=97,
                        pool_seed=98)
    run(case, *ws, check_pools=False)


@pytest.mark.parametrize("P", [8, 64, 256])
def test_fp8_page_sizes(P):
    case = W.paged_case(f"fp8p{P}", 3, 8, 2, 128, "bf16", 2, 0, 900, P, seed=100 + P,
                        pool_seed=110 + P, share_frac=0.5, share_tokens=4 * P)
    run(case)


@pytest.mark.parametrize("paged", [False, True])
def test_fp8_streamk_route_ragged_batch(paged):
    """1-8 rows per KV head take the persistent stream-K kernel with E4M3 stages: many
    requests with very different lengths (so that pieces of a segment land on several
    CTAs and are merged), results within the attention tolerance."""
    if paged:
        case = W.paged_case("fp8sk", 16, 16, 4, 128, "bf16", 1, 0, 7000, 16, seed=141,
                            pool_seed=142)
    else:
        case = W.contig_case("fp8sk", 12, 32, 8, 64, "bf16", 1,
                             [5000, 17, 0, 3100, 64, 63, 1, 4500, 2222, 129, 4999, 700],
                             seed=143)
    r = Fp8Run(case)
    try:
        ns, split_tokens = r.cache.plan(case.H_q, case.T_new, case.max_pages if paged else 0)
        assert split_tokens == 0, "expected the persistent stream-K plan"
        r.append()
        q = case.q(0)
        qd = H.to_device(q, "bf16")
        outs = []
        for on in (True, False):  # with and without programmatic dependent launch
            r.cache.set_dependent_launch(on)
            outs.append(r.cache.attend(0, qd, r.seq_lens, r.bt, scale=case.scale))
        r.cache.set_dependent_launch(True)
        r.cache.inject_replan()  # the first copies drained and the range planned again
        outs.append(r.cache.attend(0, qd, r.seq_lens, r.bt, scale=case.scale))
        assert r.cache.get_error() == kvc.KVC_OK
        for o in outs[1:]:
            assert torch.equal(outs[0].view(torch.int16), o.view(torch.int16))
        sel, ref = r.reference(q)
        H.compare(H.out_to_f64(outs[0])[sel], ref, f"{case.name} fp8 stream-K")
    finally:
        r.close()


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("paged", [False, True])
def test_fp8_append_attend_fused(D, paged):
    """kvc_append_attend on an FP8 cache is one launch of the stream-K kernel, which
    quantises the new rows itself: codes and scales bit-exact with the oracle's append
    (new rows straddling tile boundaries, an empty past), attention within tolerance."""
    if paged:
        case = W.paged_case("fp8fz", 5, 16, 4, D, "bf16", 2, 0, 2000, 16, seed=151,
                            pool_seed=152)
    else:
        case = W.contig_case("fp8fz", 5, 16, 4, D, "bf16", 2, [63, 0, 1999, 640, 127],
                             seed=153, max_T=2100)
    r = Fp8Run(case)
    try:
        mp = case.max_pages if paged else 0
        ns, split_tokens = r.cache.plan(case.H_q, case.T_new, mp)
        assert split_tokens == 0, "expected the persistent stream-K plan"
        q = case.q(0)
        out = r.cache.append_attend(0, H.to_device(case.k_new(0), "bf16"),
                                    H.to_device(case.v_new(0), "bf16"),
                                    H.to_device(q, "bf16"), r.seq_lens, r.bt, scale=case.scale)
        assert r.cache.get_error() == kvc.KVC_OK
        bt = case.block_table if paged else None
        r.o.append_fp8(r.img["kc"], r.img["ks"], case.k_new(0), case.seq_lens, bt)
        r.o.append_fp8(r.img["vc"], r.img["vs"], case.v_new(0), case.seq_lens, bt)
        r.check_pools()
        sel, ref = r.reference(q)
        H.compare(H.out_to_f64(out)[sel], ref, f"{case.name} fp8 fused append + attend")
    finally:
        r.close()


def test_fp8_gqa_b16_l4096_one_layer_full_fused():
    """One layer of the 32-layer GQA decode on an FP8 cache at full size, through the
    bench's launch (kvc_append_attend: the kernel quantises the new rows): codes and
    scales bit-exact, every request's attention within tolerance."""
    case = W.gqa_32layer(layers=1)
    r = Fp8Run(case)
    try:
        q = case.q(0)
        out = r.cache.append_attend(0, H.to_device(case.k_new(0), "bf16"),
                                    H.to_device(case.v_new(0), "bf16"),
                                    H.to_device(q, "bf16"), r.seq_lens, None, scale=case.scale)
        assert r.cache.get_error() == kvc.KVC_OK
        r.o.append_fp8(r.img["kc"], r.img["ks"], case.k_new(0), case.seq_lens, None)
        r.o.append_fp8(r.img["vc"], r.img["vs"], case.v_new(0), case.seq_lens, None)
        r.check_pools()
        sel, ref = r.reference(q)
        H.compare(H.out_to_f64(out)[sel], ref, "fp8 GQA B16 L4096 fused")
    finally:
        r.close()


def test_fp8_streamk_wait_that_runs_out():
    """Failure detection on the FP8 stream-K variant: with the next call's copies withheld
    (kvc_inject_stall) and a 2 ms wait limit, the call returns, KVC_ERR_TIMEOUT is
    reported, and the next call on the same cache is correct."""
    case = W.paged_case("fp8stall", 4, 16, 4, 128, "bf16", 1, 100, 1500, 16, seed=161,
                        pool_seed=162)
    r = Fp8Run(case)
    try:
        ns, split_tokens = r.cache.plan(case.H_q, case.T_new, case.max_pages)
        assert split_tokens == 0, "expected the persistent stream-K plan"
        r.append()
        q = case.q(0)
        qd = H.to_device(q, "bf16")
        r.cache.set_wait_limit(2_000_000)
        r.cache.inject_stall()
        r.cache.attend(0, qd, r.seq_lens, r.bt, scale=case.scale)
        assert r.cache.get_error() == kvc.KVC_ERR_TIMEOUT
        r.cache.set_wait_limit(0)
        out = r.cache.attend(0, qd, r.seq_lens, r.bt, scale=case.scale)
        assert r.cache.get_error() == kvc.KVC_OK
        sel, ref = r.reference(q)
        H.compare(H.out_to_f64(out)[sel], ref, "fp8 stream-K after a timeout")
    finally:
        r.close()


def test_fp8_long_context():
    case = W.paged_case("fp8long", 2, 32, 8, 128, "bf16", 1, 20000, 30000, 16, seed=121,
                        pool_seed=122)
    r = Fp8Run(case, random_history=True)
    try:
        r.append()
        q = case.q(0)
        out = r.cache.attend(0, H.to_device(q, "bf16"), r.seq_lens, r.bt, scale=case.scale)
        assert r.cache.get_error() == kvc.KVC_OK
        sel, ref = r.reference(q)
        H.compare(H.out_to_f64(out)[sel], ref, "fp8 long context")
    finally:
        r.close()


def test_fp8_copy_pages_moves_codes_and_scales():
    case = W.paged_case("fp8cp", 2, 8, 2, 128, "bf16", 1, 100, 400, 16, seed=131, pool_seed=132)
    r = Fp8Run(case)
    try:
        perm = W.rng(133, "pairs").permutation(case.num_pages).astype(np.int32)
        src, dst = perm[:5].copy(), perm[5:10].copy()
        r.cache.copy_pages(i32(src), i32(dst))
        assert r.cache.get_error() == kvc.KVC_OK
        for key in ("kc", "ks", "vc", "vs"):  # byte images: codes and fp32 scales alike
            assert r.o.copy_pages(r.img[key].view(np.uint16), src, dst) == 0
        r.check_pools()
    finally:
        r.close()


def test_fp8_rejections_and_bytes():
    for kwargs in (dict(dtype="fp16"), dict(D=32), dict(page_size=4, num_pages=8)):
        args = dict(B=2, H_kv=2, D=64, max_T=64, dtype="bf16", page_size=0, num_pages=0)
        args.update(kwargs)
        with pytest.raises(kvc.KvcError) as e:
            kvc.KVCache(args["B"], args["H_kv"], args["D"], args["max_T"], args["dtype"],
                        args["page_size"], 1, args["num_pages"], kv_format="fp8")
        assert e.value.status == kvc.KVC_ERR_UNSUPPORTED, kwargs
    c = kvc.KVCache(4, 8, 128, 4096, "bf16", 0, 32, 0, kv_format="fp8")
    try:
        # codes: the KV-bytes formula with 1-byte elements; scales: one fp32 a (token, head)
        assert c.nbytes == (kvc.kvc_bytes_formula(32, 8, 128, 4096, 1, 4) +
                            kvc.kvc_bytes_formula(32, 8, 1, 4096, 4, 4))
    finally:
        c.close()
