"""Run a workload through libkvc (CUDA) and through the oracle on the same inputs.

Both sides receive the same seeded storage words from ``workloads``.  The
CUDA side gets them as device tensors; the oracle gets numpy arrays.  The
oracle never sees anything the CUDA side produced: its cache image is built
by its own append from the initial pool contents.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as oracle_mod
from kv_cache_decode_03_b200 import KVCache
from workloads import Case

ATOL = 2e-3   # max_abs_err bound on the bf16/fp16 attention output (fp32 accumulate)
RTOL = 1e-2   # relative part of the per-element bound |gpu - ref| <= ATOL + RTOL |ref|

TORCH_DT = {"fp16": torch.float16, "bf16": torch.bfloat16}
ORACLE_DT = {"fp16": oracle_mod.FP16, "bf16": oracle_mod.BF16}


def to_device(bits: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.cuda().view(TORCH_DT[dtype])


def from_device(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def out_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


class DeviceCase:
    """A cache with the case's initial pools loaded, plus device copies of the per-step inputs."""

    def __init__(self, case: Case, layers: int = 1):
        self.case = case
        c = case
        self.cache = KVCache(c.B, c.H_kv, c.D, c.max_T, c.dtype, c.page_size, layers,
                             c.num_pages)
        self.seq_lens = torch.from_numpy(c.seq_lens.astype(np.int32)).cuda()
        self.block_table = (torch.from_numpy(c.block_table).cuda() if c.paged else None)
        self.layers = layers

    def load_pools(self, layer: int = 0, k_pool: np.ndarray | None = None,
                   v_pool: np.ndarray | None = None) -> None:
        c = self.case
        kp = c.k_pool(layer) if k_pool is None else k_pool
        vp = c.v_pool(layer) if v_pool is None else v_pool
        self.cache.pool(layer, "k").view(torch.int16).copy_(
            torch.from_numpy(kp.view(np.int16)).reshape(self.cache.pool(layer, "k").shape))
        self.cache.pool(layer, "v").view(torch.int16).copy_(
            torch.from_numpy(vp.view(np.int16)).reshape(self.cache.pool(layer, "v").shape))

    def append(self, layer: int, k_new: np.ndarray, v_new: np.ndarray,
               seq_lens: torch.Tensor | None = None) -> None:
        c = self.case
        self.cache.append(layer, to_device(k_new, c.dtype), to_device(v_new, c.dtype),
                          self.seq_lens if seq_lens is None else seq_lens, self.block_table)

    def attend(self, layer: int, q: np.ndarray, seq_lens: torch.Tensor | None = None
               ) -> torch.Tensor:
        c = self.case
        return self.cache.attend(layer, to_device(q, c.dtype),
                                 self.seq_lens if seq_lens is None else seq_lens,
                                 self.block_table, scale=c.scale)

    def pools(self, layer: int = 0) -> tuple[np.ndarray, np.ndarray]:
        torch.cuda.synchronize()
        return (from_device(self.cache.pool(layer, "k")),
                from_device(self.cache.pool(layer, "v")))

    def close(self) -> None:
        self.cache.close()


def oracle_pools_after_append(case: Case, layer: int = 0, k_pool=None, v_pool=None):
    """The oracle's image of the pools after the case's append (bit-exact reference)."""
    o = oracle_mod.get()
    kp = (case.k_pool(layer) if k_pool is None else k_pool).copy()
    vp = (case.v_pool(layer) if v_pool is None else v_pool).copy()
    if case.paged:
        o.append_paged(kp, case.k_new(layer), case.seq_lens, case.block_table)
        o.append_paged(vp, case.v_new(layer), case.seq_lens, case.block_table)
    else:
        o.append_contig(kp, case.k_new(layer), case.seq_lens)
        o.append_contig(vp, case.v_new(layer), case.seq_lens)
    return kp, vp


def oracle_attend(case: Case, kp: np.ndarray, vp: np.ndarray, q: np.ndarray,
                  requests=None, nthreads: int = 0) -> tuple[np.ndarray, np.ndarray]:
    """fp64 attention for the selected requests from the oracle's pool images.

    Returns (selected request indices, output (n_sel, H_q, T_new, D))."""
    o = oracle_mod.get()
    sel = np.arange(case.B) if requests is None else np.asarray(requests)
    L = case.seq_lens[sel]
    vis = L.astype(np.int64) + case.T_new
    if case.paged:
        T_cap = int(vis.max())
        bt = case.block_table[sel]
        K = o.gather_paged(kp, bt, vis, T_cap)
        V = o.gather_paged(vp, bt, vis, T_cap)
    else:
        K = np.ascontiguousarray(kp[sel])
        V = np.ascontiguousarray(vp[sel])
    out = o.attend(np.ascontiguousarray(q[sel]), K, V, L, case.scale, ORACLE_DT[case.dtype],
                   nthreads=nthreads)
    return sel, out


def compare(got: np.ndarray, ref: np.ndarray, what: str = "") -> dict:
    """Per-element |got - ref| <= ATOL + RTOL |ref|; returns error statistics."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    stats = {"max_abs_err": float(err.max()),
             "max_rel_err": float((err / np.maximum(np.abs(ref), 1e-6)).max()),
             "n_bad": int(bad.sum()), "n": int(err.size)}
    assert stats["n_bad"] == 0, f"{what}: {stats}"
    return stats
