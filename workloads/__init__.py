"""Seeded synthetic inputs for the KV-cache attention step.

This module is shared by the tests, the benchmark and the smoke check, and
it is the ONLY thing the oracle side and the CUDA side have in common.  It
holds no step of the method: it draws random values, committed lengths and
page assignments, and returns them as plain arrays (16-bit storage words for
K/V/q, int32 for lengths and block tables).  Where values land in a cache is
decided by whoever consumes the arrays.

Every array comes from ``numpy.random.default_rng`` seeded with
``[seed, *tags]`` so that any piece (one layer, one request's pool pages) can
be regenerated on its own.  Values are N(0, 1) * std drawn in float32 and
rounded to fp16 (numpy's conversion) or bf16 (round-to-nearest-even on the
float32 bits).

The five workloads reproduce the shapes named for the KV-cache decode path
(decode of one token per request, paged decode with shared prefix pages, and
speculative-verify chunks of gamma tokens); the page they come from gives
shapes and distributions, no datasets.
"""
from __future__ import annotations

import dataclasses
import math
import zlib
from typing import Sequence

import numpy as np

FP16 = "fp16"
BF16 = "bf16"
ELT_BYTES = {FP16: 2, BF16: 2}


# ---------------------------------------------------------------------------
# seeded value streams
# ---------------------------------------------------------------------------

def _tag(t) -> int:
    if isinstance(t, (int, np.integer)):
        return int(t) & 0xFFFFFFFF
    return zlib.crc32(str(t).encode())


def rng(seed: int, *tags) -> np.random.Generator:
    return np.random.default_rng([int(seed)] + [_tag(t) for t in tags])


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 storage words, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def to_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == FP16:
        return np.ascontiguousarray(x).astype(np.float16).view(np.uint16)
    if dtype == BF16:
        return f32_to_bf16_bits(x)
    raise ValueError(dtype)


def normal_bits(shape: Sequence[int], dtype: str, seed: int, *tags, std: float = 1.0,
                chunk_elems: int = 1 << 26) -> np.ndarray:
    """N(0,1)*std storage words of the given shape, drawn in chunks to bound memory."""
    g = rng(seed, *tags)
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        x = g.standard_normal(e - s, dtype=np.float32)
        if std != 1.0:
            x *= np.float32(std)
        out[s:e] = to_bits(x, dtype)
    return out.reshape(tuple(shape))


# ---------------------------------------------------------------------------
# workload descriptions
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Case:
    """One attention workload: shapes, lengths, page assignment and seeds."""

    name: str
    B: int
    H_q: int
    H_kv: int
    D: int
    dtype: str
    T_new: int
    seq_lens: np.ndarray            # int32 (B,): committed length before the new rows
    seed: int
    layers: int = 1
    page_size: int = 0              # 0 = contiguous cache
    max_T: int = 0                  # contiguous capacity per request (paged: logical cap)
    block_table: np.ndarray | None = None  # int32 (B, max_pages), -1 = unused
    num_pages: int = 0
    kv_std: float = 1.0
    q_std: float = 1.0
    shared_requests: np.ndarray | None = None  # requests sharing the prefix pages
    shared_pages: int = 0

    @property
    def paged(self) -> bool:
        return self.page_size > 0

    @property
    def group(self) -> int:
        return self.H_q // self.H_kv

    @property
    def rows(self) -> int:
        return self.group * self.T_new

    @property
    def scale(self) -> float:
        return float(np.float32(1.0 / math.sqrt(self.D)))

    @property
    def max_pages(self) -> int:
        return 0 if self.block_table is None else int(self.block_table.shape[1])

    @property
    def elt(self) -> int:
        return ELT_BYTES[self.dtype]

    def pool_shape(self) -> tuple[int, int, int, int]:
        if self.paged:
            return (self.num_pages, self.H_kv, self.page_size, self.D)
        return (self.B, self.H_kv, self.max_T, self.D)

    # -- values ---------------------------------------------------------
    def q(self, layer: int = 0) -> np.ndarray:
        return normal_bits((self.B, self.H_q, self.T_new, self.D), self.dtype, self.seed,
                           "q", layer, std=self.q_std)

    def k_new(self, layer: int = 0) -> np.ndarray:
        return normal_bits((self.B, self.H_kv, self.T_new, self.D), self.dtype, self.seed,
                           "k_new", layer, std=self.kv_std)

    def v_new(self, layer: int = 0) -> np.ndarray:
        return normal_bits((self.B, self.H_kv, self.T_new, self.D), self.dtype, self.seed,
                           "v_new", layer, std=self.kv_std)

    def k_pool(self, layer: int = 0) -> np.ndarray:
        """Initial K storage (every slot drawn): the past rows the cache already holds."""
        return normal_bits(self.pool_shape(), self.dtype, self.seed, "k_pool", layer,
                           std=self.kv_std)

    def v_pool(self, layer: int = 0) -> np.ndarray:
        return normal_bits(self.pool_shape(), self.dtype, self.seed, "v_pool", layer,
                           std=self.kv_std)

    # -- sizes ----------------------------------------------------------
    def visible(self) -> np.ndarray:
        """Positions the last new row of each request sees (committed + new)."""
        return self.seq_lens.astype(np.int64) + self.T_new

    def kv_read_bytes(self, unique: bool = True) -> int:
        """K+V bytes one attend pass must read, shared prefix pages counted once if unique."""
        tokens = int(self.visible().sum())
        if unique and self.shared_requests is not None and len(self.shared_requests) > 1:
            tokens -= (len(self.shared_requests) - 1) * self.shared_pages * self.page_size
        return tokens * 2 * self.H_kv * self.D * self.elt

    def algorithmic_bytes(self) -> int:
        """Per layer-step: K/V read (+shared once), q in, out written, appended K/V."""
        qo = 2 * self.B * self.H_q * self.T_new * self.D * self.elt
        app = 2 * self.B * self.H_kv * self.T_new * self.D * self.elt
        return self.kv_read_bytes(True) + qo + app


def _page_table(B: int, need_pages: np.ndarray, max_pages: int, shared: np.ndarray,
                shared_pages: int, seed: int) -> tuple[np.ndarray, int]:
    """Block tables over one shuffled pool.

    Requests in ``shared`` map their first ``shared_pages`` logical pages to
    the same physical pages; every other page is private.  Physical ids come
    from one seeded permutation of the pool, assigned shared pages first,
    then each request's private pages in request order.  Unused entries are -1.
    """
    is_shared = np.zeros(B, dtype=bool)
    is_shared[shared] = True
    private = need_pages - np.where(is_shared, shared_pages, 0)
    num_pages = int(shared_pages * (1 if is_shared.any() else 0) + private.sum())
    perm = rng(seed, "pool_perm").permutation(num_pages).astype(np.int32)
    bt = np.full((B, max_pages), -1, dtype=np.int32)
    cur = 0
    shared_ids = None
    if is_shared.any():
        shared_ids = perm[:shared_pages]
        cur = shared_pages
    for b in range(B):
        j0 = 0
        if is_shared[b]:
            bt[b, :shared_pages] = shared_ids
            j0 = shared_pages
        n = int(private[b])
        bt[b, j0:j0 + n] = perm[cur:cur + n]
        cur += n
    assert cur == num_pages
    return bt, num_pages


def paged_case(name: str, B: int, H_q: int, H_kv: int, D: int, dtype: str, T_new: int,
               L_lo: int, L_hi: int, page_size: int, seed: int, pool_seed: int,
               share_frac: float = 0.0, share_tokens: int = 0, kv_std: float = 1.0,
               layers: int = 1) -> Case:
    """Paged workload: committed lengths uniform in [L_lo, L_hi] (inclusive)."""
    L = rng(seed, "seq_lens").integers(L_lo, L_hi, size=B, endpoint=True).astype(np.int32)
    shared = np.zeros(0, dtype=np.int64)
    shared_pages = 0
    if share_frac > 0:
        n_share = int(round(share_frac * B))
        shared = np.sort(rng(seed, "share").permutation(B)[:n_share])
        assert share_tokens % page_size == 0
        shared_pages = share_tokens // page_size
        # a request that shares the prefix holds at least the prefix, so the
        # appended rows (positions >= L_b) fall in its private pages
        L[shared] = np.maximum(L[shared], share_tokens)
    need = -(-(L.astype(np.int64) + T_new) // page_size)
    max_pages = max(-(-(L_hi + T_new) // page_size), int(need.max()))
    bt, num_pages = _page_table(B, need, max_pages, shared, shared_pages, pool_seed)
    return Case(name=name, B=B, H_q=H_q, H_kv=H_kv, D=D, dtype=dtype, T_new=T_new,
                seq_lens=L, seed=seed, layers=layers, page_size=page_size,
                max_T=max_pages * page_size, block_table=bt, num_pages=num_pages,
                kv_std=kv_std, shared_requests=shared if len(shared) else None,
                shared_pages=shared_pages)


def contig_case(name: str, B: int, H_q: int, H_kv: int, D: int, dtype: str, T_new: int,
                L: int | Sequence[int], seed: int, max_T: int | None = None,
                kv_std: float = 1.0, layers: int = 1) -> Case:
    Ls = np.broadcast_to(np.asarray(L, dtype=np.int32), (B,)).copy()
    cap = int(max_T) if max_T is not None else int(Ls.max()) + T_new
    return Case(name=name, B=B, H_q=H_q, H_kv=H_kv, D=D, dtype=dtype, T_new=T_new,
                seq_lens=Ls, seed=seed, layers=layers, max_T=cap, kv_std=kv_std)


# ---------------------------------------------------------------------------
# the five named workloads
# ---------------------------------------------------------------------------

def mha_small(T_past: int = 512) -> Case:
    """MHA decode, 1 layer: B=1, H_q=H_kv=16, D=32, fp16, contiguous, T_new=1 (seed 1)."""
    return contig_case("mha_b1_h16_d32_fp16", 1, 16, 16, 32, FP16, 1, T_past, seed=1)


def mha_sweep(T_past: int) -> Case:
    """MHA decode: B=4, H_q=H_kv=12, D=64, fp16, contiguous, T_new=1 (seed 2)."""
    assert T_past in (512, 1024, 2048, 4096, 8192)
    return contig_case(f"mha_b4_h12_d64_fp16_L{T_past}", 4, 12, 12, 64, FP16, 1, T_past,
                       seed=2)


MHA_SWEEP_T = (512, 1024, 2048, 4096, 8192)
PREFILL_CHUNKS = (64, 128, 1000)


def gqa_32layer(layers: int = 32) -> Case:
    """GQA decode: B=16, H_q=32, H_kv=8, D=128, bf16, contiguous, T_past=4096, 32 layers;
    k,v ~ N(0,1)*0.5, q ~ N(0,1) (seed 3)."""
    return contig_case("gqa_b16_hq32_hkv8_d128_bf16_L4096_x32", 16, 32, 8, 128, BF16, 1,
                       4096, seed=3, kv_std=0.5, layers=layers)


def paged_gqa() -> Case:
    """Paged GQA decode: P=16, B=64, L ~ U[128, 8192], H_q=32, H_kv=8, D=128, bf16;
    16 of 64 requests share the first 1024-token prefix pages; T_new=1 (seeds 4, 5)."""
    return paged_case("paged_gqa_b64_hq32_hkv8_d128_bf16_P16", 64, 32, 8, 128, BF16, 1,
                      128, 8192, 16, seed=4, pool_seed=5, share_frac=0.25,
                      share_tokens=1024)


def spec_verify(gamma: int, H_kv: int) -> Case:
    """Speculative-verify chunk: B=32, T_new=gamma in {2,4,8} causal within the chunk,
    L ~ U[8192, 32768], paged P=16, bf16, D=128, H_q=32, H_kv in {8, 1} (seed 6)."""
    assert gamma in (2, 4, 8) and H_kv in (8, 1)
    return paged_case(f"verify_g{gamma}_b32_hq32_hkv{H_kv}_d128_bf16_P16", 32, 32, H_kv, 128,
                      BF16, gamma, 8192, 32768, 16, seed=6, pool_seed=7)
