"""Oracle for the KV-cache attention step -- TEST INFRASTRUCTURE ONLY.

A plain fp64 CPU statement of what the hot path computes (``oracle.c``),
plus thin numpy marshalling.  Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package; the
product package never does and shares no code with it.

What each function follows (pages cited by title and section):

* ``kv_bytes`` -- "9. 推理：从生成到性能优化" (goclawai.cn/llm/inference),
  section 9.3 "KV Cache": the KV-bytes formula.
* ``append_contig`` / ``append_paged`` / ``gather_paged`` -- the same page,
  9.3 (past K/V never change; the new token's K/V are appended) and 9.6
  (paged KV managed in blocks); "llm-perf-lab" README (preallocated
  append/commit cache).
* ``attend`` -- the naive definition: "项目 9-16" roadmap page, project 11
  (CachedSelfAttention: scores q.K^T * scale, softmax over past+new, times
  V) and project 15 (naive attention materialises the scores), with the
  causal-within-chunk and GQA readings stated in ``oracle.c``.
* ``attend_chunked`` -- "llm-perf-lab" README: chunked attention equals naive
  attention for any chunk size.

Pins (closed forms, library routines, exhaustive checks, page values) live in
``tests/test_oracle_pins.py``; planted-mistake checks in
``tests/test_oracle_mutants.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
SRC = HERE / "oracle.c"
LIB = HERE / "liboracle.so"

FP16 = 0
BF16 = 1

_lib = None
_lib_path = None


def build(src: Path = SRC, out: Path = LIB, defines: tuple[str, ...] = ()) -> Path:
    """Compile the oracle with gcc (-O2, OpenMP).  Returns the .so path."""
    # compile beside the target and rename over it: a process that still has the old
    # library mapped keeps its (unlinked) file intact
    tmp = Path(out).with_name(f".{Path(out).name}.{os.getpid()}.tmp")
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-D_GNU_SOURCE", *[f"-D{d}" for d in defines], str(src), "-o", str(tmp), "-lm"]
    try:
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    finally:
        if tmp.exists():
            tmp.unlink()
    return out


def _bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    P = ctypes.c_void_p
    I = ctypes.c_int
    I64 = ctypes.c_int64
    D = ctypes.c_double
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = I
    lib.oracle_decode.argtypes = [P, P, I64, I]
    lib.oracle_decode.restype = None
    lib.oracle_round.argtypes = [P, P, I64, I]
    lib.oracle_round.restype = None
    lib.oracle_kv_bytes.argtypes = [I64] * 6
    lib.oracle_kv_bytes.restype = ctypes.c_uint64
    lib.oracle_append_contig.argtypes = [I, I, I, I, I, P, P, P]
    lib.oracle_append_contig.restype = None
    lib.oracle_append_paged.argtypes = [I, I, I, I, I, I, P, P, P, P]
    lib.oracle_append_paged.restype = None
    lib.oracle_gather_paged.argtypes = [I, I, I, I, I, I, P, P, P, P]
    lib.oracle_gather_paged.restype = None
    lib.oracle_attend.argtypes = [I, I, I, I, I, I, P, P, P, I, P, D, P, I]
    lib.oracle_attend.restype = None
    lib.oracle_attend_chunked.argtypes = [I, I, I, I, I, I, P, P, P, I, P, D, I, P, I]
    lib.oracle_attend_chunked.restype = None
    lib.oracle_attend_window.argtypes = [I, I, I, I, I, I, P, P, P, I, P, D, I, I, P, I]
    lib.oracle_attend_window.restype = None
    lib.oracle_decode_e4m3.argtypes = [P, P, I64]
    lib.oracle_decode_e4m3.restype = None
    lib.oracle_encode_e4m3.argtypes = [P, P, I64]
    lib.oracle_encode_e4m3.restype = None
    lib.oracle_quantize_fp8.argtypes = [P, I64, I, P, P]
    lib.oracle_quantize_fp8.restype = None
    lib.oracle_append_fp8_contig.argtypes = [I, I, I, I, I, I, P, P, P, P]
    lib.oracle_append_fp8_contig.restype = None
    lib.oracle_append_fp8_paged.argtypes = [I, I, I, I, I, I, P, P, P, P, P]
    lib.oracle_append_fp8_paged.restype = None
    lib.oracle_gather_rows.argtypes = [I, I, I, I, I, I, P, P, P, P]
    lib.oracle_gather_rows.restype = None
    lib.oracle_attend_fp8.argtypes = [I, I, I, I, I, I, P, P, P, P, P, P, D, I, I, P, I]
    lib.oracle_attend_fp8.restype = None
    lib.oracle_commit.argtypes = [I, P, P, I, I]
    lib.oracle_commit.restype = I
    lib.oracle_rollback.argtypes = [I, P, P]
    lib.oracle_rollback.restype = I
    lib.oracle_copy_pages.argtypes = [I, I64, P, P, I, P]
    lib.oracle_copy_pages.restype = I
    return lib


def load(path: Path | None = None) -> ctypes.CDLL:
    """Load (building first if needed) the oracle library."""
    global _lib, _lib_path
    path = Path(path) if path is not None else LIB
    if _lib is not None and _lib_path == path:
        return _lib
    if path == LIB and (not LIB.exists() or LIB.stat().st_mtime < SRC.stat().st_mtime):
        build()
    lib = _bind(ctypes.CDLL(str(path)))
    if path == LIB:
        _lib, _lib_path = lib, path
    return lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected uint16 bit patterns, got {a.dtype}")
    return a


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def dtype_code(name: str) -> int:
    return {"fp16": FP16, "float16": FP16, "bf16": BF16, "bfloat16": BF16}[name]


class Oracle:
    """numpy-level wrappers over one oracle library (the real one or a planted mutant)."""

    def __init__(self, lib: ctypes.CDLL | None = None):
        self.lib = lib if lib is not None else load()

    # -- storage formats -------------------------------------------------
    def decode(self, bits, dtype: int) -> np.ndarray:
        bits = _u16(bits)
        out = np.empty(bits.shape, dtype=np.float64)
        self.lib.oracle_decode(_ptr(bits), _ptr(out), bits.size, dtype)
        return out

    def round(self, x, dtype: int) -> np.ndarray:
        x = np.ascontiguousarray(x, dtype=np.float64)
        out = np.empty(x.shape, dtype=np.uint16)
        self.lib.oracle_round(_ptr(x), _ptr(out), x.size, dtype)
        return out

    # -- KV bytes ---------------------------------------------------------
    def kv_bytes(self, layers, kv_heads, head_dim, seq_len, bytes_per_elem, batch) -> int:
        return int(self.lib.oracle_kv_bytes(layers, kv_heads, head_dim, seq_len,
                                            bytes_per_elem, batch))

    # -- append / gather ------------------------------------------------
    def append_contig(self, cache, new_kv, seq_lens) -> None:
        """cache (B,H_kv,T_cap,D) uint16, updated in place; new_kv (B,H_kv,T_new,D)."""
        new_kv = _u16(new_kv)
        assert cache.dtype == np.uint16 and cache.flags["C_CONTIGUOUS"]
        B, H_kv, T_cap, D = cache.shape
        T_new = new_kv.shape[2]
        sl = _i32(seq_lens)
        assert new_kv.shape == (B, H_kv, T_new, D)
        assert np.all(sl + T_new <= T_cap) and np.all(sl >= 0)
        self.lib.oracle_append_contig(B, H_kv, T_new, D, T_cap, _ptr(new_kv), _ptr(sl),
                                      _ptr(cache))

    def append_paged(self, pool, new_kv, seq_lens, block_table) -> None:
        """pool (num_pages,H_kv,P,D) uint16, updated in place."""
        new_kv = _u16(new_kv)
        assert pool.dtype == np.uint16 and pool.flags["C_CONTIGUOUS"]
        num_pages, H_kv, P, D = pool.shape
        B, _, T_new, _ = new_kv.shape
        sl = _i32(seq_lens)
        bt = _i32(block_table)
        max_pages = bt.shape[1]
        last = (sl + T_new - 1) // P
        assert np.all(last < max_pages)
        rows = np.arange(B)
        for j in range(int(T_new)):
            pages = bt[rows, (sl + j) // P]
            assert np.all((pages >= 0) & (pages < num_pages))
        self.lib.oracle_append_paged(B, H_kv, T_new, D, P, max_pages, _ptr(new_kv),
                                     _ptr(sl), _ptr(bt), _ptr(pool))

    # -- FP8 (E4M3) cache ------------------------------------------------
    def decode_e4m3(self, codes) -> np.ndarray:
        c = np.ascontiguousarray(codes, dtype=np.uint8)
        out = np.empty(c.shape, dtype=np.float64)
        self.lib.oracle_decode_e4m3(_ptr(c), _ptr(out), c.size)
        return out

    def encode_e4m3(self, values) -> np.ndarray:
        v = np.ascontiguousarray(values, dtype=np.float32)
        out = np.empty(v.shape, dtype=np.uint8)
        self.lib.oracle_encode_e4m3(_ptr(v), _ptr(out), v.size)
        return out

    def quantize_fp8(self, rows) -> tuple[np.ndarray, np.ndarray]:
        """bf16 words (..., D) -> E4M3 codes (..., D) and fp32 scales (...)."""
        r = _u16(rows)
        D = r.shape[-1]
        n = r.size // D
        codes = np.empty(r.shape, dtype=np.uint8)
        scales = np.empty(r.shape[:-1], dtype=np.float32)
        self.lib.oracle_quantize_fp8(_ptr(r), n, D, _ptr(codes), _ptr(scales))
        return codes, scales

    def append_fp8(self, codes, scales, new_kv, seq_lens, block_table=None) -> None:
        """Quantise the new rows (B, H_kv, T_new, D) and write codes and scales into the
        pool images in place (oracle.c: oracle_append_fp8_contig / _paged): contiguous
        codes (B, H_kv, T_cap, D) with scales (B, H_kv, T_pad); paged codes
        (num_pages, H_kv, P, D) with scales (num_pages, H_kv, P); row L_b + i of (b, g)
        as for the 16-bit append."""
        nk = _u16(new_kv)
        B, H_kv, T_new, D = nk.shape
        sl = _i32(seq_lens)
        assert codes.dtype == np.uint8 and codes.flags["C_CONTIGUOUS"]
        assert scales.dtype == np.float32 and scales.flags["C_CONTIGUOUS"]
        if block_table is None:
            assert codes.shape[:2] == (B, H_kv) and codes.shape[3] == D
            T_cap, T_pad = codes.shape[2], scales.shape[2]
            assert scales.shape == (B, H_kv, T_pad) and T_pad >= T_cap
            assert np.all((sl >= 0) & (sl + T_new <= T_cap))
            self.lib.oracle_append_fp8_contig(B, H_kv, T_new, D, T_cap, T_pad, _ptr(nk),
                                              _ptr(sl), _ptr(codes), _ptr(scales))
            return
        num_pages, hk, P, d = codes.shape
        assert (hk, d) == (H_kv, D) and scales.shape == (num_pages, H_kv, P)
        bt = _i32(block_table)
        max_pages = bt.shape[1]
        assert np.all((sl + T_new - 1) // P < max_pages)
        rows = np.arange(B)
        for j in range(int(T_new)):
            pages = bt[rows, (sl + j) // P]
            assert np.all((pages >= 0) & (pages < num_pages))
        self.lib.oracle_append_fp8_paged(B, H_kv, T_new, D, P, max_pages, _ptr(nk), _ptr(sl),
                                         _ptr(bt), _ptr(codes), _ptr(scales))

    def gather_rows(self, pool, block_table, n_visible, T_cap: int) -> np.ndarray:
        """Logical (B, H_kv, T_cap, ...) view of a paged pool (num_pages, H_kv, P, ...) of
        any element type: the first n_visible[b] positions, the rest zero."""
        pool = np.ascontiguousarray(pool)
        num_pages, H_kv, P = pool.shape[:3]
        row_bytes = int(np.prod(pool.shape[3:], dtype=np.int64)) * pool.itemsize
        bt = _i32(block_table)
        nv = _i32(n_visible)
        B, max_pages = bt.shape
        assert np.all(nv <= T_cap)
        out = np.zeros((B, H_kv, T_cap) + pool.shape[3:], dtype=pool.dtype)
        self.lib.oracle_gather_rows(B, H_kv, row_bytes, P, max_pages, T_cap, _ptr(pool),
                                    _ptr(bt), _ptr(nv), _ptr(out))
        return out

    def attend_fp8(self, q, Kc, Ks, Vc, Vs, seq_lens, scale: float, window: int = 0,
                   sink: int = 0, nthreads: int = 0) -> np.ndarray:
        """fp64 attention of bf16 queries (B,H_q,T_new,D) over K = Kc * Ks, V = Vc * Vs
        (codes (B,H_kv,T_cap,D), scales (B,H_kv,T_cap))."""
        q = _u16(q)
        Kc = np.ascontiguousarray(Kc, dtype=np.uint8)
        Vc = np.ascontiguousarray(Vc, dtype=np.uint8)
        B, H_kv, T_cap, D = Kc.shape
        Ks = np.ascontiguousarray(Ks[..., :T_cap], dtype=np.float32)
        Vs = np.ascontiguousarray(Vs[..., :T_cap], dtype=np.float32)
        _, H_q, T_new, _ = q.shape
        sl = _i32(seq_lens)
        assert q.shape == (B, H_q, T_new, D) and Vc.shape == Kc.shape
        assert Ks.shape == (B, H_kv, T_cap) and Vs.shape == Ks.shape
        assert np.all(sl + T_new <= T_cap)
        out = np.empty((B, H_q, T_new, D), dtype=np.float64)
        self.lib.oracle_attend_fp8(B, H_q, H_kv, T_new, D, T_cap, _ptr(q), _ptr(Kc), _ptr(Ks),
                                   _ptr(Vc), _ptr(Vs), _ptr(sl), float(scale), int(window),
                                   int(sink), _ptr(out), int(nthreads))
        return out

    # -- commit / rollback / page copy -----------------------------------
    def commit(self, seq_lens, accepted, T_new: int, max_T: int) -> tuple[np.ndarray, int]:
        """New lengths after accepting accepted[b] of T_new appended tokens, and the
        number of requests left unchanged because their count was out of range."""
        sl = _i32(seq_lens).copy()
        acc = _i32(accepted)
        assert acc.shape == sl.shape
        bad = self.lib.oracle_commit(sl.size, _ptr(sl), _ptr(acc), int(T_new), int(max_T))
        return sl, int(bad)

    def rollback(self, seq_lens, drop) -> tuple[np.ndarray, int]:
        """New lengths after dropping drop[b] committed tokens, and the number of
        requests left unchanged because their count was out of range."""
        sl = _i32(seq_lens).copy()
        dr = _i32(drop)
        assert dr.shape == sl.shape
        bad = self.lib.oracle_rollback(sl.size, _ptr(sl), _ptr(dr))
        return sl, int(bad)

    def copy_pages(self, pool, src, dst) -> int:
        """pool (num_pages, ...) uint16, updated in place: page dst[i] := page src[i].
        Returns the number of pairs skipped for an id outside the pool."""
        assert pool.dtype == np.uint16 and pool.flags["C_CONTIGUOUS"]
        s, d = _i32(src), _i32(dst)
        assert s.shape == d.shape
        page_elems = int(np.prod(pool.shape[1:]))
        return int(self.lib.oracle_copy_pages(pool.shape[0], page_elems, _ptr(s), _ptr(d),
                                              s.size, _ptr(pool)))

    def gather_paged(self, pool, block_table, n_visible, T_cap: int) -> np.ndarray:
        """Logical (B,H_kv,T_cap,D) view of the first n_visible[b] positions (rest zero)."""
        pool = _u16(pool)
        num_pages, H_kv, P, D = pool.shape
        bt = _i32(block_table)
        nv = _i32(n_visible)
        B, max_pages = bt.shape
        assert np.all(nv <= T_cap)
        assert np.all((nv + P - 1) // P <= max_pages)
        out = np.zeros((B, H_kv, T_cap, D), dtype=np.uint16)
        self.lib.oracle_gather_paged(B, H_kv, D, P, max_pages, T_cap, _ptr(pool), _ptr(bt),
                                     _ptr(nv), _ptr(out))
        return out

    # -- attention --------------------------------------------------------
    def _check_attend(self, q, K, V, seq_lens):
        q, K, V = _u16(q), _u16(K), _u16(V)
        B, H_q, T_new, D = q.shape
        Bk, H_kv, T_cap, Dk = K.shape
        assert K.shape == V.shape and Bk == B and Dk == D
        assert H_q % H_kv == 0
        sl = _i32(seq_lens)
        assert sl.shape == (B,) and np.all(sl + T_new <= T_cap)
        return q, K, V, sl, B, H_q, H_kv, T_new, D, T_cap

    def attend(self, q, K, V, seq_lens, scale: float, dtype: int, nthreads: int = 0):
        """fp64 output (B,H_q,T_new,D) of exact attention over each request's visible rows."""
        q, K, V, sl, B, H_q, H_kv, T_new, D, T_cap = self._check_attend(q, K, V, seq_lens)
        out = np.empty((B, H_q, T_new, D), dtype=np.float64)
        self.lib.oracle_attend(B, H_q, H_kv, T_new, D, T_cap, _ptr(q), _ptr(K), _ptr(V),
                               dtype, _ptr(sl), float(scale), _ptr(out), int(nthreads))
        return out

    def attend_window(self, q, K, V, seq_lens, scale: float, dtype: int, window: int,
                      sink: int = 0, nthreads: int = 0):
        """fp64 output of attention over each row's last `window` positions and the
        first `sink` positions (window 0: all positions)."""
        q, K, V, sl, B, H_q, H_kv, T_new, D, T_cap = self._check_attend(q, K, V, seq_lens)
        assert window >= 0 and sink >= 0
        out = np.empty((B, H_q, T_new, D), dtype=np.float64)
        self.lib.oracle_attend_window(B, H_q, H_kv, T_new, D, T_cap, _ptr(q), _ptr(K), _ptr(V),
                                      dtype, _ptr(sl), float(scale), int(window), int(sink),
                                      _ptr(out), int(nthreads))
        return out

    def attend_chunked(self, q, K, V, seq_lens, scale: float, dtype: int, chunk: int,
                       nthreads: int = 0):
        q, K, V, sl, B, H_q, H_kv, T_new, D, T_cap = self._check_attend(q, K, V, seq_lens)
        assert chunk >= 1
        out = np.empty((B, H_q, T_new, D), dtype=np.float64)
        self.lib.oracle_attend_chunked(B, H_q, H_kv, T_new, D, T_cap, _ptr(q), _ptr(K),
                                       _ptr(V), dtype, _ptr(sl), float(scale), int(chunk),
                                       _ptr(out), int(nthreads))
        return out


_default: Oracle | None = None


def get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def threads_used(nthreads: int = 0) -> int:
    """The OpenMP thread count ``attend`` uses for ``nthreads`` (0 = OpenMP's default)."""
    return nthreads if nthreads > 0 else int(load().oracle_max_threads())
