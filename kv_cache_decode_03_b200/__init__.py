"""kv_cache_decode_03_b200 -- Python binding of libkvc, the B200 KV-cache attention library.

Argument marshalling only: every step of the path (append, split-K attend,
log-sum-exp combine) runs in the CUDA kernels of ``libkvc.so``.  The
functions below carry the names of the C ABI in ``include/kvc.h`` and take
plain integers (device addresses, sizes); ``KVCache`` is a small convenience
wrapper that takes torch CUDA tensors and passes their addresses and the
current CUDA stream.

There is no fallback: importing works without a GPU (for symbol checks), but
any call fails loudly if ``libkvc.so`` is missing or the CUDA call fails.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

LIB_PATH = Path(__file__).resolve().with_name("libkvc.so")

KVC_OK = 0
KVC_ERR_INVALID_ARG = 1
KVC_ERR_UNSUPPORTED = 2
KVC_ERR_OOM = 3
KVC_ERR_CUDA = 4
KVC_ERR_BOUNDS = 5
KVC_ERR_TIMEOUT = 6
KVC_ERR_SCRATCH = 7

KVC_FP16 = 0
KVC_BF16 = 1

_DTYPE_CODES = {"fp16": KVC_FP16, "float16": KVC_FP16, "bf16": KVC_BF16, "bfloat16": KVC_BF16}


class KvcError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {kvc_status_string(status)} ({status})")


_lib: ctypes.CDLL | None = None


def library() -> ctypes.CDLL:
    """Load libkvc.so (once).  Raises ImportError if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not LIB_PATH.exists():
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m kv_cache_decode_03_b200.build`")
    lib = ctypes.CDLL(str(LIB_PATH))
    P, I, F, LL, SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_longlong,
                       ctypes.c_size_t)
    sig = {
        "kvc_create": ([I, I, I, I, I, I, I, I, ctypes.POINTER(P)], I),
        "kvc_destroy": ([P], I),
        "kvc_bytes": ([P], SZ),
        "kvc_bytes_formula": ([I, I, I, LL, I, I], SZ),
        "kvc_append": ([P, I, P, P, I, P, I, P, P], I),
        "kvc_attend": ([P, I, P, I, I, P, I, P, F, P, P], I),
        "kvc_attend_noalloc": ([P, I, P, I, I, P, I, P, F, P, P], I),
        "kvc_attend_window": ([P, I, P, I, I, P, I, P, F, I, I, P, P], I),
        "kvc_append_attend": ([P, I, P, P, P, I, I, P, I, P, F, P, P], I),
        "kvc_reserve": ([P, I, I, I], I),
        "kvc_get_error": ([P], I),
        "kvc_status_string": ([I], ctypes.c_char_p),
        "kvc_k_pool": ([P, I], P),
        "kvc_v_pool": ([P, I], P),
        "kvc_layer_pool_bytes": ([P], SZ),
        "kvc_plan_splits": ([P, I, I, I, ctypes.POINTER(I), ctypes.POINTER(I)], I),
        "kvc_create_quantized": ([I, I, I, I, I, I, I, I, I, ctypes.POINTER(P)], I),
        "kvc_k_scales": ([P, I], P),
        "kvc_v_scales": ([P, I], P),
        "kvc_layer_scale_floats": ([P], SZ),
        "kvc_commit": ([P, P, P, I, P], I),
        "kvc_rollback": ([P, P, P, P], I),
        "kvc_copy_pages": ([P, P, P, I, P], I),
        "kvc_set_dependent_launch": ([P, I], I),
        "kvc_set_wait_limit": ([P, ctypes.c_ulonglong], I),
        "kvc_inject_stall": ([P], I),
        "kvc_inject_replan": ([P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _check(status: int, where: str) -> None:
    if status != KVC_OK:
        raise KvcError(status, where)


# ---------------------------------------------------------------------------
# the C ABI, one function each
# ---------------------------------------------------------------------------

def kvc_status_string(status: int) -> str:
    return library().kvc_status_string(int(status)).decode()


def kvc_create(B: int, H_kv: int, D: int, max_T: int, dtype, page_size: int = 0,
               num_layers: int = 1, num_pages: int = 0) -> int:
    code = _DTYPE_CODES[dtype] if isinstance(dtype, str) else int(dtype)
    h = ctypes.c_void_p()
    _check(library().kvc_create(B, H_kv, D, max_T, code, page_size, num_layers, num_pages,
                                ctypes.byref(h)), "kvc_create")
    return int(h.value)


KV_FORMATS = {"native": 0, "fp8": 1}


def kvc_create_quantized(B: int, H_kv: int, D: int, max_T: int, dtype, kv_format,
                         page_size: int = 0, num_layers: int = 1, num_pages: int = 0) -> int:
    code = _DTYPE_CODES[dtype] if isinstance(dtype, str) else int(dtype)
    fmt = KV_FORMATS[kv_format] if isinstance(kv_format, str) else int(kv_format)
    h = ctypes.c_void_p()
    _check(library().kvc_create_quantized(B, H_kv, D, max_T, code, fmt, page_size, num_layers,
                                          num_pages, ctypes.byref(h)), "kvc_create_quantized")
    return int(h.value)


def kvc_destroy(cache: int) -> None:
    _check(library().kvc_destroy(cache), "kvc_destroy")


def kvc_bytes(cache: int) -> int:
    return int(library().kvc_bytes(cache))


def kvc_bytes_formula(layers: int, kv_heads: int, head_dim: int, seq_len: int,
                      bytes_per_elem: int, batch: int) -> int:
    return int(library().kvc_bytes_formula(layers, kv_heads, head_dim, seq_len,
                                           bytes_per_elem, batch))


def kvc_append(cache: int, layer: int, k_new: int, v_new: int, T_new: int, block_table: int,
               max_pages: int, seq_lens: int, stream: int) -> None:
    _check(library().kvc_append(cache, layer, k_new, v_new, T_new, block_table or None,
                                max_pages, seq_lens, stream or None), "kvc_append")


def kvc_attend(cache: int, layer: int, q: int, H_q: int, T_new: int, block_table: int,
               max_pages: int, seq_lens: int, scale: float, out: int, stream: int) -> None:
    _check(library().kvc_attend(cache, layer, q, H_q, T_new, block_table or None, max_pages,
                                seq_lens, scale, out, stream or None), "kvc_attend")


def kvc_attend_window(cache: int, layer: int, q: int, H_q: int, T_new: int, block_table: int,
                      max_pages: int, seq_lens: int, scale: float, window: int, sink: int,
                      out: int, stream: int) -> None:
    _check(library().kvc_attend_window(cache, layer, q, H_q, T_new, block_table or None,
                                       max_pages, seq_lens, scale, window, sink, out,
                                       stream or None), "kvc_attend_window")


def kvc_append_attend(cache: int, layer: int, k_new: int, v_new: int, q: int, H_q: int,
                      T_new: int, block_table: int, max_pages: int, seq_lens: int, scale: float,
                      out: int, stream: int) -> None:
    _check(library().kvc_append_attend(cache, layer, k_new, v_new, q, H_q, T_new,
                                       block_table or None, max_pages, seq_lens, scale, out,
                                       stream or None), "kvc_append_attend")


def kvc_attend_noalloc(cache: int, layer: int, q: int, H_q: int, T_new: int, block_table: int,
                       max_pages: int, seq_lens: int, scale: float, out: int,
                       stream: int) -> None:
    """kvc_attend with its split-K scratch in the library's fixed device array (no
    device allocation; see include/kvc.h for who needs this and the limits)."""
    _check(library().kvc_attend_noalloc(cache, layer, q, H_q, T_new, block_table or None,
                                        max_pages, seq_lens, scale, out, stream or None),
           "kvc_attend_noalloc")


def kvc_reserve(cache: int, H_q: int, T_new: int, max_pages: int = 0) -> None:
    _check(library().kvc_reserve(cache, H_q, T_new, max_pages), "kvc_reserve")


def kvc_get_error(cache: int) -> int:
    """Synchronise and return (and clear) the sticky device status; does not raise."""
    return int(library().kvc_get_error(cache))


def kvc_k_pool(cache: int, layer: int) -> int:
    return int(library().kvc_k_pool(cache, layer) or 0)


def kvc_v_pool(cache: int, layer: int) -> int:
    return int(library().kvc_v_pool(cache, layer) or 0)


def kvc_layer_pool_bytes(cache: int) -> int:
    return int(library().kvc_layer_pool_bytes(cache))


def kvc_k_scales(cache: int, layer: int) -> int:
    return int(library().kvc_k_scales(cache, layer) or 0)


def kvc_v_scales(cache: int, layer: int) -> int:
    return int(library().kvc_v_scales(cache, layer) or 0)


def kvc_layer_scale_floats(cache: int) -> int:
    return int(library().kvc_layer_scale_floats(cache))


def kvc_plan_splits(cache: int, H_q: int, T_new: int, max_pages: int = 0) -> tuple[int, int]:
    ns, st = ctypes.c_int(), ctypes.c_int()
    _check(library().kvc_plan_splits(cache, H_q, T_new, max_pages, ctypes.byref(ns),
                                     ctypes.byref(st)), "kvc_plan_splits")
    return ns.value, st.value


def kvc_commit(cache: int, seq_lens: int, accepted: int, T_new: int, stream: int) -> None:
    _check(library().kvc_commit(cache, seq_lens, accepted, T_new, stream or None), "kvc_commit")


def kvc_rollback(cache: int, seq_lens: int, drop: int, stream: int) -> None:
    _check(library().kvc_rollback(cache, seq_lens, drop, stream or None), "kvc_rollback")


def kvc_copy_pages(cache: int, src: int, dst: int, n: int, stream: int) -> None:
    _check(library().kvc_copy_pages(cache, src or None, dst or None, n, stream or None),
           "kvc_copy_pages")


def kvc_set_dependent_launch(cache: int, on: bool) -> None:
    _check(library().kvc_set_dependent_launch(cache, 1 if on else 0), "kvc_set_dependent_launch")


def kvc_set_wait_limit(cache: int, ns: int) -> None:
    _check(library().kvc_set_wait_limit(cache, int(ns)), "kvc_set_wait_limit")


def kvc_inject_stall(cache: int) -> None:
    _check(library().kvc_inject_stall(cache), "kvc_inject_stall")


def kvc_inject_replan(cache: int) -> None:
    _check(library().kvc_inject_replan(cache), "kvc_inject_replan")


# ---------------------------------------------------------------------------
# torch convenience wrapper
# ---------------------------------------------------------------------------

class _DeviceView:
    """__cuda_array_interface__ over memory the cache owns (keeps the cache alive)."""

    def __init__(self, owner, ptr: int, nbytes: int, typestr: str = "<i2"):
        self._owner = owner
        size = int(typestr[-1])
        self.__cuda_array_interface__ = {
            "shape": (nbytes // size,), "typestr": typestr, "data": (ptr, False),
            "version": 3, "strides": None,
        }


class KVCache:
    """A cache handle plus torch-tensor marshalling for append / attend."""

    def __init__(self, B: int, H_kv: int, D: int, max_T: int, dtype: str = "bf16",
                 page_size: int = 0, num_layers: int = 1, num_pages: int = 0,
                 kv_format: str = "native"):
        import torch
        self.torch_dtype = {"fp16": torch.float16, "bf16": torch.bfloat16}[dtype]
        self.B, self.H_kv, self.D, self.max_T = B, H_kv, D, max_T
        self.dtype, self.page_size, self.num_layers, self.num_pages = (dtype, page_size,
                                                                      num_layers, num_pages)
        self.kv_format = kv_format
        if kv_format == "native":
            self.handle = kvc_create(B, H_kv, D, max_T, dtype, page_size, num_layers, num_pages)
        else:
            self.handle = kvc_create_quantized(B, H_kv, D, max_T, dtype, kv_format, page_size,
                                               num_layers, num_pages)

    def close(self) -> None:
        if self.handle:
            kvc_destroy(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def nbytes(self) -> int:
        return kvc_bytes(self.handle)

    def pool(self, layer: int, which: str):
        """A torch view of one layer's K or V pool, in its layout: contiguous
        (B, H_kv, max_T, D) or paged (num_pages, H_kv, page_size, D); the cache's dtype,
        or uint8 E4M3 codes for an FP8 cache."""
        import torch
        ptr = kvc_k_pool(self.handle, layer) if which == "k" else kvc_v_pool(self.handle, layer)
        if not ptr:
            raise IndexError(layer)
        nbytes = kvc_layer_pool_bytes(self.handle)
        shape = ((self.num_pages, self.H_kv, self.page_size, self.D) if self.page_size
                 else (self.B, self.H_kv, self.max_T, self.D))
        if self.kv_format == "fp8":
            t = torch.as_tensor(_DeviceView(self, ptr, nbytes, "|u1"), device="cuda")
            return t.view(shape)
        t = torch.as_tensor(_DeviceView(self, ptr, nbytes), device="cuda")
        return t.view(self.torch_dtype).view(shape)

    def scales(self, layer: int, which: str):
        """fp32 scales of an FP8 cache: contiguous (B, H_kv, T_pad), paged
        (num_pages, H_kv, page_size)."""
        import torch
        ptr = (kvc_k_scales(self.handle, layer) if which == "k"
               else kvc_v_scales(self.handle, layer))
        if not ptr:
            raise IndexError(layer)
        n = kvc_layer_scale_floats(self.handle)
        t = torch.as_tensor(_DeviceView(self, ptr, 4 * n, "<f4"), device="cuda")
        if self.page_size:
            return t.view(self.num_pages, self.H_kv, self.page_size)
        return t.view(self.B, self.H_kv, n // (self.B * self.H_kv))

    def _stream(self, stream) -> int:
        import torch
        s = stream if stream is not None else torch.cuda.current_stream()
        return int(s.cuda_stream)

    def _dev(self, t, name: str, dtype=None):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
        if dtype is not None and t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
        return int(t.data_ptr())

    def append(self, layer: int, k_new, v_new, seq_lens, block_table=None, stream=None):
        import torch
        T_new = int(k_new.shape[2])
        assert tuple(k_new.shape) == (self.B, self.H_kv, T_new, self.D) == tuple(v_new.shape)
        bt = 0 if block_table is None else self._dev(block_table, "block_table", torch.int32)
        mp = 0 if block_table is None else int(block_table.shape[1])
        kvc_append(self.handle, layer, self._dev(k_new, "k_new", self.torch_dtype),
                   self._dev(v_new, "v_new", self.torch_dtype), T_new, bt, mp,
                   self._dev(seq_lens, "seq_lens", torch.int32), self._stream(stream))

    def attend(self, layer: int, q, seq_lens, block_table=None, scale: float | None = None,
               out=None, stream=None):
        import torch
        B, H_q, T_new, D = (int(x) for x in q.shape)
        assert B == self.B and D == self.D
        if out is None:
            out = torch.empty_like(q)
        if scale is None:
            scale = 1.0 / D ** 0.5
        bt = 0 if block_table is None else self._dev(block_table, "block_table", torch.int32)
        mp = 0 if block_table is None else int(block_table.shape[1])
        kvc_attend(self.handle, layer, self._dev(q, "q", self.torch_dtype), H_q, T_new, bt, mp,
                   self._dev(seq_lens, "seq_lens", torch.int32), float(scale),
                   self._dev(out, "out", self.torch_dtype), self._stream(stream))
        return out

    def attend_window(self, layer: int, q, seq_lens, window: int, sink: int = 0,
                      block_table=None, scale: float | None = None, out=None, stream=None):
        """Attention over the last `window` positions plus the first `sink` of each row."""
        import torch
        B, H_q, T_new, D = (int(x) for x in q.shape)
        assert B == self.B and D == self.D
        if out is None:
            out = torch.empty_like(q)
        if scale is None:
            scale = 1.0 / D ** 0.5
        bt = 0 if block_table is None else self._dev(block_table, "block_table", torch.int32)
        mp = 0 if block_table is None else int(block_table.shape[1])
        kvc_attend_window(self.handle, layer, self._dev(q, "q", self.torch_dtype), H_q, T_new,
                          bt, mp, self._dev(seq_lens, "seq_lens", torch.int32), float(scale),
                          int(window), int(sink), self._dev(out, "out", self.torch_dtype),
                          self._stream(stream))
        return out

    def append_attend(self, layer: int, k_new, v_new, q, seq_lens, block_table=None,
                      scale: float | None = None, out=None, stream=None):
        """kvc_append then kvc_attend for the same tokens, fused where possible."""
        import torch
        B, H_q, T_new, D = (int(x) for x in q.shape)
        assert tuple(k_new.shape) == (self.B, self.H_kv, T_new, self.D) == tuple(v_new.shape)
        if out is None:
            out = torch.empty_like(q)
        if scale is None:
            scale = 1.0 / D ** 0.5
        bt = 0 if block_table is None else self._dev(block_table, "block_table", torch.int32)
        mp = 0 if block_table is None else int(block_table.shape[1])
        kvc_append_attend(self.handle, layer, self._dev(k_new, "k_new", self.torch_dtype),
                          self._dev(v_new, "v_new", self.torch_dtype),
                          self._dev(q, "q", self.torch_dtype), H_q, T_new, bt, mp,
                          self._dev(seq_lens, "seq_lens", torch.int32), float(scale),
                          self._dev(out, "out", self.torch_dtype), self._stream(stream))
        return out

    def reserve(self, H_q: int, T_new: int, max_pages: int = 0) -> None:
        kvc_reserve(self.handle, H_q, T_new, max_pages)

    def get_error(self) -> int:
        return kvc_get_error(self.handle)

    def plan(self, H_q: int, T_new: int, max_pages: int = 0) -> tuple[int, int]:
        return kvc_plan_splits(self.handle, H_q, T_new, max_pages)

    def set_dependent_launch(self, on: bool) -> None:
        kvc_set_dependent_launch(self.handle, on)

    def set_wait_limit(self, ns: int) -> None:
        kvc_set_wait_limit(self.handle, ns)

    def inject_stall(self) -> None:
        kvc_inject_stall(self.handle)

    def inject_replan(self) -> None:
        kvc_inject_replan(self.handle)

    def commit(self, seq_lens, accepted, T_new: int, stream=None) -> None:
        """seq_lens[b] += accepted[b] on the device (0 <= accepted[b] <= T_new)."""
        import torch
        kvc_commit(self.handle, self._dev(seq_lens, "seq_lens", torch.int32),
                   self._dev(accepted, "accepted", torch.int32), int(T_new), self._stream(stream))

    def rollback(self, seq_lens, drop, stream=None) -> None:
        """seq_lens[b] -= drop[b] on the device (0 <= drop[b] <= seq_lens[b])."""
        import torch
        kvc_rollback(self.handle, self._dev(seq_lens, "seq_lens", torch.int32),
                     self._dev(drop, "drop", torch.int32), self._stream(stream))

    def copy_pages(self, src, dst, stream=None) -> None:
        """Page dst[i] := page src[i] in every layer, K and V (paged caches)."""
        import torch
        n = int(src.numel())
        if int(dst.numel()) != n:
            raise ValueError("src and dst must hold the same number of pages")
        kvc_copy_pages(self.handle, self._dev(src, "src", torch.int32) if n else 0,
                       self._dev(dst, "dst", torch.int32) if n else 0, n, self._stream(stream))
