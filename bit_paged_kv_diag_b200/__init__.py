"""Python binding of libkvq.so: rotated-INT4 paged KV cache for NVIDIA B200 (sm_100a).

Argument marshalling only -- every step of the path runs in the library's CUDA kernels.
The names mirror the C ABI in ``include/kvq.h``:

* ``kvq_alloc_pages``          -> :func:`alloc_pages`
* ``kvq_rotate_quant_append``  -> :func:`rotate_quant_append`
* ``kvq_decode_attention``     -> :func:`decode_attention`
* ``kvq_append_decode_attention`` -> :func:`append_decode_attention`
* ``kvq_prefill_attention``    -> :func:`prefill_attention`
* ``kvq_free``                 -> :func:`free`
* ``kvq_assign_pages``, ``kvq_pool_bytes``, ``kvq_get_device_status`` likewise.

PyTorch provides device memory and streams (tensors are passed by ``data_ptr()``, the
stream by ``torch.cuda.current_stream().cuda_stream``).  There is no CPU fallback: if
``libkvq.so`` is missing and cannot be built, importing :func:`lib` raises.
"""
import ctypes
import os

import numpy as np

from . import build as _build

__all__ = [
    "KVQError", "Desc", "Cache", "lib", "pool_bytes", "assign_pages", "alloc_pages",
    "rotate_quant_append", "decode_attention", "append_decode_attention", "prefill_attention",
    "decode_attention_noalloc", "free",
    "get_device_status", "status_string",
    "EXPORTED",
]

KVQ_OK, KVQ_EINVAL, KVQ_EUNSUPPORTED, KVQ_ENOPAGES, KVQ_ECUDA = 0, -1, -2, -3, -4
KVQ_DEV_BAD_PAGE, KVQ_DEV_BAD_POS, KVQ_DEV_TIMEOUT = 1, 2, 4

EXPORTED = (
    "kvq_pool_bytes", "kvq_assign_pages", "kvq_alloc_pages", "kvq_rotate_quant_append",
    "kvq_decode_attention", "kvq_pool_ptr", "kvq_get_device_status", "kvq_free",
    "kvq_status_string", "kvq_decode_attention_noalloc", "kvq_append_decode_attention",
    "kvq_prefill_attention",
)


class KVQError(RuntimeError):
    def __init__(self, what, status):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


FORMAT_INT4 = 0
FORMAT_NVFP4 = 1


class Desc(ctypes.Structure):
    """``kvq_desc``: cache geometry (host integers); ``kv_format`` 0 = rotated INT4,
    1 = NVFP4 (``FORMAT_NVFP4``); omitted trailing fields are 0."""
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_layers", "num_kv_heads", "num_q_heads", "head_dim", "hadamard_block",
        "page_size", "num_pages", "max_batch", "max_pages_per_seq", "kv_format")]

    def __repr__(self):
        return "Desc(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


_lib = None


def lib() -> ctypes.CDLL:
    """Load libkvq.so (building it first with nvcc if it is missing or stale)."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        vp, i32, i32p = ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)
        dp = ctypes.POINTER(Desc)
        sig = {
            "kvq_pool_bytes": (ctypes.c_size_t, [dp]),
            "kvq_assign_pages": (ctypes.c_int, [dp, i32, i32p, i32p, i32p]),
            "kvq_alloc_pages": (ctypes.c_int, [dp, vp, ctypes.c_size_t, i32, i32p, i32p, i32p,
                                               ctypes.POINTER(vp)]),
            "kvq_rotate_quant_append": (ctypes.c_int, [vp, i32, vp, vp, vp, vp, vp, i32, i32, vp]),
            "kvq_decode_attention": (ctypes.c_int, [vp, i32, vp, vp, vp, i32, ctypes.c_float, vp,
                                                    vp]),
            "kvq_pool_ptr": (vp, [vp]),
            "kvq_get_device_status": (ctypes.c_int, [vp, i32p, vp]),
            "kvq_free": (ctypes.c_int, [vp]),
            "kvq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "kvq_decode_attention_noalloc": (ctypes.c_int, [dp, vp, ctypes.c_size_t, i32, vp, vp,
                                                            vp, i32, ctypes.c_float, vp, vp, vp]),
            "kvq_append_decode_attention": (ctypes.c_int, [vp, i32, vp, vp, vp, vp, vp, i32,
                                                           ctypes.c_float, vp, vp]),
            "kvq_prefill_attention": (ctypes.c_int, [vp, i32, vp, vp, vp, vp, i32, i32,
                                                     ctypes.c_float, vp, vp]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().kvq_status_string(int(status)).decode()


def _check(rc, what):
    if rc != KVQ_OK:
        raise KVQError(what, rc)


def _i32(a):
    a = np.ascontiguousarray(a, dtype=np.int32)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def pool_bytes(desc: Desc) -> int:
    return int(lib().kvq_pool_bytes(ctypes.byref(desc)))


def assign_pages(desc: Desc, capacity_tokens, page_order=None) -> np.ndarray:
    """Host-only deterministic page table [batch][max_pages_per_seq] (unused = -1)."""
    cap, capp = _i32(capacity_tokens)
    order, orderp = (None, None) if page_order is None else _i32(page_order)
    pt = np.full((cap.shape[0], desc.max_pages_per_seq), -7, np.int32)
    rc = lib().kvq_assign_pages(ctypes.byref(desc), cap.shape[0], capp, orderp,
                                pt.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    _check(rc, "kvq_assign_pages")
    return pt


def _stream_ptr(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dev_ptr(t, what, dtype=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{what} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    return t.data_ptr()


class Cache:
    """Owner of a ``kvq_cache*`` handle.  ``pool`` is the torch tensor backing the pool
    when the caller supplied one (kept alive here)."""

    def __init__(self, handle, desc, pool_tensor):
        self.handle = handle
        self.desc = desc
        self.pool = pool_tensor

    @property
    def pool_ptr(self) -> int:
        return int(lib().kvq_pool_ptr(self.handle) or 0)

    def close(self):
        if self.handle:
            rc = lib().kvq_free(self.handle)
            self.handle = None
            _check(rc, "kvq_free")

    def __del__(self):
        try:
            if self.handle:
                lib().kvq_free(self.handle)
                self.handle = None
        except Exception:
            pass


def alloc_pages(desc: Desc, capacity_tokens=None, page_order=None, pool=None):
    """Create a cache handle; returns ``(cache, page_table)`` with the host page table
    (np.int32 [batch][max_pages_per_seq]).  ``pool``: optional torch uint8 CUDA tensor of
    at least :func:`pool_bytes` bytes (the library allocates one otherwise)."""
    cap = np.zeros(0, np.int32) if capacity_tokens is None else capacity_tokens
    cap, capp = _i32(cap)
    order, orderp = (None, None) if page_order is None else _i32(page_order)
    pt = np.full((cap.shape[0], desc.max_pages_per_seq), -7, np.int32)
    pool_ptr, nbytes = None, 0
    if pool is not None:
        import torch
        pool_ptr = _dev_ptr(pool, "pool", torch.uint8)
        nbytes = pool.numel()
    h = ctypes.c_void_p()
    rc = lib().kvq_alloc_pages(ctypes.byref(desc), pool_ptr, nbytes, cap.shape[0], capp,
                               orderp, pt.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                               ctypes.byref(h))
    _check(rc, "kvq_alloc_pages")
    return Cache(h, desc, pool), pt


def rotate_quant_append(cache: Cache, layer: int, k, v, cu_new_tokens, seq_lens, page_table,
                        stream=None) -> None:
    """Fused rotate + quantise + paged append of fp16 k, v [T][Hkv][128] (CUDA): INT4 rows,
    or NVFP4 rows for a cache made with kv_format = FORMAT_NVFP4.  Token t of sequence b
    (cu_new_tokens[b] <= t < cu_new_tokens[b+1]) lands at position seq_lens[b] + t -
    cu_new_tokens[b]; seq_lens is not updated."""
    import torch
    T = int(k.shape[0])
    batch = int(seq_lens.shape[0])
    rc = lib().kvq_rotate_quant_append(
        cache.handle, int(layer), _dev_ptr(k, "k", torch.float16), _dev_ptr(v, "v", torch.float16),
        _dev_ptr(cu_new_tokens, "cu_new_tokens", torch.int32),
        _dev_ptr(seq_lens, "seq_lens", torch.int32), _dev_ptr(page_table, "page_table", torch.int32),
        batch, T, _stream_ptr(stream))
    _check(rc, "kvq_rotate_quant_append")


def decode_attention(cache: Cache, layer: int, q, seq_lens, page_table, softmax_scale=0.0,
                     out=None, stream=None):
    """Paged GQA decode attention; q fp16 [batch][Hq][128] -> out fp16 (same shape)."""
    import torch
    if out is None:
        out = torch.empty_like(q)
    batch = int(seq_lens.shape[0])
    rc = lib().kvq_decode_attention(
        cache.handle, int(layer), _dev_ptr(q, "q", torch.float16),
        _dev_ptr(seq_lens, "seq_lens", torch.int32), _dev_ptr(page_table, "page_table", torch.int32),
        batch, float(softmax_scale), _dev_ptr(out, "out", torch.float16), _stream_ptr(stream))
    _check(rc, "kvq_decode_attention")
    return out


def append_decode_attention(cache: Cache, layer: int, k_new, v_new, q, seq_lens, page_table,
                            softmax_scale=0.0, out=None, stream=None):
    """One new token per sequence appended at seq_lens[b] (lengths before the append) and
    decode attention over seq_lens[b] + 1 tokens, in one launch."""
    import torch
    if out is None:
        out = torch.empty_like(q)
    batch = int(seq_lens.shape[0])
    rc = lib().kvq_append_decode_attention(
        cache.handle, int(layer), _dev_ptr(k_new, "k_new", torch.float16),
        _dev_ptr(v_new, "v_new", torch.float16), _dev_ptr(q, "q", torch.float16),
        _dev_ptr(seq_lens, "seq_lens", torch.int32), _dev_ptr(page_table, "page_table", torch.int32),
        batch, float(softmax_scale), _dev_ptr(out, "out", torch.float16), _stream_ptr(stream))
    _check(rc, "kvq_append_decode_attention")
    return out


def prefill_attention(cache: Cache, layer: int, q, cu_q, seq_lens, page_table, softmax_scale=0.0,
                      out=None, stream=None, total_q=None):
    """Causal chunked-prefill attention: q fp16 [total_q][Hq][128] (chunks concatenated),
    cu_q int32 [batch+1], seq_lens int32 [batch] (lengths with the chunk appended)."""
    import torch
    if out is None:
        out = torch.empty_like(q)
    batch = int(seq_lens.shape[0])
    tq = int(q.shape[0]) if total_q is None else int(total_q)
    rc = lib().kvq_prefill_attention(
        cache.handle, int(layer), _dev_ptr(q, "q", torch.float16),
        _dev_ptr(cu_q, "cu_q", torch.int32), _dev_ptr(seq_lens, "seq_lens", torch.int32),
        _dev_ptr(page_table, "page_table", torch.int32), batch, tq, float(softmax_scale),
        _dev_ptr(out, "out", torch.float16), _stream_ptr(stream))
    _check(rc, "kvq_prefill_attention")
    return out


def decode_attention_noalloc(desc: Desc, pool, layer: int, q, seq_lens, page_table,
                             softmax_scale=0.0, out=None, status=None, stream=None):
    """Decode attention without a handle and without any device allocation by the library
    (its scratch lives in a fixed device array; limits in include/kvq.h).  ``status``: an
    optional int32 CUDA tensor of one element that receives the KVQ_DEV_* bits."""
    import torch
    if out is None:
        out = torch.empty_like(q)
    batch = int(seq_lens.shape[0])
    st = None if status is None else _dev_ptr(status, "status", torch.int32)
    rc = lib().kvq_decode_attention_noalloc(
        ctypes.byref(desc), _dev_ptr(pool, "pool", torch.uint8), int(pool.numel()), int(layer),
        _dev_ptr(q, "q", torch.float16), _dev_ptr(seq_lens, "seq_lens", torch.int32),
        _dev_ptr(page_table, "page_table", torch.int32), batch, float(softmax_scale),
        _dev_ptr(out, "out", torch.float16), st, _stream_ptr(stream))
    _check(rc, "kvq_decode_attention_noalloc")
    return out


def get_device_status(cache: Cache, stream=None) -> int:
    """Read and clear the device status word (KVQ_DEV_* bits); synchronises the stream."""
    v = ctypes.c_int32(0)
    rc = lib().kvq_get_device_status(cache.handle, ctypes.byref(v), _stream_ptr(stream))
    _check(rc, "kvq_get_device_status")
    return int(v.value)


def free(cache: Cache) -> None:
    cache.close()
