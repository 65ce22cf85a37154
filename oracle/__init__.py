"""CPU oracle for the rotated-INT4 paged KV cache -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (``bit_paged_kv_diag_b200``)
never imports it, and this package never imports the product.

Thin numpy wrappers around ``kvq_oracle.c`` (plain loops, IEEE fp32 rotation with a
fixed butterfly order, fp16 scale, round-half-even codes, paged store, fp64 softmax
attention).  Sources, cited by page title and section:

* [P1] "KVキャッシュを4ビットへ — SAW-INT4とシステムを踏まえたINT4量子化" (youngju.dev)
* [P2] "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM Serving"
  (gist.science)
* [P3] "BitDecoding-FP4:FP4 KVキャッシュのネイティブ復号" (sns.style): the NVFP4 cache
  format (``fmt = 1``: E2M1 codes, one E4M3 scale per 16 channels)

Every function is pinned by a ``-m "not gpu"`` test against something other than
itself (explicit matrices, closed forms, invariants, brute force).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    """Load (building first if needed) ``liboracle.so``."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i32p = ctypes.POINTER(ctypes.c_int32)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        i8p = ctypes.POINTER(ctypes.c_int8)
        c_int = ctypes.c_int
        sig = {
            "oracle_half_to_float": (ctypes.c_float, [ctypes.c_uint16]),
            "oracle_float_to_half": (ctypes.c_uint16, [ctypes.c_float]),
            "oracle_hadamard_scale_f32": (ctypes.c_float, [c_int]),
            "oracle_fwht_f32": (c_int, [f32p, c_int, c_int]),
            "oracle_fwht_f64": (c_int, [f64p, c_int, c_int]),
            "oracle_quant_row": (ctypes.c_uint16, [f32p, c_int, i8p]),
            "oracle_pack_codes": (None, [i8p, c_int, u8p]),
            "oracle_unpack_codes": (None, [u8p, c_int, i8p]),
            "oracle_assign_pages": (c_int, [c_int, i32p, c_int, c_int, c_int, i32p, i32p]),
            "oracle_block_bytes": (ctypes.c_size_t, [c_int, c_int, c_int]),
            "oracle_rotate_quant_append": (c_int, [u8p, c_int, c_int, c_int, c_int, c_int, c_int,
                                                   c_int, u16p, u16p, i32p, i32p, i32p, c_int,
                                                   c_int]),
            "oracle_read_row": (c_int, [u8p, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                        c_int, c_int, f32p, c_int]),
            "oracle_decode_one": (c_int, [u8p, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                          c_int, u16p, i32p, i32p, c_int, c_int, ctypes.c_double,
                                          f64p, c_int]),
            "oracle_decode_attention": (c_int, [u8p, c_int, c_int, c_int, c_int, c_int, c_int,
                                                c_int, c_int, u16p, i32p, i32p, c_int,
                                                ctypes.c_double, f64p, c_int]),
            "oracle_e4m3_to_float": (ctypes.c_float, [ctypes.c_uint8]),
            "oracle_float_to_e4m3": (ctypes.c_uint8, [ctypes.c_float]),
            "oracle_e2m1_to_float": (ctypes.c_float, [ctypes.c_uint8]),
            "oracle_float_to_e2m1": (ctypes.c_uint8, [ctypes.c_float]),
            "oracle_quant_row_nvfp4": (None, [f32p, c_int, u8p, u8p]),
            "oracle_attention_dense": (c_int, [f64p, f64p, f64p, c_int, c_int, c_int, c_int,
                                               ctypes.c_double, f64p]),
            "oracle_prefill_attention": (c_int, [u8p, c_int, c_int, c_int, c_int, c_int, c_int,
                                                 c_int, c_int, u16p, i32p, i32p, i32p, c_int,
                                                 ctypes.c_double, f64p, c_int]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def _opt_i32(a):
    if a is None:
        return None, None
    a = _c(a, np.int32)
    return a, _p(a, ctypes.c_int32)


class OracleError(RuntimeError):
    pass


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what} returned {rc}")


# ----------------------------------------------------------------- fp16 ----
def half_to_float(bits: int) -> float:
    return float(lib().oracle_half_to_float(int(bits)))


def float_to_half(x: float) -> int:
    return int(lib().oracle_float_to_half(float(x)))


# ------------------------------------------------------------- rotation ----
def hadamard_scale_f32(b: int) -> np.float32:
    """fp32 constant nearest 1/sqrt(b) used by the fp32 rotation."""
    return np.float32(lib().oracle_hadamard_scale_f32(int(b)))


def fwht_f32(x, b: int) -> np.ndarray:
    """Block-diagonal orthonormal FWHT (fp32, fixed butterfly order) along the last axis."""
    y = _c(x, np.float32).copy()
    n = y.shape[-1]
    flat = y.reshape(-1, n)
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        _check(lib().oracle_fwht_f32(_p(row, ctypes.c_float), n, int(b)), "fwht_f32")
        flat[r] = row
    return flat.reshape(y.shape)


def fwht_f64(x, b: int) -> np.ndarray:
    """Block-diagonal orthonormal FWHT in fp64 along the last axis."""
    y = _c(x, np.float64).copy()
    n = y.shape[-1]
    flat = y.reshape(-1, n)
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        _check(lib().oracle_fwht_f64(_p(row, ctypes.c_double), n, int(b)), "fwht_f64")
        flat[r] = row
    return flat.reshape(y.shape)


# --------------------------------------------------------- quantisation ----
def quant_row(y):
    """Token-wise INT4 quantisation of one rotated fp32 row -> (scale fp16 bits, codes int8)."""
    y = _c(y, np.float32)
    codes = np.zeros(y.shape[-1], np.int8)
    s = lib().oracle_quant_row(_p(y, ctypes.c_float), y.shape[-1], _p(codes, ctypes.c_int8))
    return int(s), codes


def pack_codes(codes) -> np.ndarray:
    codes = _c(codes, np.int8)
    out = np.zeros(codes.shape[-1] // 2, np.uint8)
    lib().oracle_pack_codes(_p(codes, ctypes.c_int8), codes.shape[-1], _p(out, ctypes.c_uint8))
    return out


def unpack_codes(packed, d: int) -> np.ndarray:
    packed = _c(packed, np.uint8)
    out = np.zeros(d, np.int8)
    lib().oracle_unpack_codes(_p(packed, ctypes.c_uint8), d, _p(out, ctypes.c_int8))
    return out


# --------------------------------------------------------------- paging ----
def assign_pages(capacity, page_size: int, num_pages: int, max_pages_per_seq: int,
                 page_order=None) -> np.ndarray:
    """Deterministic page table [batch][max_pages_per_seq] (unused = -1)."""
    cap = _c(capacity, np.int32)
    order, order_p = _opt_i32(page_order)
    pt = np.full((cap.shape[0], max_pages_per_seq), -7, np.int32)
    rc = lib().oracle_assign_pages(cap.shape[0], _p(cap, ctypes.c_int32), page_size, num_pages,
                                   max_pages_per_seq, order_p, _p(pt, ctypes.c_int32))
    _check(rc, "assign_pages")
    return pt


def block_bytes(page_size: int, head_dim: int, fmt: int = 0) -> int:
    return int(lib().oracle_block_bytes(page_size, head_dim, fmt))


# ---------------------------------------------------------------- NVFP4 ----
def e4m3_to_float(b: int) -> float:
    return float(lib().oracle_e4m3_to_float(int(b)))


def float_to_e4m3(x: float) -> int:
    """Nearest E4M3 code (ties to even, saturating at 448)."""
    return int(lib().oracle_float_to_e4m3(float(x)))


def e2m1_to_float(c: int) -> float:
    return float(lib().oracle_e2m1_to_float(int(c)))


def float_to_e2m1(x: float) -> int:
    """Nearest E2M1 code (ties to even, saturating at 6, sign kept)."""
    return int(lib().oracle_float_to_e2m1(float(x)))


def quant_row_nvfp4(y):
    """NVFP4 codes (one per channel, 0..15) and E4M3 block scales of a rotated fp32 row."""
    y = _c(y, np.float32)
    codes = np.zeros(y.shape[0], np.uint8)
    scales = np.zeros(y.shape[0] // 16, np.uint8)
    lib().oracle_quant_row_nvfp4(_p(y, ctypes.c_float), y.shape[0], _p(codes, ctypes.c_uint8),
                                 _p(scales, ctypes.c_uint8))
    return codes, scales


class Geometry:
    """Cache geometry shared by the oracle entry points (plain record); fmt 0 = rotated
    INT4 with one fp16 scale per token, 1 = NVFP4 (E2M1 codes, E4M3 scale per 16)."""

    def __init__(self, num_layers, num_kv_heads, num_q_heads, head_dim, block, page_size,
                 num_pages, max_pages_per_seq, fmt=0):
        self.num_layers = int(num_layers)
        self.num_kv_heads = int(num_kv_heads)
        self.num_q_heads = int(num_q_heads)
        self.head_dim = int(head_dim)
        self.block = int(block)
        self.page_size = int(page_size)
        self.num_pages = int(num_pages)
        self.max_pages_per_seq = int(max_pages_per_seq)
        self.fmt = int(fmt)

    @property
    def pool_bytes(self) -> int:
        return (self.num_layers * self.num_pages * self.num_kv_heads
                * block_bytes(self.page_size, self.head_dim, self.fmt))

    def new_pool(self) -> np.ndarray:
        return np.zeros(self.pool_bytes, np.uint8)


def rotate_quant_append(g: Geometry, pool: np.ndarray, layer: int, k16, v16, cu_new_tokens,
                        seq_lens, page_table) -> None:
    """Append fp16 K/V rows ([T][Hkv][D], given as uint16 bit patterns or float16)
    into ``pool`` (uint8, modified in place)."""
    assert pool.dtype == np.uint8 and pool.flags.c_contiguous
    k = _c(np.asarray(k16).view(np.uint16), np.uint16)
    v = _c(np.asarray(v16).view(np.uint16), np.uint16)
    cu = _c(cu_new_tokens, np.int32)
    sl = _c(seq_lens, np.int32)
    pt = _c(page_table, np.int32)
    rc = lib().oracle_rotate_quant_append(
        _p(pool, ctypes.c_uint8), layer, g.num_pages, g.num_kv_heads, g.head_dim, g.block,
        g.page_size, g.max_pages_per_seq, _p(k, ctypes.c_uint16), _p(v, ctypes.c_uint16),
        _p(cu, ctypes.c_int32), _p(sl, ctypes.c_int32), _p(pt, ctypes.c_int32), cu.shape[0] - 1,
        g.fmt)
    _check(rc, "rotate_quant_append")


def read_row(g: Geometry, pool, layer, page, head, slot, kv) -> np.ndarray:
    out = np.zeros(g.head_dim, np.float32)
    pool = _c(pool, np.uint8)
    rc = lib().oracle_read_row(_p(pool, ctypes.c_uint8), layer, g.num_pages, g.num_kv_heads,
                               g.head_dim, g.page_size, page, head, slot, kv,
                               _p(out, ctypes.c_float), g.fmt)
    _check(rc, "read_row")
    return out


def decode_one(g: Geometry, pool, layer, q16, seq_lens, page_table, b, hq,
               softmax_scale=0.0) -> np.ndarray:
    """fp64 attention output [D] for one (sequence, query head)."""
    pool = _c(pool, np.uint8)
    q = _c(np.asarray(q16).view(np.uint16), np.uint16)
    sl = _c(seq_lens, np.int32)
    pt = _c(page_table, np.int32)
    out = np.zeros(g.head_dim, np.float64)
    rc = lib().oracle_decode_one(_p(pool, ctypes.c_uint8), layer, g.num_pages, g.num_kv_heads,
                                 g.num_q_heads, g.head_dim, g.block, g.page_size,
                                 g.max_pages_per_seq, _p(q, ctypes.c_uint16),
                                 _p(sl, ctypes.c_int32), _p(pt, ctypes.c_int32), int(b), int(hq),
                                 float(softmax_scale), _p(out, ctypes.c_double), g.fmt)
    _check(rc, "decode_one")
    return out


def decode_attention(g: Geometry, pool, layer, q16, seq_lens, page_table,
                     softmax_scale=0.0) -> np.ndarray:
    """fp64 attention outputs [batch][Hq][D]."""
    pool = _c(pool, np.uint8)
    q = _c(np.asarray(q16).view(np.uint16), np.uint16)
    sl = _c(seq_lens, np.int32)
    pt = _c(page_table, np.int32)
    out = np.zeros((sl.shape[0], g.num_q_heads, g.head_dim), np.float64)
    rc = lib().oracle_decode_attention(_p(pool, ctypes.c_uint8), layer, g.num_pages,
                                       g.num_kv_heads, g.num_q_heads, g.head_dim, g.block,
                                       g.page_size, g.max_pages_per_seq, _p(q, ctypes.c_uint16),
                                       _p(sl, ctypes.c_int32), _p(pt, ctypes.c_int32),
                                       sl.shape[0], float(softmax_scale),
                                       _p(out, ctypes.c_double), g.fmt)
    _check(rc, "decode_attention")
    return out


def prefill_attention(g: Geometry, pool, layer, q16, cu_q, seq_lens, page_table,
                      softmax_scale=0.0) -> np.ndarray:
    """Causal chunked-prefill attention, fp64 outputs [cu_q[-1]][Hq][D]: the chunk of
    sequence b is its last cu_q[b+1] - cu_q[b] tokens of seq_lens[b]."""
    pool = _c(pool, np.uint8)
    q = _c(np.asarray(q16).view(np.uint16), np.uint16)
    cu = _c(cu_q, np.int32)
    sl = _c(seq_lens, np.int32)
    pt = _c(page_table, np.int32)
    out = np.zeros((int(cu[-1]), g.num_q_heads, g.head_dim), np.float64)
    rc = lib().oracle_prefill_attention(_p(pool, ctypes.c_uint8), layer, g.num_pages,
                                        g.num_kv_heads, g.num_q_heads, g.head_dim, g.block,
                                        g.page_size, g.max_pages_per_seq, _p(q, ctypes.c_uint16),
                                        _p(cu, ctypes.c_int32), _p(sl, ctypes.c_int32),
                                        _p(pt, ctypes.c_int32), sl.shape[0], float(softmax_scale),
                                        _p(out, ctypes.c_double), g.fmt)
    _check(rc, "prefill_attention")
    return out


def attention_dense(q, keys, values, block, rotate, softmax_scale=0.0) -> np.ndarray:
    q = _c(q, np.float64)
    keys = _c(keys, np.float64)
    values = _c(values, np.float64)
    L, D = keys.shape if keys.size else (0, q.shape[0])
    out = np.zeros(D, np.float64)
    rc = lib().oracle_attention_dense(_p(q, ctypes.c_double), _p(keys, ctypes.c_double),
                                      _p(values, ctypes.c_double), int(L), int(D), int(block),
                                      int(rotate), float(softmax_scale), _p(out, ctypes.c_double))
    _check(rc, "attention_dense")
    return out
