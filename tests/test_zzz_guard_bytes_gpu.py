"""Writes stay inside their buffers: every call of the C ABI on a pool and on outputs that
sit between guard bytes (a stand-in for a memory checker, which is not available here).

The case: 3 KV heads (not a power of two), G = 4, ragged lengths with an empty sequence,
the last of two layers (so the first layer's bytes must stay zero and the pool's end is
next to a guard), every call in turn -- a prefill append, a chunk append and the chunk's
causal prefill attention, a decode, a fused one-token append + decode, an allocation-free
decode -- on both cache formats.  Afterwards the guards hold their fill, the status word
is clear and every output is finite.  This file runs last, after every parity test."""
import dataclasses

import numpy as np
import pytest

import workloads
from harness import make_case

pytestmark = pytest.mark.gpu

GUARD = 4096
FILL = 0xA5


def _guarded(nbytes, dev):
    import torch
    buf = torch.full((nbytes + 2 * GUARD,), FILL, dtype=torch.uint8, device=dev)
    return buf, buf[GUARD:GUARD + nbytes]


def _intact(buf):
    return bool((buf[:GUARD] == FILL).all().item()) and bool((buf[-GUARD:] == FILL).all().item())


def _guarded_like(q, dev):
    import torch
    buf, b8 = _guarded(q.numel() * 2, dev)
    return buf, b8.view(torch.float16).view(q.shape)


@pytest.mark.parametrize("fmt", [0, 1])
def test_calls_write_only_inside_their_buffers(fmt):
    import torch
    import bit_paged_kv_diag_b200 as kvq
    w = dataclasses.replace(workloads.WORKLOADS["qwen3_4b_decode"], num_kv_heads=3,
                            num_q_heads=12)
    lengths = np.array([300, 1, 513, 0, 64], np.int32)
    chunk = np.array([3, 1, 2, 1, 4], np.int32)
    B = len(lengths)
    case = make_case(w, lengths, chunk + 1, permute=True, pool_factor=1.3, layer=1,
                     num_layers=2, fmt=fmt)
    dev = torch.device("cuda")
    t = lambda a: torch.as_tensor(a).to(dev)  # noqa: E731
    d = case.desc()
    nbytes = kvq.pool_bytes(d)
    pbuf, pool = _guarded(nbytes, dev)
    pool.zero_()
    cache, page_table = kvq.alloc_pages(d, case.capacity, case.page_order, pool=pool)
    try:
        pt = t(page_table)
        L = 1
        # prefill append, then the chunk's append at the cached lengths
        kvq.rotate_quant_append(cache, L, t(workloads.kv_rows(w, L, 0, int(lengths.sum()), 1)),
                                t(workloads.kv_rows(w, L, 1, int(lengths.sum()), 1)),
                                t(workloads.cu_seqlens(lengths)), t(np.zeros(B, np.int32)), pt)
        kvq.rotate_quant_append(cache, L, t(workloads.kv_rows(w, L, 0, int(chunk.sum()), 2)),
                                t(workloads.kv_rows(w, L, 1, int(chunk.sum()), 2)),
                                t(workloads.cu_seqlens(chunk)), t(lengths), pt)
        lens = lengths + chunk
        # the chunk's causal attention
        qc = t(workloads.q_rows_chunk(w, L, int(chunk.sum())))
        b_pre, o_pre = _guarded_like(qc, dev)
        kvq.prefill_attention(cache, L, qc, t(workloads.cu_seqlens(chunk)), t(lens), pt,
                              out=o_pre)
        # decode over the same lengths
        wq = dataclasses.replace(w, batch=B)
        q = t(workloads.q_rows(wq, L))
        b_dec, o_dec = _guarded_like(q, dev)
        kvq.decode_attention(cache, L, q, t(lens), pt, out=o_dec)
        # one more token per sequence, appended inside the decode launch
        b_fus, o_fus = _guarded_like(q, dev)
        kvq.append_decode_attention(cache, L, t(workloads.kv_rows(w, L, 0, B, 3)),
                                    t(workloads.kv_rows(w, L, 1, B, 3)), q, t(lens), pt,
                                    out=o_fus)
        lens = lens + 1
        # the allocation-free decode over the final lengths
        b_na, o_na = _guarded_like(q, dev)
        st_na = torch.zeros(1, dtype=torch.int32, device=dev)
        kvq.decode_attention_noalloc(d, pool, L, q, t(lens), pt, out=o_na, status=st_na)
        torch.cuda.synchronize()
        assert kvq.get_device_status(cache) == 0
        assert int(st_na.item()) == 0
        assert _intact(pbuf), "a kernel wrote outside the pool"
        layer_bytes = nbytes // 2
        assert not bool(pool[:layer_bytes].any().item()), "a kernel wrote into the other layer"
        for name, buf, out in (("prefill", b_pre, o_pre), ("decode", b_dec, o_dec),
                               ("fused", b_fus, o_fus), ("noalloc", b_na, o_na)):
            assert _intact(buf), f"{name}: a kernel wrote outside its output"
            assert bool(torch.isfinite(out).all().item()), name
        # the fused call and the allocation-free decode attend the same cache and lengths
        a, b = o_fus.double(), o_na.double()
        assert bool(((a - b).abs() <= 2e-3 + 1e-2 * b.abs()).all().item())
    finally:
        cache.close()
