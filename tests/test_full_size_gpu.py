"""Parity at the workloads' full sizes, on samples the oracle computes one by one.

The long-context (4 sequences up to 131072 tokens, G = 8, b = 64, page 64), ragged (256
sequences of 128..8192 tokens, pages scattered through a 1.2x pool) and prefill-append
(8 x 8192 new tokens in one call, Student-t(3), every b) workloads run through the C ABI
at full size, with inputs drawn on the device by the seeded generators.  Checked:

* the page table, bit-exact against the oracle's allocator (whole table);
* appended rows: for a seeded sample of (token, KV head, K|V) rows, the oracle's rotation,
  scale and codes of the same input row against the bytes the kernel wrote at the row's
  page and slot (scale bit-exact, codes exact up to counted +-1 flips; for the NVFP4
  format the 8 E4M3 scales and the E2M1 codes);
* decode outputs: for a few whole sequences (the longest, the shortest, one more), the
  fp64 oracle over the GPU-written cache against the kernel's fp16 output rows, within
  |d| <= 2e-3 + 1e-2 |ref|.
"""
import dataclasses

import numpy as np
import pytest

import oracle
import workloads
from harness import check_outputs

pytestmark = pytest.mark.gpu

W = workloads.WORKLOADS
ROW_SAMPLES = 1500


def _run_full(w, block, fmt=0):
    """Prefill every cached token, append the step's tokens, decode; returns host views."""
    import torch

    import bit_paged_kv_diag_b200 as kvq
    dev = torch.device("cuda")
    lengths = workloads.context_lengths(w)
    new = np.full(w.batch, w.new_tokens, np.int32)
    cap = lengths + new
    S, H = w.page_size, w.num_kv_heads
    P = workloads.pool_pages(w, cap)
    order = workloads.page_order(w, P)
    mp = int((cap.max() + S - 1) // S)
    desc = kvq.Desc(1, H, w.num_q_heads, 128, block, S, P, w.batch, mp, fmt)
    pool = torch.zeros(kvq.pool_bytes(desc), dtype=torch.uint8, device=dev)
    cache, pt = kvq.alloc_pages(desc, cap, order, pool=pool)
    ptd = torch.from_numpy(pt).to(dev)
    npre, nnew = int(lengths.sum()), int(new.sum())
    rows = {}
    if npre:
        rows["pre"] = (workloads.kv_rows_torch(w, 0, 0, npre, stream=1, device=dev),
                       workloads.kv_rows_torch(w, 0, 1, npre, stream=1, device=dev),
                       workloads.cu_seqlens(lengths), np.zeros(w.batch, np.int32))
    rows["new"] = (workloads.kv_rows_torch(w, 0, 0, nnew, stream=2, device=dev),
                   workloads.kv_rows_torch(w, 0, 1, nnew, stream=2, device=dev),
                   workloads.cu_seqlens(new), lengths)
    for k, v, cu, before in rows.values():
        kvq.rotate_quant_append(cache, 0, k, v, torch.from_numpy(cu).to(dev),
                                torch.from_numpy(before).to(dev), ptd)
    q = workloads.q_rows_torch(w, 0, device=dev)
    out = kvq.decode_attention(cache, 0, q, torch.from_numpy(cap).to(dev), ptd)
    torch.cuda.synchronize()
    status = kvq.get_device_status(cache)
    res = dict(lengths=lengths, cap=cap, P=P, order=order, mp=mp, page_table=pt,
               pool=pool.cpu().numpy(), q=q.cpu().numpy(), out=out.float().cpu().numpy(),
               rows=rows, status=status)
    cache.close()
    return res


def _check_rows(w, block, r, rng, fmt=0):
    """Sampled appended rows against the oracle's rotation + quantisation of the same row."""
    S, H = w.page_size, w.num_kv_heads
    blk = oracle.block_bytes(S, 128, fmt)
    flips = total = 0
    for name, (k, v, cu, before) in r["rows"].items():
        n = k.shape[0]
        take = rng.integers(0, n, size=min(ROW_SAMPLES, n))
        heads = rng.integers(0, H, size=take.size)
        kvs = rng.integers(0, 2, size=take.size)
        import torch
        idx = torch.as_tensor(take, device=k.device)
        ks, vs = k[idx].cpu().numpy(), v[idx].cpu().numpy()
        for i, t in enumerate(take):
            b = int(np.searchsorted(cu, t, side="right") - 1)
            pos = int(before[b]) + int(t - cu[b])
            page = int(r["page_table"][b, pos // S])
            slot = pos % S
            h, kv = int(heads[i]), int(kvs[i])
            x = (vs if kv else ks)[i, h].astype(np.float32)
            base = (page * H + h) * blk
            packed = r["pool"][base + kv * S * 64 + slot * 64:][:64]
            if fmt == 1:
                codes, scales = oracle.quant_row_nvfp4(oracle.fwht_f32(x, block))
                got_scales = r["pool"][base + S * 128 + kv * S * 8 + slot * 8:][:8]
                assert np.array_equal(got_scales, scales), (name, int(t), h, kv)
                got = np.stack([packed & 0xF, packed >> 4], 1).reshape(-1)
                same = (got & 8) == (codes & 8)
                d = np.where(got == codes, 0, np.where(same, np.abs((got & 7).astype(np.int16) -
                                                                   (codes & 7).astype(np.int16)), 99))
                assert d.max() <= 1, (name, int(t), h, kv)
                flips += int(np.count_nonzero(d))
                total += 128
                continue
            bits, codes = oracle.quant_row(oracle.fwht_f32(x, block))
            got_scale = int(r["pool"][base + S * 128 + kv * S * 2 + slot * 2:][:2].view(np.uint16)[0])
            assert got_scale == bits, (name, int(t), h, kv, got_scale, bits)
            got = oracle.unpack_codes(packed, 128)
            d = np.abs(got.astype(np.int16) - codes.astype(np.int16))
            assert d.max() <= 1, (name, int(t), h, kv)
            flips += int(np.count_nonzero(d))
            total += 128
    assert flips <= max(1, 1e-5 * total), f"{flips} +-1 flips in {total} sampled codes"


def _check_decode(w, block, r, seqs, fmt=0):
    g = oracle.Geometry(1, w.num_kv_heads, w.num_q_heads, 128, block, w.page_size, r["P"],
                        r["mp"], fmt)
    for b in seqs:
        ref = oracle.decode_attention(g, r["pool"], 0, r["q"][b:b + 1], r["cap"][b:b + 1],
                                      r["page_table"][b:b + 1])
        check_outputs(r["out"][b:b + 1], ref, f"{w.name} sequence {b}")


def _full_size_parity(w, block, seed, fmt=0):
    r = _run_full(w, block, fmt)
    assert r["status"] == 0, f"device status {r['status']}"
    pt_ref = oracle.assign_pages(r["cap"], w.page_size, r["P"], r["mp"], r["order"])
    assert np.array_equal(r["page_table"], pt_ref), "page table differs from the oracle's"
    rng = np.random.default_rng(seed)
    _check_rows(w, block, r, rng, fmt)
    cap = r["cap"]
    seqs = sorted({int(np.argmax(cap)), int(np.argmin(cap)), int(rng.integers(0, len(cap)))})
    _check_decode(w, block, r, seqs, fmt)


def test_long_context_full_size():
    """4 sequences of 32K / 64K / 128K / 128K tokens, G = 8, b = 64, page 64."""
    w = W["long_context"]
    _full_size_parity(w, w.block, 101)


def test_ragged_full_size():
    """256 sequences of U{128..8192} tokens, pages scattered through a 1.2x pool."""
    w = W["ragged"]
    _full_size_parity(w, w.block, 102)


@pytest.mark.parametrize("block", [1, 32, 64, 128])
def test_prefill_append_full_size(block):
    """8 x 8192 new tokens in one append call, then decode over them (b = 1 is plain INT4)."""
    w = W["prefill_append"]
    _full_size_parity(w, block, 103 + block)


def test_nvfp4_ragged_full_size():
    """The NVFP4 cache on the ragged workload at full size (256 sequences, scattered pages)."""
    w = W["ragged"]
    _full_size_parity(w, w.block, 202, fmt=1)


def test_nvfp4_prefill_append_full_size():
    """8 x 8192 new tokens into an NVFP4 cache in one call, then decode (b = 128)."""
    _full_size_parity(W["prefill_append"], 128, 203, fmt=1)


@pytest.mark.parametrize("fmt", [0, 1])
def test_chunked_prefill_full_size(fmt):
    """16 sequences x a 512-token chunk after 3584 cached tokens (one layer), on the INT4
    and the NVFP4 cache: sampled query rows of the chunk against the oracle (query i of a
    chunk is the one query of a chunk of length 1 over the first L - C + i + 1 tokens)."""
    import torch

    import bit_paged_kv_diag_b200 as kvq
    w = W["chunked_prefill"]
    dev = torch.device("cuda")
    L0 = workloads.context_lengths(w)
    chunk = np.full(w.batch, w.new_tokens, np.int32)
    cap = L0 + chunk
    S, H = w.page_size, w.num_kv_heads
    P = workloads.pool_pages(w, cap)
    mp = int((cap.max() + S - 1) // S)
    desc = kvq.Desc(1, H, w.num_q_heads, 128, w.block, S, P, w.batch, mp, fmt)
    pool = torch.zeros(kvq.pool_bytes(desc), dtype=torch.uint8, device=dev)
    cache, pt = kvq.alloc_pages(desc, cap, None, pool=pool)
    ptd = torch.from_numpy(pt).to(dev)
    k = workloads.kv_rows_torch(w, 0, 0, int(cap.sum()), stream=1, device=dev)
    v = workloads.kv_rows_torch(w, 0, 1, int(cap.sum()), stream=1, device=dev)
    kvq.rotate_quant_append(cache, 0, k, v, torch.from_numpy(workloads.cu_seqlens(cap)).to(dev),
                            torch.zeros(w.batch, dtype=torch.int32, device=dev), ptd)
    cu_q = workloads.cu_seqlens(chunk)
    q = workloads.q_rows_chunk(w, 0, int(cu_q[-1]))
    out = kvq.prefill_attention(cache, 0, torch.from_numpy(q).to(dev),
                                torch.from_numpy(cu_q).to(dev), torch.from_numpy(cap).to(dev), ptd)
    torch.cuda.synchronize()
    assert kvq.get_device_status(cache) == 0
    host_pool = pool.cpu().numpy()
    host_out = out.float().cpu().numpy()
    cache.close()
    g = oracle.Geometry(1, H, w.num_q_heads, 128, w.block, S, P, mp, fmt)
    rng = np.random.default_rng(104 + fmt)
    for b in rng.choice(w.batch, 3, replace=False):
        for i in sorted({0, int(chunk[b]) - 1, *rng.integers(0, int(chunk[b]), 4).tolist()}):
            row = int(cu_q[b]) + i
            pos = int(cap[b] - chunk[b]) + i
            ref = oracle.prefill_attention(g, host_pool, 0, q[row:row + 1], np.array([0, 1], np.int32),
                                           np.array([pos + 1], np.int32), pt[b:b + 1])
            check_outputs(host_out[row:row + 1], ref, f"chunked prefill fmt={fmt} b={b} i={i}")


@pytest.mark.parametrize("fmt", [0, 1])
def test_chunked_prefill_long_context(fmt):
    """The long-context shape (4 KV / 32 query heads, G = 8, page 64, b = 64): a 256-token
    chunk after 32 512 and after 65 280 cached tokens, so a CTA walks up to 512 KV tiles
    and its softmax frame moves across hundreds of them; sampled query rows against the
    oracle."""
    import torch

    import bit_paged_kv_diag_b200 as kvq
    w = W["long_context"]
    dev = torch.device("cuda")
    chunk = np.array([256, 256], np.int32)
    cap = np.array([32768, 65536], np.int32)
    S, H, B = w.page_size, w.num_kv_heads, len(cap)
    P = int(((cap + S - 1) // S).sum())
    mp = int((cap.max() + S - 1) // S)
    desc = kvq.Desc(1, H, w.num_q_heads, 128, w.block, S, P, B, mp, fmt)
    pool = torch.zeros(kvq.pool_bytes(desc), dtype=torch.uint8, device=dev)
    cache, pt = kvq.alloc_pages(desc, cap, None, pool=pool)
    ptd = torch.from_numpy(pt).to(dev)
    k = workloads.kv_rows_torch(w, 0, 0, int(cap.sum()), stream=1, device=dev)
    v = workloads.kv_rows_torch(w, 0, 1, int(cap.sum()), stream=1, device=dev)
    kvq.rotate_quant_append(cache, 0, k, v, torch.from_numpy(workloads.cu_seqlens(cap)).to(dev),
                            torch.zeros(B, dtype=torch.int32, device=dev), ptd)
    del k, v
    cu_q = workloads.cu_seqlens(chunk)
    q = workloads.q_rows_chunk(w, 0, int(cu_q[-1]))
    out = kvq.prefill_attention(cache, 0, torch.from_numpy(q).to(dev),
                                torch.from_numpy(cu_q).to(dev), torch.from_numpy(cap).to(dev), ptd)
    torch.cuda.synchronize()
    assert kvq.get_device_status(cache) == 0
    host_pool = pool.cpu().numpy()
    host_out = out.float().cpu().numpy()
    cache.close()
    g = oracle.Geometry(1, H, w.num_q_heads, 128, w.block, S, P, mp, fmt)
    rng = np.random.default_rng(204 + fmt)
    for b in range(B):
        for i in sorted({0, int(chunk[b]) - 1, *rng.integers(0, int(chunk[b]), 3).tolist()}):
            row = int(cu_q[b]) + i
            pos = int(cap[b] - chunk[b]) + i
            ref = oracle.prefill_attention(g, host_pool, 0, q[row:row + 1], np.array([0, 1], np.int32),
                                           np.array([pos + 1], np.int32), pt[b:b + 1])
            check_outputs(host_out[row:row + 1], ref, f"long-context prefill fmt={fmt} b={b} i={i}")
