"""GPU parity of the NVFP4 cache format (kv_format = 1) against the CPU oracle.

"BitDecoding-FP4:FP4 KVキャッシュのネイティブ復号" (sns.style), sections "背景と概要" and
"深掘り分析": 4-bit microscaling elements (E2M1) with E4M3 block scales.  The same bars
as the INT4 path: page tables and E4M3 scales bit-exact, E2M1 codes exact up to counted
neighbour flips (< 1e-5), decode outputs within |d| <= 2e-3 + 1e-2 |ref| of the fp64 oracle
on the GPU-written cache.  Covered: every workload's heads and value distribution, every
Hadamard block (1 = no rotation), every G and page size, ragged lengths and empty
sequences; the fused one-token append + decode; and causal chunked prefill.
"""
import numpy as np
import pytest

import workloads
from harness import full_parity, make_case

pytestmark = pytest.mark.gpu

W = workloads.WORKLOADS


def test_nvfp4_tiny():
    w = W["tiny"]
    full_parity(make_case(w, w.context, [1], fmt=1))


@pytest.mark.parametrize("name,lengths", [
    ("qwen3_4b_decode", [517, 300, 64, 1, 0, 129, 63, 65]),
    ("long_context", [1000, 2049, 64, 777]),
    ("ragged", [130, 700, 129, 1024, 0, 2, 350, 64, 191, 1500, 17, 33]),
])
def test_nvfp4_scaled_workloads(name, lengths):
    w = W[name]
    full_parity(make_case(w, lengths, [1] * len(lengths), fmt=1))


@pytest.mark.parametrize("block", [1, 32, 64, 128])
def test_nvfp4_prefill_append_student_t(block):
    """Student-t(3) rows, 4 sequences x up to 300 new tokens in one call, then decode."""
    w = W["prefill_append"]
    full_parity(make_case(w, [0, 0, 0, 0], [300, 257, 64, 1], block=block, fmt=1))


@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
def test_nvfp4_group_and_page_size_grid(group, page_size):
    import dataclasses
    w = dataclasses.replace(W["qwen3_4b_decode"], num_kv_heads=2, num_q_heads=2 * group,
                            page_size=page_size, block=64)
    full_parity(make_case(w, [300, 1, 513, 0, 64], [2, 1, 1, 3, 1], permute=True,
                          pool_factor=1.3, fmt=1))


def test_nvfp4_multi_layer_pool_and_custom_softmax_scale():
    """Layer offsets inside a multi-layer NVFP4 pool, and an explicit softmax scale."""
    w = W["ragged"]
    full_parity(make_case(w, [200, 90, 333], [1, 1, 1], layer=2, num_layers=3, fmt=1),
                softmax_scale=0.05)


@pytest.mark.parametrize("name,lengths,block", [
    ("tiny", [256], 32),
    ("qwen3_4b_decode", [517, 300, 64, 1, 0, 129, 63, 65], 128),
    ("ragged", [130, 700, 129, 1024, 0, 2, 350, 64, 191, 1500, 17, 33], 1),
])
def test_nvfp4_fused_append_decode(name, lengths, block):
    """The step's one-token append inside the decode launch, on the NVFP4 cache."""
    w = W[name]
    full_parity(make_case(w, lengths, [1] * len(lengths), block=block, fmt=1), fused=True)


@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("page_size", [16, 32, 64, 256])
def test_nvfp4_fused_group_and_page_size_grid(group, page_size):
    import dataclasses
    w = dataclasses.replace(W["qwen3_4b_decode"], num_kv_heads=2, num_q_heads=2 * group,
                            page_size=page_size, block=64)
    full_parity(make_case(w, [300, 0, 513, 31, 64], [1] * 5, permute=True, pool_factor=1.3,
                          fmt=1), fused=True)


@pytest.mark.parametrize("name,lengths,chunks", [
    ("tiny", [0], [257]),
    ("qwen3_4b_decode", [0, 300, 31, 64, 1000, 7], [100, 17, 1, 65, 16, 0]),
    ("long_context", [2000, 0, 513], [40, 130, 7]),
    ("ragged", [128, 700, 0, 95, 33], [64, 3, 80, 1, 31]),
    ("prefill_append", [0, 0], [300, 129]),
])
def test_nvfp4_prefill_workloads(name, lengths, chunks):
    """Causal chunked prefill over the NVFP4 cache."""
    from harness import prefill_parity
    prefill_parity(make_case(W[name], lengths, chunks, fmt=1))


@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
def test_nvfp4_prefill_group_and_page_size_grid(group, page_size):
    import dataclasses
    from harness import prefill_parity
    w = dataclasses.replace(W["qwen3_4b_decode"], num_kv_heads=2, num_q_heads=2 * group,
                            page_size=page_size, block=64)
    prefill_parity(make_case(w, [300, 0, 47], [70, 65, 9], permute=True, pool_factor=1.3, fmt=1))


@pytest.mark.parametrize("block", [1, 32])
def test_nvfp4_prefill_blocks_and_softmax_scale(block):
    from harness import prefill_parity
    prefill_parity(make_case(W["ragged"], [200, 5], [33, 64], block=block, fmt=1),
                   softmax_scale=0.05)


def _edge_rows(n, H, rng):
    """fp16 rows [n][H][128] whose 16-channel blocks hit the format's edges: saturating
    scales (max |y| / 6 > 448), scales that round to zero or to subnormal E4M3 values, exact
    E2M1 ties (scale 0.5 so that y * (1/s) is exact), signed zeros, all-zero blocks, and
    ordinary Gaussian blocks."""
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float64)
    rows = np.zeros((n, H, 128), np.float64)
    for t in range(n):
        for h in range(H):
            for blk in range(8):
                kind = (t * 7 + h * 3 + blk) % 7
                x = rng.standard_normal(16)
                if kind == 0:      # saturating: up to 60000
                    x = x / np.abs(x).max() * 60000.0
                elif kind == 1:    # max / 6 below half the smallest E4M3 step: scale 0
                    x = x / np.abs(x).max() * 4e-3
                elif kind == 2:    # subnormal E4M3 scale
                    x = x / np.abs(x).max() * 0.05
                elif kind == 3:    # exact ties at scale 0.5 (max = 3)
                    x = np.concatenate([mids * 0.5, -mids * 0.5, [3.0, -0.0]])
                    rng.shuffle(x)
                elif kind == 4:    # all zero, some negative zeros
                    x = np.where(rng.integers(0, 2, 16) == 1, -0.0, 0.0)
                elif kind == 5:    # ties at scale 0.5 plus tiny values rounding to +-0
                    x = np.concatenate([mids * 0.5, [3.0, 0.01, -0.01, 0.1, -0.1, 0.2, -0.2, 0.12, -0.12]])
                rows[t, h, 16 * blk:16 * blk + 16] = x
    return rows.astype(np.float16)


@pytest.mark.parametrize("block", [1, 32])
def test_nvfp4_edge_rows(block):
    """Constructed rows through append and decode: the pool must equal the oracle's byte for
    byte (ties, saturation, zero and subnormal scales, signed zeros), outputs within the
    tolerance of the fp64 oracle on that pool."""
    import torch

    import bit_paged_kv_diag_b200 as kvq
    import oracle
    from harness import check_outputs
    rng = np.random.default_rng(31)
    H, HQ, S, L = 2, 8, 16, 77
    k = _edge_rows(L, H, rng)
    v = _edge_rows(L, H, rng)
    P = 8
    d = kvq.Desc(1, H, HQ, 128, block, S, P, 1, P, kvq.FORMAT_NVFP4)
    dev = torch.device("cuda")
    pool = torch.zeros(kvq.pool_bytes(d), dtype=torch.uint8, device=dev)
    cap = np.array([L], np.int32)
    cache, pt = kvq.alloc_pages(d, cap, None, pool=pool)
    try:
        ptd = torch.from_numpy(pt).to(dev)
        kvq.rotate_quant_append(cache, 0, torch.from_numpy(k).to(dev), torch.from_numpy(v).to(dev),
                                torch.tensor([0, L], dtype=torch.int32, device=dev),
                                torch.zeros(1, dtype=torch.int32, device=dev), ptd)
        q = rng.standard_normal((1, HQ, 128)).astype(np.float16)
        out = kvq.decode_attention(cache, 0, torch.from_numpy(q).to(dev),
                                   torch.from_numpy(cap).to(dev), ptd)
        torch.cuda.synchronize()
        assert kvq.get_device_status(cache) == 0
        gpool = pool.cpu().numpy()
        gout = out.float().cpu().numpy()
    finally:
        cache.close()
    g = oracle.Geometry(1, H, HQ, 128, block, S, P, P, fmt=1)
    ref_pool = g.new_pool()
    oracle.rotate_quant_append(g, ref_pool, 0, k, v, np.array([0, L], np.int32),
                               np.array([0], np.int32), pt)
    diff = np.nonzero(gpool != ref_pool)[0]
    assert diff.size == 0, f"{diff.size} pool bytes differ, first at {diff[:8]}"
    ref = oracle.decode_attention(g, gpool, 0, q, cap, pt)
    check_outputs(gout, ref, f"nvfp4 edge rows b={block}")


def test_nvfp4_nan_bytes_past_the_end_do_not_leak():
    """A pool pre-filled with 0x7F bytes (E4M3 NaN): slots past each sequence's end keep
    NaN scales, which must not reach the outputs (their probabilities are zero)."""
    import torch

    import bit_paged_kv_diag_b200 as kvq
    import oracle
    from harness import check_outputs
    w = W["qwen3_4b_decode"]
    lengths = np.array([37, 1, 100, 16, 17], np.int32)
    case = make_case(w, lengths, [0] * len(lengths), fmt=1)
    dev = torch.device("cuda")
    d = case.desc()
    pool = torch.full((kvq.pool_bytes(d),), 0x7F, dtype=torch.uint8, device=dev)
    cache, pt = kvq.alloc_pages(d, case.capacity, case.page_order, pool=pool)
    try:
        ptd = torch.from_numpy(pt).to(dev)
        n = int(lengths.sum())
        k = workloads.kv_rows(w, 0, 0, n, stream=1)
        v = workloads.kv_rows(w, 0, 1, n, stream=1)
        kvq.rotate_quant_append(cache, 0, torch.from_numpy(k).to(dev), torch.from_numpy(v).to(dev),
                                torch.from_numpy(workloads.cu_seqlens(lengths)).to(dev),
                                torch.zeros(len(lengths), dtype=torch.int32, device=dev), ptd)
        q = workloads.q_rows(dataclasses_replace(w, batch=len(lengths)), 0)
        out = kvq.decode_attention(cache, 0, torch.from_numpy(q).to(dev),
                                   torch.from_numpy(lengths).to(dev), ptd)
        torch.cuda.synchronize()
        assert kvq.get_device_status(cache) == 0
        host_pool = pool.cpu().numpy()
        got = out.float().cpu().numpy()
    finally:
        cache.close()
    assert np.isfinite(got).all()
    ref = oracle.decode_attention(case.geometry(), host_pool, 0, q, lengths, pt)
    check_outputs(got, ref, "nvfp4 with NaN bytes past the end")


def dataclasses_replace(w, **kw):
    import dataclasses
    return dataclasses.replace(w, **kw)
