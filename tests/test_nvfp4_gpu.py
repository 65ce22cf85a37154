"""GPU parity of the NVFP4 cache format (kv_format = 1) against the CPU oracle.

"BitDecoding-FP4:FP4 KVキャッシュのネイティブ復号" (sns.style), sections "背景と概要" and
"深掘り分析": 4-bit microscaling elements (E2M1) with E4M3 block scales.  The same bars
as the INT4 path: page tables and E4M3 scales bit-exact, E2M1 codes exact up to counted
neighbour flips (< 1e-5), decode outputs within |d| <= 2e-3 + 1e-2 |ref| of the fp64 oracle
on the GPU-written cache.  Covered: every workload's heads and value distribution, every
Hadamard block (1 = no rotation), every G and page size, ragged lengths and empty
sequences; and the calls NVFP4 does not implement return KVQ_EUNSUPPORTED.
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


def test_nvfp4_unsupported_calls():
    import torch

    import bit_paged_kv_diag_b200 as kvq
    w = W["tiny"]
    case = make_case(w, w.context, [1], fmt=1)
    dev = torch.device("cuda")
    cache, pt = kvq.alloc_pages(case.desc(), case.capacity, case.page_order)
    try:
        ptd = torch.from_numpy(pt).to(dev)
        H, HQ = w.num_kv_heads, w.num_q_heads
        kn = torch.zeros((1, H, 128), dtype=torch.float16, device=dev)
        q = torch.zeros((1, HQ, 128), dtype=torch.float16, device=dev)
        lens = torch.tensor([256], dtype=torch.int32, device=dev)
        with pytest.raises(kvq.KVQError) as e:
            kvq.append_decode_attention(cache, 0, kn, kn, q, lens, ptd)
        assert e.value.status == kvq.KVQ_EUNSUPPORTED
        with pytest.raises(kvq.KVQError) as e:
            kvq.prefill_attention(cache, 0, q, torch.tensor([0, 1], dtype=torch.int32, device=dev),
                                  lens, ptd)
        assert e.value.status == kvq.KVQ_EUNSUPPORTED
    finally:
        cache.close()
