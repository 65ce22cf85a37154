"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle.

Sizes here are ones the oracle finishes in seconds yet span several 64-token tiles, several
pages and ragged tails; every workload's heads / GQA group / Hadamard block / page size /
value distribution is covered, plus the degenerate cases (empty sequences, one token,
lengths on and off tile and page boundaries, every supported G, S and b).

Acceptance: page tables and scales bit-exact, codes exact up to counted +-1 flips
(< 1e-5), outputs within |d| <= 2e-3 + 1e-2 |ref| of the fp64 oracle run on the same
GPU-written cache.
"""
import dataclasses

import numpy as np
import pytest

import workloads
from harness import full_parity, make_case

pytestmark = pytest.mark.gpu

W = workloads.WORKLOADS


def test_tiny_workload_exact():
    """The tiny workload at its full size: 256 cached tokens, append 1, decode."""
    w = W["tiny"]
    r = full_parity(make_case(w, w.context, [1]))
    assert r["flips"] == 0


@pytest.mark.parametrize("name,lengths", [
    ("qwen3_4b_decode", [517, 300, 64, 1, 0, 129, 63, 65]),
    ("long_context", [1000, 2049, 64, 777]),
    ("ragged", [130, 700, 129, 1024, 0, 2, 350, 64, 191, 1500, 17, 33]),
])
def test_scaled_workloads(name, lengths):
    w = W[name]
    new = [1] * len(lengths)
    r = full_parity(make_case(w, lengths, new))
    assert r["flips"] == 0


@pytest.mark.parametrize("block", [32, 64, 128])
def test_prefill_append_student_t(block):
    """Student-t(3) rows, 4 sequences x 300 new tokens appended in one call, then decode."""
    w = W["prefill_append"]
    full_parity(make_case(w, [0, 0, 0, 0], [300, 257, 64, 1], block=block))


@pytest.mark.parametrize("name,lengths", [
    ("qwen3_4b_decode", [517, 300, 64, 1, 0, 129, 63, 65]),
    ("long_context", [1000, 2049, 64, 777]),
])
def test_plain_int4_variant(name, lengths):
    """b = 1: the same kernels without the rotation (plain token-wise INT4)."""
    w = W[name]
    r = full_parity(make_case(w, lengths, [1] * len(lengths), block=1))
    assert r["flips"] == 0


def test_plain_int4_prefill_student_t():
    w = W["prefill_append"]
    full_parity(make_case(w, [0, 0, 0, 0], [300, 257, 64, 1], block=1))


@pytest.mark.parametrize("name,lengths,block", [
    ("tiny", [256], None),
    ("qwen3_4b_decode", [517, 300, 64, 1, 0, 129, 63, 65, 31, 32, 33, 4095], None),
    ("long_context", [1000, 2049, 64, 777], None),
    ("ragged", [130, 700, 129, 1024, 0, 2, 350, 64, 191, 1500, 17, 33], None),
    ("ragged", [130, 700, 0, 95], 1),
])
def test_fused_append_decode(name, lengths, block):
    """kvq_append_decode_attention: the pool gets exactly the oracle's append of the new
    token (bit-exact, whole pool) and the outputs match the oracle's decode over it; the
    new token lands on tile and page boundaries and in empty sequences."""
    w = W[name]
    r = full_parity(make_case(w, lengths, [1] * len(lengths), block=block), fused=True)
    assert r["flips"] == 0


@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
def test_fused_group_and_page_size_grid(group, page_size):
    w = dataclasses.replace(W["qwen3_4b_decode"], num_kv_heads=2, num_q_heads=2 * group,
                            page_size=page_size, block=64)
    full_parity(make_case(w, [300, 0, 513, 31, 64], [1] * 5, permute=True, pool_factor=1.3),
                fused=True)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("kv_heads", [3, 5])
def test_kv_heads_not_a_power_of_two(kv_heads, fmt):
    """3 and 5 KV heads (G = 4): the append's split of its (token, KV head) pairs and the
    decode's units, with multi-token appends after cached tokens, on both cache formats."""
    w = dataclasses.replace(W["qwen3_4b_decode"], num_kv_heads=kv_heads,
                            num_q_heads=4 * kv_heads)
    full_parity(make_case(w, [300, 1, 513, 0, 64], [37, 1, 200, 3, 9], permute=True,
                          pool_factor=1.3, fmt=fmt))


@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
def test_group_and_page_size_grid(group, page_size):
    w = dataclasses.replace(W["qwen3_4b_decode"], num_kv_heads=2, num_q_heads=2 * group,
                            page_size=page_size, block=64)
    full_parity(make_case(w, [300, 1, 513, 0, 64], [2, 1, 1, 3, 1], permute=True,
                          pool_factor=1.3))


def test_qwen_shape_one_layer_full_size():
    """Qwen3-4B-shaped layer at full size (16 x 4096 cached tokens, append 1, decode)."""
    w = W["qwen3_4b_decode"]
    full_parity(make_case(w, w.context, [1] * w.batch))


def test_multi_layer_pool_and_custom_softmax_scale():
    """Layer offsets inside a multi-layer pool, and an explicit softmax scale."""
    w = W["ragged"]
    case = make_case(w, [200, 90, 333], [1, 1, 1], layer=2, num_layers=3)
    full_parity(case, softmax_scale=0.05)


def test_bad_page_id_sets_status_without_fault():
    """A page-table entry outside the pool is never dereferenced: the append skips it,
    the decode redirects it, and the device status word reports it."""
    import torch
    import bit_paged_kv_diag_b200 as kvq
    w = W["tiny"]
    case = make_case(w, [40], [0])
    d = case.desc()
    pool = torch.zeros(kvq.pool_bytes(d), dtype=torch.uint8, device="cuda")
    cache, pt = kvq.alloc_pages(d, case.capacity, None, pool=pool)
    bad = pt.copy()
    bad[0, 1] = case.num_pages + 5
    ptd = torch.from_numpy(bad).cuda()
    k = torch.randn(40, 2, 128, device="cuda").half()
    lens0 = torch.zeros(1, dtype=torch.int32, device="cuda")
    cu = torch.tensor([0, 40], dtype=torch.int32, device="cuda")
    kvq.rotate_quant_append(cache, 0, k, k, cu, lens0, ptd)
    assert kvq.get_device_status(cache) & kvq.KVQ_DEV_BAD_PAGE
    q = torch.randn(1, 8, 128, device="cuda").half()
    kvq.decode_attention(cache, 0, q, torch.tensor([40], dtype=torch.int32, device="cuda"), ptd)
    assert kvq.get_device_status(cache) & kvq.KVQ_DEV_BAD_PAGE
    # a length beyond the sequence's page budget is clamped and reported
    kvq.decode_attention(cache, 0, q, torch.tensor([10 ** 6], dtype=torch.int32, device="cuda"),
                         torch.from_numpy(pt).cuda())
    assert kvq.get_device_status(cache) & kvq.KVQ_DEV_BAD_POS
    assert kvq.get_device_status(cache) == 0
    cache.close()


def test_empty_batch_calls_are_no_ops():
    import torch
    import bit_paged_kv_diag_b200 as kvq
    w = W["tiny"]
    case = make_case(w, [0], [0])
    cache, pt = kvq.alloc_pages(case.desc(), case.capacity, None)
    e = torch.zeros(0, 2, 128, dtype=torch.float16, device="cuda")
    z = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.rotate_quant_append(cache, 0, e, e, torch.zeros(2, dtype=torch.int32, device="cuda"), z,
                            torch.from_numpy(pt).cuda())
    out = kvq.decode_attention(cache, 0, torch.ones(1, 8, 128, dtype=torch.float16, device="cuda"),
                               z, torch.from_numpy(pt).cuda())
    torch.cuda.synchronize()
    assert not out.any()
    assert kvq.get_device_status(cache) == 0
    cache.close()


def test_repeated_decode_is_bit_identical():
    """The cross-CTA merge counters reset themselves: the same call twice gives the same
    bytes (long units split over many CTAs, plus short ones finished inside one CTA)."""
    import torch
    import bit_paged_kv_diag_b200 as kvq
    w = W["long_context"]
    case = make_case(w, [5000, 31, 1, 2600], [1, 1, 1, 1])
    from harness import CudaRun, host_inputs
    kp, vp, kn, vn, q = host_inputs(case)
    run = CudaRun(case, kp, vp, kn, vn, q)
    try:
        pt = torch.from_numpy(run.page_table).cuda()
        lens = torch.as_tensor(run.lens_after).cuda()
        qd = torch.as_tensor(q).cuda()
        a = kvq.decode_attention(run.cache, 0, qd, lens, pt)
        b = kvq.decode_attention(run.cache, 0, qd, lens, pt)
        torch.cuda.synchronize()
        assert torch.equal(a, b)
        assert torch.equal(a.float().cpu(), torch.from_numpy(run.host_out))
        assert kvq.get_device_status(run.cache) == 0
    finally:
        run.close()


def test_many_short_units_per_cta():
    """Hundreds of sequences of 1..40 tokens: many units inside one CTA's range."""
    w = dataclasses.replace(W["ragged"], num_kv_heads=2, num_q_heads=8)
    rng = np.random.default_rng(5)
    lengths = rng.integers(0, 40, size=300).tolist()
    full_parity(make_case(w, lengths, [1] * 300, pool_factor=1.1))
