"""GPU parity of causal chunked-prefill attention (kvq_prefill_attention) against the CPU
oracle: a chunk of each sequence's last tokens, already appended, attends the cache
causally.  Covers every GQA group and page size, chunks of 1 token up to whole prompts,
chunk boundaries off the 64-row blocks and 32-token tiles, empty chunks, b = 1 (plain
INT4) and the workloads' value distributions."""
import dataclasses

import pytest

import workloads
from harness import make_case, prefill_parity

pytestmark = pytest.mark.gpu

W = workloads.WORKLOADS


@pytest.mark.parametrize("name,lengths,chunks", [
    ("tiny", [0], [257]),
    ("qwen3_4b_decode", [0, 300, 31, 64, 1000, 7], [100, 17, 1, 65, 16, 0]),
    ("long_context", [2000, 0, 513], [40, 130, 7]),
    ("ragged", [128, 700, 0, 95, 33], [64, 3, 80, 1, 31]),
    ("prefill_append", [0, 0], [300, 129]),
])
def test_prefill_workloads(name, lengths, chunks):
    w = W[name]
    prefill_parity(make_case(w, lengths, chunks))


@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
def test_prefill_group_and_page_size_grid(group, page_size):
    w = dataclasses.replace(W["qwen3_4b_decode"], num_kv_heads=2, num_q_heads=2 * group,
                            page_size=page_size, block=64)
    prefill_parity(make_case(w, [300, 0, 47], [70, 65, 9], permute=True, pool_factor=1.3))


@pytest.mark.parametrize("block", [1, 32])
def test_prefill_blocks_and_softmax_scale(block):
    w = W["ragged"]
    prefill_parity(make_case(w, [200, 5], [33, 64], block=block), softmax_scale=0.05)


def test_prefill_and_fused_bad_inputs_set_status_without_fault():
    """Out-of-range inputs never fault: a chunk longer than its sequence or a length
    beyond the page budget (prefill), a new token past the page budget or on a bad page id
    (fused append + decode) are reported in the status word; the valid sequence of the
    same call still matches the oracle."""
    import numpy as np
    import torch

    import bit_paged_kv_diag_b200 as kvq
    import oracle
    from harness import check_outputs
    w = W["tiny"]
    case = make_case(w, [40, 20], [0, 0])
    d = case.desc()
    pool = torch.zeros(kvq.pool_bytes(d), dtype=torch.uint8, device="cuda")
    cache, pt = kvq.alloc_pages(d, case.capacity, None, pool=pool)
    ptd = torch.from_numpy(pt).cuda()
    k = torch.from_numpy(workloads.kv_rows(w, 0, 0, 60, 1)).cuda()
    v = torch.from_numpy(workloads.kv_rows(w, 0, 1, 60, 1)).cuda()
    kvq.rotate_quant_append(cache, 0, k, v, torch.tensor([0, 40, 60], dtype=torch.int32).cuda(),
                            torch.zeros(2, dtype=torch.int32).cuda(), ptd)
    assert kvq.get_device_status(cache) == 0
    # prefill: sequence 1's chunk (30) is longer than its 20 tokens
    q = torch.from_numpy(workloads.q_rows_chunk(w, 0, 35)).cuda()
    cu = np.array([0, 5, 35], np.int32)
    lens = np.array([40, 20], np.int32)
    out = kvq.prefill_attention(cache, 0, q, torch.from_numpy(cu).cuda(),
                                torch.from_numpy(lens).cuda(), ptd)
    assert kvq.get_device_status(cache) & kvq.KVQ_DEV_BAD_POS
    ref = oracle.prefill_attention(case.geometry(), pool.cpu().numpy(), 0,
                                   q[:5].cpu().numpy(), cu[:2], lens[:1], pt[:1])
    check_outputs(out[:5].float().cpu().numpy(), ref, "valid sequence beside a bad chunk")
    # prefill: a length beyond the page budget
    kvq.prefill_attention(cache, 0, q[:5], torch.tensor([0, 5], dtype=torch.int32).cuda(),
                          torch.tensor([10 ** 6], dtype=torch.int32).cuda(), ptd[:1])
    assert kvq.get_device_status(cache) & kvq.KVQ_DEV_BAD_POS
    assert kvq.get_device_status(cache) == 0
    # fused: sequence 0's new token would land past its page budget; sequence 1's page id
    # is out of range
    bad = pt.copy()
    bad[1, 1] = case.num_pages + 3
    kn = torch.from_numpy(workloads.kv_rows(w, 0, 0, 2, 2)).cuda()
    vn = torch.from_numpy(workloads.kv_rows(w, 0, 1, 2, 2)).cuda()
    qd = torch.from_numpy(workloads.q_rows(dataclasses.replace(w, batch=2), 0)).cuda()
    cap0 = int(case.max_pages_per_seq * w.page_size)
    kvq.append_decode_attention(cache, 0, kn, vn, qd,
                                torch.tensor([cap0, 20], dtype=torch.int32).cuda(),
                                torch.from_numpy(bad).cuda())
    st = kvq.get_device_status(cache)
    assert st & kvq.KVQ_DEV_BAD_POS and st & kvq.KVQ_DEV_BAD_PAGE
    assert kvq.get_device_status(cache) == 0
    cache.close()


@pytest.mark.parametrize("fmt", [0, 1])
def test_prefill_at_the_batch_limit(fmt):
    """4096 sequences (the descriptor's maximum, where the kernel's per-sequence prefix takes
    the most shared memory) of 0..6 cached tokens with chunks of 0..2 tokens."""
    import numpy as np
    rng = np.random.default_rng(4096 + fmt)
    lengths = rng.integers(0, 7, 4096)
    chunks = rng.integers(0, 3, 4096)
    w = dataclasses.replace(W["tiny"], batch=4096)
    prefill_parity(make_case(w, lengths, chunks, max_batch=4096, fmt=fmt))
