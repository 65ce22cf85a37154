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
@pytest.mark.parametrize("page_size", [16, 32, 64, 256])
def test_prefill_group_and_page_size_grid(group, page_size):
    w = dataclasses.replace(W["qwen3_4b_decode"], num_kv_heads=2, num_q_heads=2 * group,
                            page_size=page_size, block=64)
    prefill_parity(make_case(w, [300, 0, 47], [70, 65, 9], permute=True, pool_factor=1.3))


@pytest.mark.parametrize("block", [1, 32])
def test_prefill_blocks_and_softmax_scale(block):
    w = W["ragged"]
    prefill_parity(make_case(w, [200, 5], [33, 64], block=block), softmax_scale=0.05)
