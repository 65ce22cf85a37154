"""The bench's algorithmic byte counts (the numerator of every reported GB/s and roofline
fraction) against the pool layout and the workloads' sizes.

Per (token, KV head) the decode streams one cache row: the oracle's block size over the
page size (64 B K codes + 64 B V codes + the two rows' scales).  A decode launch also
reads the page-table entries of every live page and q, and writes out (fp16, 128 channels
per query head).  An append reads the fp16 K and V rows (2 x 256 B) and writes one cache
row per (token, KV head)."""
import numpy as np

import bench
import oracle
import workloads


def test_bytes_per_row_follow_the_pool_layout():
    assert bench.BYTES_PER_TOKEN_HEAD == oracle.block_bytes(16, 128, 0) // 16 == 132
    assert bench.BYTES_PER_TOKEN_HEAD_NVFP4 == oracle.block_bytes(16, 128, 1) // 16 == 144


def test_decode_bytes_of_the_qwen3_4b_layer():
    w = workloads.WORKLOADS["qwen3_4b_decode"]
    lens = np.asarray(w.context, np.int64) + w.new_tokens      # 16 x 4097 after the append
    pages = sum(-(-int(n) // w.page_size) for n in lens)          # 16 x 257
    want = (int(lens.sum()) * w.num_kv_heads * 132 + 4 * pages
            + 2 * w.batch * w.num_q_heads * 128 * 2)
    assert want == 69_501_504
    assert bench.decode_bytes(lens, w.num_kv_heads, w.num_q_heads, w.page_size) == want
    nv = bench.decode_bytes(lens, w.num_kv_heads, w.num_q_heads, w.page_size,
                            bench.BYTES_PER_TOKEN_HEAD_NVFP4)
    assert nv - want == int(lens.sum()) * w.num_kv_heads * (144 - 132)


def test_decode_bytes_edge_cases():
    # empty sequences read no cache and no page, but their q and out rows count
    assert bench.decode_bytes([0, 0], 2, 8, 16) == 2 * 2 * 8 * 128 * 2
    # one token: one row per KV head and one page-table entry
    assert bench.decode_bytes([1], 2, 8, 16) == 2 * 132 + 4 + 2 * 8 * 128 * 2
    # a page boundary: 17 tokens use two pages
    assert bench.decode_bytes([17], 1, 1, 16) - bench.decode_bytes([16], 1, 1, 16) == 132 + 4


def test_append_bytes_of_the_prefill_append_workload():
    w = workloads.WORKLOADS["prefill_append"]
    T = w.batch * w.new_tokens
    assert bench.append_bytes(T, w.num_kv_heads) == T * w.num_kv_heads * (2 * 128 * 2 + 132)
    assert bench.append_bytes(T, w.num_kv_heads) == 337_641_472
    assert bench.append_bytes(T, w.num_kv_heads, 144) - bench.append_bytes(T, w.num_kv_heads) \
        == T * w.num_kv_heads * 12
