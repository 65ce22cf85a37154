"""The allocation-free decode entry point against the handle-based one and the oracle (GPU).

kvq_decode_attention_noalloc serves callers that cannot call cudaMalloc -- a runtime that
owns all of device memory, a plugin whose host framework does every allocation, or a path
that cannot afford cudaMalloc's implicit synchronisation.  It runs the same decode kernel
with its scratch in a fixed device array inside the library, so its output must equal the
handle-based decode's bit for bit (the kernel is deterministic) and the CPU oracle's within
the decode tolerance.  This file is collected last, so a run that stops at the first
failure has already run every other test; it passes both alone in a fresh process and after
the others (the array keeps its state between calls).
"""
import ctypes

import numpy as np
import pytest

import oracle
import workloads
from harness import CudaRun, check_outputs, host_inputs, make_case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,lengths,fmt", [
    ("long_context", [5000, 31, 1, 2600], 0),    # units split over many CTAs, and short ones
    ("qwen3_4b_decode", [517, 300, 64, 1, 0, 129, 63, 65], 0),
    ("qwen3_4b_decode", [517, 300, 64, 1, 0, 129, 63, 65], 1),   # NVFP4 cache
])
def test_noalloc_decode_matches_handle_decode_twice(name, lengths, fmt):
    import torch
    import bit_paged_kv_diag_b200 as kvq
    w = workloads.WORKLOADS[name]
    case = make_case(w, lengths, [1] * len(lengths), fmt=fmt)
    kp, vp, kn, vn, q = host_inputs(case)
    run = CudaRun(case, kp, vp, kn, vn, q)
    try:
        d = case.desc()
        qd = torch.as_tensor(q).cuda()
        lens = torch.as_tensor(run.lens_after).cuda()
        pt = torch.from_numpy(run.page_table).cuda()
        ref = oracle.decode_attention(case.geometry(), run.host_pool, case.layer, q,
                                      run.lens_after, run.page_table)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        for _ in range(2):   # two calls in a row on the shared scratch
            out = torch.full_like(qd, float("nan"))
            stream = torch.cuda.current_stream().cuda_stream
            rc = kvq.lib().kvq_decode_attention_noalloc(
                ctypes.byref(d), run.pool.data_ptr(), run.pool.numel(), case.layer,
                qd.data_ptr(), lens.data_ptr(), pt.data_ptr(), len(lengths), ctypes.c_float(0.0),
                out.data_ptr(), status.data_ptr(), stream)
            assert rc == kvq.KVQ_OK, kvq.status_string(rc)
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            assert torch.equal(out, run.out), "differs from the handle-based decode"
            check_outputs(out.float().cpu().numpy(), ref, "allocation-free decode")
    finally:
        run.close()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Both limits of the fixed array: the unit counters (batch * Hkv <= 4096) and the
    partial records ((batch * Hkv + grid) * G <= 4096), each answered before any launch."""
    import torch
    import bit_paged_kv_diag_b200 as kvq
    stream = torch.cuda.current_stream().cuda_stream
    for batch, hkv, hq in [(4096, 8, 32),     # 32768 units: beyond the counter array
                           (128, 8, 32)]:     # 1024 units, (1024 + grid) * 4 > 4096 records
        d = kvq.Desc(1, hkv, hq, 128, 128, 16, 8192, batch, 4)
        pool = torch.zeros(kvq.pool_bytes(d), dtype=torch.uint8, device="cuda")
        z = torch.zeros(batch * hq * 128, dtype=torch.float16, device="cuda")
        lens = torch.ones(batch, dtype=torch.int32, device="cuda")
        pt = torch.zeros(batch * 4, dtype=torch.int32, device="cuda")
        rc = kvq.lib().kvq_decode_attention_noalloc(
            ctypes.byref(d), pool.data_ptr(), pool.numel(), 0, z.data_ptr(), lens.data_ptr(),
            pt.data_ptr(), batch, ctypes.c_float(0.0), z.data_ptr(), None, stream)
        assert rc == kvq.KVQ_EUNSUPPORTED, (batch, rc)
        del pool


def test_noalloc_rejects_a_pool_smaller_than_its_descriptor():
    import torch
    import bit_paged_kv_diag_b200 as kvq
    d = kvq.Desc(2, 8, 32, 128, 128, 16, 64, 4, 16)
    pool = torch.zeros(kvq.pool_bytes(d) // 2, dtype=torch.uint8, device="cuda")  # one layer
    q = torch.zeros(4, 32, 128, dtype=torch.float16, device="cuda")
    lens = torch.ones(4, dtype=torch.int32, device="cuda")
    pt = torch.from_numpy(kvq.assign_pages(d, np.full(4, 16 * 16, np.int32))).cuda()
    with pytest.raises(kvq.KVQError) as e:
        kvq.decode_attention_noalloc(d, pool, 1, q, lens, pt)
    assert e.value.status == kvq.KVQ_EINVAL
