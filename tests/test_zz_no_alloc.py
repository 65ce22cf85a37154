"""The allocation-free decode entry point against the handle-based one (GPU).

kvq_decode_attention_noalloc serves callers that cannot call cudaMalloc -- a runtime that
owns all of device memory, a plugin whose host framework does every allocation, or a path
that cannot afford cudaMalloc's implicit synchronisation.  It runs the same decode kernel
with its scratch in a fixed device array inside the library.  This file is collected last,
so a run that stops at the first failure has already run every other test; it passes both
alone in a fresh process and after the others (the array keeps its state between calls).
"""
import ctypes

import numpy as np
import pytest

import workloads
from harness import ATOL, RTOL, CudaRun, host_inputs, make_case

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
        ref = run.out.float()
        for _ in range(2):   # two calls in a row on the shared scratch
            out = torch.full_like(qd, float("nan"))
            stream = torch.cuda.current_stream().cuda_stream
            rc = kvq.lib().kvq_decode_attention_noalloc(
                ctypes.byref(d), run.pool.data_ptr(), case.layer, qd.data_ptr(),
                lens.data_ptr(), pt.data_ptr(), len(lengths), ctypes.c_float(0.0),
                out.data_ptr(), stream)
            assert rc == kvq.KVQ_OK, kvq.status_string(rc)
            torch.cuda.synchronize()
            got = out.float()
            assert torch.isfinite(got).all()
            err = (got - ref).abs()
            assert bool((err <= ATOL + RTOL * ref.abs()).all()), float(err.max())
    finally:
        run.close()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import torch
    import bit_paged_kv_diag_b200 as kvq
    d = kvq.Desc(1, 8, 32, 128, 128, 16, 8192, 4096, 4)
    pool = torch.zeros(16, dtype=torch.uint8, device="cuda")
    z = torch.zeros(4096 * 32 * 128, dtype=torch.float16, device="cuda")
    lens = torch.ones(4096, dtype=torch.int32, device="cuda")
    pt = torch.zeros(4096 * 4, dtype=torch.int32, device="cuda")
    rc = kvq.lib().kvq_decode_attention_noalloc(
        ctypes.byref(d), pool.data_ptr(), 0, z.data_ptr(), lens.data_ptr(), pt.data_ptr(),
        4096, ctypes.c_float(0.0), z.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == kvq.KVQ_EUNSUPPORTED
