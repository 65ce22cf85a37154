"""Shared parity machinery: run one workload through the CUDA path (via the C ABI binding)
and through the CPU oracle on the same seeded inputs, and compare.

Acceptance (the tolerance readings stated in the design notes):
* page tables and fp16 scales bit-exact (NVFP4: E4M3 scales bit-exact);
* INT4 codes exact except +-1 flips, counted, fewer than 1e-5 of all codes (NVFP4: E2M1
  codes likewise, a flip being a step to the neighbouring magnitude with the same sign);
* decode outputs |gpu - ref| <= 2e-3 + 1e-2 * |ref| elementwise, ref = fp64 oracle on the
  GPU-written (same dequantised) cache.
"""
import dataclasses

import numpy as np

import oracle
import workloads

ATOL, RTOL = 2e-3, 1e-2
MAX_FLIP_FRACTION = 1e-5


@dataclasses.dataclass
class Case:
    w: workloads.Workload
    lengths: np.ndarray          # tokens cached before the step
    new: np.ndarray              # tokens appended by the step, per sequence
    block: int
    num_pages: int
    page_order: object
    max_pages_per_seq: int
    layer: int = 0
    num_layers: int = 1
    max_batch: int = 0
    fmt: int = 0                 # 0 = rotated INT4, 1 = NVFP4

    @property
    def capacity(self):
        return self.lengths + self.new

    def desc(self):
        import bit_paged_kv_diag_b200 as kvq
        return kvq.Desc(self.num_layers, self.w.num_kv_heads, self.w.num_q_heads, 128,
                        self.block, self.w.page_size, self.num_pages,
                        max(self.max_batch, len(self.lengths)), self.max_pages_per_seq, self.fmt)

    def geometry(self):
        return oracle.Geometry(self.num_layers, self.w.num_kv_heads, self.w.num_q_heads, 128,
                               self.block, self.w.page_size, self.num_pages,
                               self.max_pages_per_seq, self.fmt)


def make_case(w, lengths, new, block=None, pool_factor=None, permute=None, extra_pages_per_seq=0,
              layer=0, num_layers=1, max_batch=0, fmt=0):
    lengths = np.asarray(lengths, np.int32)
    new = np.asarray(new, np.int32)
    S = w.page_size
    cap = lengths + new
    need_pages = (cap.astype(np.int64) + S - 1) // S
    factor = w.pool_factor if pool_factor is None else pool_factor
    P = max(1, int(np.ceil(factor * need_pages.sum())))
    perm = w.permute_pages if permute is None else permute
    order = workloads.rng_for(w, 2, len(lengths)).permutation(P).astype(np.int32) if perm else None
    mp = max(1, int(need_pages.max()) + extra_pages_per_seq)
    return Case(w, lengths, new, block or w.block, P, order, mp, layer, num_layers, max_batch, fmt)


def host_inputs(case: Case):
    """numpy fp16 inputs: prefill rows, step rows, q (token-major, sequences concatenated)."""
    w = case.w
    npre, nnew = int(case.lengths.sum()), int(case.new.sum())
    kp = workloads.kv_rows(w, case.layer, 0, npre, stream=1)
    vp = workloads.kv_rows(w, case.layer, 1, npre, stream=1)
    kn = workloads.kv_rows(w, case.layer, 0, nnew, stream=2)
    vn = workloads.kv_rows(w, case.layer, 1, nnew, stream=2)
    wq = dataclasses.replace(w, batch=len(case.lengths))
    q = workloads.q_rows(wq, case.layer)
    return kp, vp, kn, vn, q


class CudaRun:
    """The CUDA path through the C ABI: alloc, prefill append, step append, decode (or,
    with fused=True and one new token per sequence, the step's append and the decode in
    one kvq_append_decode_attention call)."""

    def __init__(self, case: Case, kp, vp, kn, vn, q, softmax_scale=0.0, fused=False):
        import torch
        import bit_paged_kv_diag_b200 as kvq
        self.case = case
        dev = torch.device("cuda")
        d = case.desc()
        self.pool = torch.zeros(kvq.pool_bytes(d), dtype=torch.uint8, device=dev)
        self.cache, self.page_table = kvq.alloc_pages(d, case.capacity, case.page_order,
                                                      pool=self.pool)
        pt = torch.from_numpy(self.page_table).to(dev)
        t = lambda a: torch.as_tensor(a).to(dev)  # noqa: E731
        zeros = torch.zeros(len(case.lengths), dtype=torch.int32, device=dev)
        lens = t(case.lengths)
        if kp.shape[0] > 0:
            kvq.rotate_quant_append(self.cache, case.layer, t(kp), t(vp),
                                    t(workloads.cu_seqlens(case.lengths)), zeros, pt)
        self.lens_after = case.lengths + case.new
        if fused:
            assert np.all(case.new == 1), "the fused call appends one token per sequence"
            self.out = kvq.append_decode_attention(self.cache, case.layer, t(kn), t(vn), t(q),
                                                   lens, pt, softmax_scale=softmax_scale)
        else:
            if kn.shape[0] > 0:
                kvq.rotate_quant_append(self.cache, case.layer, t(kn), t(vn),
                                        t(workloads.cu_seqlens(case.new)), lens, pt)
            self.out = kvq.decode_attention(self.cache, case.layer, t(q), t(self.lens_after), pt,
                                            softmax_scale=softmax_scale)
        torch.cuda.synchronize()
        self.status = kvq.get_device_status(self.cache)
        self.host_pool = self.pool.cpu().numpy()
        self.host_out = self.out.float().cpu().numpy()

    def close(self):
        self.cache.close()


def compare_pools(case: Case, gpu_pool: np.ndarray, ref_pool: np.ndarray):
    """(scale mismatches, code flips (+-1), other code mismatches, total codes)."""
    g = case.geometry()
    S = g.page_size
    blk = oracle.block_bytes(S, 128, g.fmt)
    a = gpu_pool.reshape(-1, blk)
    b = ref_pool.reshape(-1, blk)
    scale_mis = int(np.count_nonzero(a[:, S * 128:] != b[:, S * 128:]))
    ca, cb = a[:, :S * 128], b[:, :S * 128]
    diff_bytes = np.nonzero(ca != cb)
    flips = other = 0
    if diff_bytes[0].size:
        xa = ca[diff_bytes].astype(np.int16)
        xb = cb[diff_bytes].astype(np.int16)
        for sh in (0, 4):
            na = ((xa >> sh) & 0xF)
            nb = ((xb >> sh) & 0xF)
            if g.fmt == 1:  # E2M1: sign bit 3, magnitude index 0..7
                same_sign = (na & 8) == (nb & 8)
                d = np.where(same_sign, np.abs((na & 7) - (nb & 7)), 99)
                d = np.where(na == nb, 0, d)
            else:
                na = np.where(na >= 8, na - 16, na)
                nb = np.where(nb >= 8, nb - 16, nb)
                d = np.abs(na - nb)
            flips += int(np.count_nonzero(d == 1))
            other += int(np.count_nonzero(d > 1))
    total_codes = int(ca.size) * 2
    return scale_mis, flips, other, total_codes


def oracle_pool(case: Case, kp, vp, kn, vn, page_table):
    g = case.geometry()
    pool = g.new_pool()
    zeros = np.zeros(len(case.lengths), np.int32)
    if kp.shape[0]:
        oracle.rotate_quant_append(g, pool, case.layer, kp, vp,
                                   workloads.cu_seqlens(case.lengths), zeros, page_table)
    if kn.shape[0]:
        oracle.rotate_quant_append(g, pool, case.layer, kn, vn, workloads.cu_seqlens(case.new),
                                   case.lengths, page_table)
    return pool


def check_outputs(gpu_out, ref_out, what=""):
    err = np.abs(gpu_out.astype(np.float64) - ref_out)
    lim = ATOL + RTOL * np.abs(ref_out)
    bad = err > lim
    worst = float(np.max(err / lim)) if err.size else 0.0
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outputs out of tolerance; "
                           f"worst err/limit {worst:.3f}, max abs err {float(err.max()):.3e}")
    return worst


def full_parity(case: Case, softmax_scale=0.0, fused=False):
    """Run everything at a size the oracle finishes in seconds; assert all bars."""
    kp, vp, kn, vn, q = host_inputs(case)
    run = CudaRun(case, kp, vp, kn, vn, q, softmax_scale, fused=fused)
    try:
        assert run.status == 0, f"device status {run.status}"
        pt_ref = oracle.assign_pages(case.capacity, case.w.page_size, case.num_pages,
                                     case.max_pages_per_seq, case.page_order)
        assert np.array_equal(run.page_table, pt_ref), "page table differs from the oracle's"
        ref_pool = oracle_pool(case, kp, vp, kn, vn, pt_ref)
        scale_mis, flips, other, total = compare_pools(case, run.host_pool, ref_pool)
        assert scale_mis == 0, f"{scale_mis} scale bytes differ"
        assert other == 0, f"{other} codes differ by more than 1"
        assert flips <= MAX_FLIP_FRACTION * total, f"{flips} +-1 flips of {total} codes"
        ref = oracle.decode_attention(case.geometry(), run.host_pool, case.layer, q,
                                      run.lens_after, pt_ref, softmax_scale)
        worst = check_outputs(run.host_out, ref, case.w.name)
        return dict(flips=flips, total_codes=total, worst=worst)
    finally:
        run.close()


def prefill_parity(case: Case, softmax_scale=0.0):
    """Chunked prefill: the cache holds case.lengths tokens, the chunk of case.new tokens per
    sequence is appended, then kvq_prefill_attention runs the chunk's queries causally.
    Bars: page table and pool as for full_parity, outputs against the oracle's causal
    attention on the GPU-written cache."""
    import torch
    import bit_paged_kv_diag_b200 as kvq
    kp, vp, kn, vn, _ = host_inputs(case)
    cu_q = workloads.cu_seqlens(case.new)
    q = workloads.q_rows_chunk(case.w, case.layer, int(cu_q[-1]))
    dev = torch.device("cuda")
    d = case.desc()
    pool = torch.zeros(kvq.pool_bytes(d), dtype=torch.uint8, device=dev)
    cache, page_table = kvq.alloc_pages(d, case.capacity, case.page_order, pool=pool)
    try:
        pt = torch.from_numpy(page_table).to(dev)
        t = lambda a: torch.as_tensor(a).to(dev)  # noqa: E731
        zeros = torch.zeros(len(case.lengths), dtype=torch.int32, device=dev)
        if kp.shape[0] > 0:
            kvq.rotate_quant_append(cache, case.layer, t(kp), t(vp),
                                    t(workloads.cu_seqlens(case.lengths)), zeros, pt)
        if kn.shape[0] > 0:
            kvq.rotate_quant_append(cache, case.layer, t(kn), t(vn), t(cu_q), t(case.lengths), pt)
        lens_after = case.lengths + case.new
        out = kvq.prefill_attention(cache, case.layer, t(q), t(cu_q), t(lens_after), pt,
                                    softmax_scale=softmax_scale)
        torch.cuda.synchronize()
        status = kvq.get_device_status(cache)
        assert status == 0, f"device status {status}"
        host_pool = pool.cpu().numpy()
        host_out = out.float().cpu().numpy()
    finally:
        cache.close()
    pt_ref = oracle.assign_pages(case.capacity, case.w.page_size, case.num_pages,
                                 case.max_pages_per_seq, case.page_order)
    assert np.array_equal(page_table, pt_ref), "page table differs from the oracle's"
    ref_pool = oracle_pool(case, kp, vp, kn, vn, pt_ref)
    scale_mis, flips, other, total = compare_pools(case, host_pool, ref_pool)
    assert scale_mis == 0 and other == 0 and flips <= MAX_FLIP_FRACTION * total
    ref = oracle.prefill_attention(case.geometry(), host_pool, case.layer, q, cu_q, lens_after,
                                   pt_ref, softmax_scale)
    worst = check_outputs(host_out, ref, case.w.name + " prefill")
    return dict(worst=worst, total_q=int(cu_q[-1]))
