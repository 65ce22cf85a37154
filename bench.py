#!/usr/bin/env python
"""Benchmark of the rotated-INT4 paged KV-cache hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]

One step = one decode step of the Qwen3-4B-shaped workload (36 layers, 8 KV heads, 32
query heads, head_dim 128, Hadamard block 128, page 16, 16 sequences of 4096 cached
tokens): for every layer, the fused rotate-quant-append of the step's token of each
sequence and paged GQA decode attention over 4097 tokens, in one launch per layer
(kvq_append_decode_attention).  The step is captured once as a CUDA graph and replayed.
The same step as two calls per layer (kvq_rotate_quant_append, kvq_decode_attention) is
reported beside it (``step_separate_calls``).  ``value`` is effective HBM GB/s: the step's algorithmic
bytes (132 B per cached (token, KV head) + page-table, q and out bytes for decode; 2 x 256
B read + 132 B written per appended (token, KV head)) over the device time per step, all
ranks summed.  The cache (2.5 GB) is far larger than the 126 MB L2, so nothing is reused
across steps.

Also reported: the roofline of the step's kernel (the fused append + decode launch, the only
kernel of the timed step) and of the plain decode-attention call, the prefill-append
throughput (8 x 8192 new tokens in one call, b = 32/64/128, and b = 1: plain INT4 without
rotation; L2 flushed between calls), rotated against plain INT4 decode, the NVFP4 cache's
decode, fused step and append, the chunked-prefill attention, the long-context (4 sequences
up to 128K tokens, G = 8) and ragged (256 sequences, scattered pages) workloads' decode and
decode step at full size, the tiny workload's step latency, end-to-end throughput through
the C ABI with host buffers, and the CPU oracle timed on a bounded sample of the same
workload on one host core (``cpu_baseline``) and on every host core
(``cpu_baseline_all_cores``), and its append throughput (``cpu_baseline_append``).

    python bench.py --kernel-case decode|fused|append|prefill|decode_nvfp4|fused_nvfp4|
                                  append_nvfp4|prefill_nvfp4 [--calls C]

runs one case of one kernel (for profiler captures) and prints only its status.

Multi-GPU: replicas only (each rank runs the whole workload on its own GPU; the path has
no exchange step), timing = max over ranks.
"""
import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = ("INT4 paged decode-attn effective HBM GB/s (% of peak); fused quant-append tok/s")
WORKLOAD = "qwen3_4b_decode"
BYTES_PER_TOKEN_HEAD = 132
NOMINAL_HBM_GBS = 8000.0  # the B200's nominal HBM3e bandwidth, for context beside the measured peak


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def decode_bytes(lengths_after, num_kv_heads, num_q_heads, page_size, per_token_head=None):
    lengths_after = np.asarray(lengths_after, np.int64)
    per = BYTES_PER_TOKEN_HEAD if per_token_head is None else per_token_head
    cache = int(lengths_after.sum()) * num_kv_heads * per
    table = int(((lengths_after + page_size - 1) // page_size).sum()) * 4
    qo = 2 * len(lengths_after) * num_q_heads * 128 * 2
    return cache + table + qo


def append_bytes(tokens, num_kv_heads, row_bytes=132):
    return int(tokens) * num_kv_heads * (2 * 256 + row_bytes)


# NVFP4 rows: 64 B of E2M1 codes and 8 E4M3 scales for K and for V.
BYTES_PER_TOKEN_HEAD_NVFP4 = 2 * 64 + 2 * 8

# A write larger than the 126 MB L2 between timed calls whose inputs and outputs would fit.
FLUSH_BYTES = 512 << 20


def _timed_calls(fn, reps, flush=None):
    """Median device time (ms) of fn() over reps calls, events around each call on the
    current stream; with flush, a write of that buffer (512 MB, four times L2) before every
    call, not timed."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    for a, b in ev:
        if flush is not None:
            flush.zero_()
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    return float(np.median([a.elapsed_time(b) for a, b in ev]))


# --------------------------------------------------------------------- clocks --
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.2)
        return self

    def __exit__(self, *a):
        self.result = None
        if self.proc is None:
            return False
        time.sleep(0.1)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        if sm:
            self.result = {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)),
                           "reasons": sorted(reasons), "samples": len(sm)}
        return False


# ------------------------------------------------------------ rank plumbing --
def max_over_ranks(value, world, device=None):
    """The largest of a per-rank value (a device time) over all ranks; every rank calls it
    with the same world and gets the max back.  NCCL (CUDA device) or gloo (CPU)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world, bytes_per_rank_step, ms_per_step):
    """Weak scaling: every rank runs the whole workload; the job's throughput is all ranks'
    bytes over the slowest rank's time."""
    return world * bytes_per_rank_step / (ms_per_step * 1e-3) / 1e9


# ------------------------------------------------------------------- GPU arm --
def run_kvq(args, rank, world, local_rank):
    import torch

    import bit_paged_kv_diag_b200 as kvq

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workloads.WORKLOADS[WORKLOAD]
    L = np.asarray(w.context, np.int32)                 # cached before the step
    B, H, HQ, S, NL = w.batch, w.num_kv_heads, w.num_q_heads, w.page_size, w.num_layers
    cap = L + 1
    P = workloads.pool_pages(w, cap)
    mp = int((cap.max() + S - 1) // S)
    desc = kvq.Desc(NL, H, HQ, 128, w.block, S, P, B, mp)
    cache, pt = kvq.alloc_pages(desc, cap, None)
    ptd = torch.from_numpy(pt).to(dev)

    # Prefill the cache through the append kernel (not timed).
    zeros = torch.zeros(B, dtype=torch.int32, device=dev)
    cu_pre = torch.from_numpy(workloads.cu_seqlens(L)).to(dev)
    for layer in range(NL):
        kp = workloads.kv_rows_torch(w, layer, 0, int(L.sum()), stream=1, device=dev)
        vp = workloads.kv_rows_torch(w, layer, 1, int(L.sum()), stream=1, device=dev)
        kvq.rotate_quant_append(cache, layer, kp, vp, cu_pre, zeros, ptd)
        del kp, vp
    torch.cuda.synchronize()

    # Step inputs, resident in HBM.
    q = torch.stack([workloads.q_rows_torch(w, l, device=dev) for l in range(NL)])
    kn = torch.stack([workloads.kv_rows_torch(w, l, 0, B, stream=2, device=dev) for l in range(NL)])
    vn = torch.stack([workloads.kv_rows_torch(w, l, 1, B, stream=2, device=dev) for l in range(NL)])
    out = torch.empty_like(q)
    lens_before = torch.from_numpy(L).to(dev)
    lens_after = torch.from_numpy(cap).to(dev)
    cu_new = torch.arange(B + 1, dtype=torch.int32, device=dev)

    # Timing events captured into the graph as event-record nodes ("external" events),
    # so every replay stamps the start and end of each layer's decode-attention call.
    ev = [(torch.cuda.Event(enable_timing=True, external=True),
           torch.cuda.Event(enable_timing=True, external=True)) for _ in range(NL)]

    def step(instrument):
        """One decode step: per layer, the token's append and decode attention in one
        fused launch (kvq_append_decode_attention)."""
        for l in range(NL):
            if instrument:
                ev[l][0].record()
            kvq.append_decode_attention(cache, l, kn[l], vn[l], q[l], lens_before, ptd, out=out[l])
            if instrument:
                ev[l][1].record()

    def step_separate():
        """The same step as two calls per layer: kvq_rotate_quant_append, then
        kvq_decode_attention."""
        for l in range(NL):
            kvq.rotate_quant_append(cache, l, kn[l], vn[l], cu_new, lens_before, ptd)
            kvq.decode_attention(cache, l, q[l], lens_after, ptd, out=out[l])

    # Eager warm-up (also initialises the library's launch state), then graph capture.
    # The timed graph has no event nodes between kernels, so consecutive launches keep
    # their programmatic (early-launch) dependencies.
    step(False)
    torch.cuda.synchronize()
    assert kvq.get_device_status(cache) == 0
    side = torch.cuda.Stream(device=dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step(False)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier(device_ids=[local_rank])
        torch.cuda.synchronize()

    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    with ClockSampler(local_rank) as clk:
        t0.record()
        for _ in range(args.steps):
            graph.replay()
        t1.record()
        torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)

    # The same step as separate append and decode calls (2 launches per layer).
    sgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(sgraph, stream=side):
        step_separate()
    for _ in range(3):
        sgraph.replay()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s0.record()
    for _ in range(max(3, args.steps // 2)):
        sgraph.replay()
    s1.record()
    torch.cuda.synchronize()
    sep_ms = max_over_ranks(s0.elapsed_time(s1) / max(3, args.steps // 2), world, dev)
    del sgraph

    # Decode-attention launches: a graph of the 36 decode calls back to back, timed with
    # events around its replays (mean device time per launch, launch overlap included),
    # and each fused launch alone between event nodes of the step graph.
    dgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(dgraph, stream=side):
        for l in range(NL):
            kvq.decode_attention(cache, l, q[l], lens_after, ptd, out=out[l])
    for _ in range(3):
        dgraph.replay()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = max(3, args.steps // 2)
    torch.cuda.synchronize()
    d0.record()
    for _ in range(reps):
        dgraph.replay()
    d1.record()
    torch.cuda.synchronize()
    dec_ms = d0.elapsed_time(d1) / (reps * NL)
    dec_how = "graph of the 36 decode calls back to back, events around the replays"
    igraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(igraph, stream=side):
        step(True)
    for _ in range(3):
        igraph.replay()
    torch.cuda.synchronize()
    iso_ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    del dgraph, igraph
    status = kvq.get_device_status(cache)

    ms_step = ms / args.steps
    dec_b = decode_bytes(cap, H, HQ, S)
    app_b = append_bytes(B, H)
    step_bytes = NL * (dec_b + app_b)
    value = whole_job_gbs(world, step_bytes, ms_step)
    peak, peak_kind = _peaks()

    # End to end through the C ABI with host buffers.  Every step copies its inputs (q and the
    # step's K/V rows of all layers) from pinned host memory and its outputs back.  Main leg:
    # two buffer sets and one captured graph per set; the H2D copies of step s + 1 and the
    # D2H copies of step s run on their own streams under step s's compute (the copy engines
    # work beside the SMs).  'serial' = the same with every copy in line on one stream;
    # 'per_call' = the double-buffered loop issuing the 36 kvq_append_decode_attention calls
    # per step through the Python binding instead of a graph.
    hq = q.cpu().pin_memory()
    hk, hv = kn.cpu().pin_memory(), vn.cpu().pin_memory()
    hout = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    e2e_steps = max(3, min(args.steps, 200))
    s_h2d, s_d2h, s_comp = (torch.cuda.Stream(device=dev) for _ in range(3))
    bufs = []
    for b in range(2):
        qb, knb, vnb, ob = (torch.empty_like(t) for t in (q, kn, vn, out))
        qb.copy_(q), knb.copy_(kn), vnb.copy_(vn)
        gb = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gb, stream=side):
            for l in range(NL):
                kvq.append_decode_attention(cache, l, knb[l], vnb[l], qb[l], lens_before, ptd, out=ob[l])
        bufs.append((qb, knb, vnb, ob, gb))
    torch.cuda.synchronize()

    def step_calls(b):
        qb, knb, vnb, ob, _ = bufs[b]
        for l in range(NL):
            kvq.append_decode_attention(cache, l, knb[l], vnb[l], qb[l], lens_before, ptd, out=ob[l])

    def e2e_pipelined(K, use_graph=True):
        ev = lambda: torch.cuda.Event(enable_timing=False)  # noqa: E731
        in_ready, computed, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def h2d(b):
            qb, knb, vnb, _, _ = bufs[b]
            qb.copy_(hq, non_blocking=True)
            knb.copy_(hk, non_blocking=True)
            vnb.copy_(hv, non_blocking=True)
            in_ready[b].record(s_h2d)

        with torch.cuda.stream(s_h2d):
            t0.record(s_h2d)
            h2d(0)
        for st in range(K):
            b = st % 2
            s_comp.wait_event(in_ready[b])
            if st >= 2:
                s_comp.wait_event(out_done[b])     # step st - 2's outputs have left buffer b
            with torch.cuda.stream(s_comp):
                if use_graph:
                    bufs[b][4].replay()
                else:
                    step_calls(b)
                computed[b].record(s_comp)
            if st + 1 < K:
                nb = (st + 1) % 2
                with torch.cuda.stream(s_h2d):
                    if st >= 1:
                        s_h2d.wait_event(computed[nb])  # step st - 1 has read buffer nb
                    h2d(nb)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(computed[b])
                hout[b].copy_(bufs[b][3], non_blocking=True)
                out_done[b].record(s_d2h)
        with torch.cuda.stream(s_d2h):
            t1.record(s_d2h)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / K

    def e2e_serial(K):
        qb, knb, vnb, ob, gb = bufs[0]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s_comp):
            t0.record(s_comp)
            for _ in range(K):
                qb.copy_(hq, non_blocking=True)
                knb.copy_(hk, non_blocking=True)
                vnb.copy_(hv, non_blocking=True)
                gb.replay()
                hout[0].copy_(ob, non_blocking=True)
            t1.record(s_comp)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / K

    e2e_pipelined(3)
    barrier()
    e2e_ms = max_over_ranks(e2e_pipelined(e2e_steps), world, dev)
    e2e_serial(3)
    e2e_serial_ms = max_over_ranks(e2e_serial(e2e_steps), world, dev)
    e2e_pipelined(3, use_graph=False)
    call_steps = max(3, min(args.steps, 50))
    e2e_call_ms = max_over_ranks(e2e_pipelined(call_steps, use_graph=False), world, dev)
    h2d = (hq.numel() + hk.numel() + hv.numel()) * 2
    d2h = hout[0].numel() * 2
    assert kvq.get_device_status(cache) == 0
    del bufs

    del graph
    cache.close()
    append = run_append_bench(dev) if rank == 0 else None
    plain = run_plain_decode_bench(dev) if rank == 0 else None
    nvfp4 = run_nvfp4_bench(dev) if rank == 0 else None
    prefill = run_prefill_bench(dev) if rank == 0 else None
    configs = run_decode_configs(dev) if rank == 0 else {}

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int4+fp16",
        "data": "synthetic (seeded K/V with lognormal outlier channels and RMS multipliers)",
        "config": {**workload_config(world),
                   "l2": "inputs larger than L2: 2.5 GB cache per step vs 126 MB L2",
                   "graph": "one CUDA graph per step",
                   "step": "per layer one kvq_append_decode_attention (fused 1-token append + decode)"},
        "step_separate_calls": {"ms_per_step": round(sep_ms, 5),
                                "value": round(whole_job_gbs(world, step_bytes, sep_ms), 1),
                                "how": "per layer kvq_rotate_quant_append then kvq_decode_attention"},
        "gpu_launches": args.steps * NL,  # per layer: one fused append + decode launch
        "device_status": status,
        "e2e": {"value": round(whole_job_gbs(world, step_bytes, e2e_ms), 1), "unit": "GB/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": round(e2e_ms, 5),
                "how": "per step: H2D of q and the step's K/V rows from pinned host memory, the "
                       "36-layer step (one captured graph per buffer set), D2H of the outputs; "
                       "two buffer sets, copies of the neighbouring steps on their own streams "
                       "under the compute",
                "serial": {"value": round(whole_job_gbs(world, step_bytes, e2e_serial_ms), 1),
                           "ms_per_step": round(e2e_serial_ms, 5),
                           "how": "every copy in line with the step on one stream"},
                "per_call": {"value": round(whole_job_gbs(world, step_bytes, e2e_call_ms), 1),
                             "ms_per_step": round(e2e_call_ms, 5), "steps": call_steps,
                             "how": "as the main leg, the 36 kvq_append_decode_attention calls "
                                    "per step issued through the Python binding (ctypes), no "
                                    "graph"}},
    }
    # The timed step is 36 launches of one kernel (the fused append + decode), so that is
    # the roofline kernel: its algorithmic bytes per launch over its mean launch time in
    # the timed graph (events around the timed replays, on the replay stream).
    fused_b = dec_b + app_b
    fused_us = ms_step * 1e3 / NL
    ach = fused_b / (fused_us * 1e-6) / 1e9
    line["roofline"] = {
        "kernel": "decode_kernel<G, S, fused> (one-token append + decode attention of one "
                  "layer, one launch; the only kernel of the timed step)",
        "bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
        "frac": round(ach / peak, 4), "peak_kind": peak_kind,
        "frac_of_nominal": round(ach / NOMINAL_HBM_GBS, 4),
        "traffic": _traffic("fused", fused_b), "us_per_launch": round(fused_us, 3),
        "us_per_launch_alone": round(iso_ms * 1e3, 3),
        "bytes_per_launch": fused_b,
        "timing": "timed step graph: mean device time per launch (36 launches per step, "
                  "programmatic launch overlap included); 'alone' = between event nodes"}
    dach = dec_b / (dec_ms * 1e-3) / 1e9
    line["decode_attention"] = {
        "kernel": "decode_kernel<G, S> (decode attention of one layer, one launch)",
        "achieved": round(dach, 1), "unit": "GB/s", "frac": round(dach / peak, 4),
        "frac_of_nominal": round(dach / NOMINAL_HBM_GBS, 4),
        "traffic": _traffic("decode", dec_b), "us_per_launch": round(dec_ms * 1e3, 3),
        "bytes_per_launch": dec_b, "timing": dec_how}
    line["append"] = append
    line["plain_int4"] = plain
    line["nvfp4"] = nvfp4
    line["prefill"] = prefill
    line["long_context"] = configs.get("long_context")
    line["ragged"] = configs.get("ragged")
    line["tiny"] = configs.get("tiny")
    line["clocks"] = clk.result
    return line


def _traffic(kernel, alg_bytes):
    """DRAM bytes per launch from the committed ncu summary, if it is for the current
    kernel source; else None."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel]
        src = os.path.join(ROOT, "bit_paged_kv_diag_b200", "csrc", rec["source"])
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if h != rec["source_sha256_16"]:
            return None
        return int(rec["dram_bytes_per_launch"])
    except Exception:
        return None


def run_append_bench(dev, reps=20):
    """Prefill-append stress: 8 x 8192 new tokens through one call, b = 32, 64, 128, and
    b = 1 (the plain INT4 variant, no rotation)."""
    import torch

    import bit_paged_kv_diag_b200 as kvq
    w = workloads.WORKLOADS["prefill_append"]
    B, H, S, T = w.batch, w.num_kv_heads, w.page_size, w.batch * w.new_tokens
    cap = np.full(B, w.new_tokens, np.int32)
    P = workloads.pool_pages(w, cap)
    mp = int((cap.max() + S - 1) // S)
    k = workloads.kv_rows_torch(w, 0, 0, T, stream=1, device=dev)
    v = workloads.kv_rows_torch(w, 0, 1, T, stream=1, device=dev)
    cu = torch.from_numpy(workloads.cu_seqlens(cap)).to(dev)
    z = torch.zeros(B, dtype=torch.int32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    res = {}
    peak, _ = _peaks()
    for block in [1] + list(w.blocks_sweep):
        desc = kvq.Desc(1, H, w.num_q_heads, 128, block, S, P, B, mp)
        cache, pt = kvq.alloc_pages(desc, cap, None)
        ptd = torch.from_numpy(pt).to(dev)
        for _ in range(3):
            kvq.rotate_quant_append(cache, 0, k, v, cu, z, ptd)
        torch.cuda.synchronize()
        us = _timed_calls(lambda: kvq.rotate_quant_append(cache, 0, k, v, cu, z, ptd), reps,
                          flush) * 1e3
        gbs = append_bytes(T, H) / (us * 1e-6) / 1e9
        res[f"b{block}"] = {"us_per_call": round(us, 2), "tok_s": round(T / (us * 1e-6), 1),
                            "gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}
        assert kvq.get_device_status(cache) == 0
        cache.close()
    res["workload"] = ("prefill_append: 8 x 8192 tokens, 8 KV heads, page 16, Student-t(3); "
                       "b1 = plain INT4 (no rotation)")
    res["timing"] = ("median of 20 calls, events around each, a 512 MB write between calls "
                     "(flushes the 126 MB L2; its dirty lines are written back during the next "
                     "call)")
    res["traffic"] = _traffic("append", append_bytes(T, H))
    return res


def run_plain_decode_bench(dev, reps=10):
    """Rotated (b = 128) against plain INT4 (b = 1) decode on the Qwen3-4B-shaped layer
    shape: a graph of 36 decode calls cycling over 4 layer pools (276 MB > L2), per-launch
    device time from events around the replays."""
    import torch

    import bit_paged_kv_diag_b200 as kvq
    w = workloads.WORKLOADS[WORKLOAD]
    L = np.asarray(w.context, np.int32)
    B, H, HQ, S, NL = w.batch, w.num_kv_heads, w.num_q_heads, w.page_size, 4
    cap = L + 1
    P = workloads.pool_pages(w, cap)
    mp = int((cap.max() + S - 1) // S)
    res = {}
    for block in (w.block, 1):
        desc = kvq.Desc(NL, H, HQ, 128, block, S, P, B, mp)
        cache, pt = kvq.alloc_pages(desc, cap, None)
        ptd = torch.from_numpy(pt).to(dev)
        zeros = torch.zeros(B, dtype=torch.int32, device=dev)
        cu = torch.from_numpy(workloads.cu_seqlens(cap)).to(dev)
        for layer in range(NL):
            kp = workloads.kv_rows_torch(w, layer, 0, int(cap.sum()), stream=1, device=dev)
            vp = workloads.kv_rows_torch(w, layer, 1, int(cap.sum()), stream=1, device=dev)
            kvq.rotate_quant_append(cache, layer, kp, vp, cu, zeros, ptd)
            del kp, vp
        q = torch.stack([workloads.q_rows_torch(w, l, device=dev) for l in range(NL)])
        out = torch.empty_like(q)
        lens = torch.from_numpy(cap).to(dev)
        side = torch.cuda.Stream(device=dev)
        kvq.decode_attention(cache, 0, q[0], lens, ptd, out=out[0])
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for i in range(36):
                kvq.decode_attention(cache, i % NL, q[i % NL], lens, ptd, out=out[i % NL])
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        res[f"decode_us_b{block}"] = round(a.elapsed_time(b) * 1e3 / (reps * 36), 3)
        assert kvq.get_device_status(cache) == 0
        del g
        cache.close()
    res["how"] = ("graph of 36 decode calls over 4 layer pools of the qwen3_4b_decode shape, "
                  "b = 128 (rotated) and b = 1 (plain INT4)")
    return res


def run_nvfp4_bench(dev, reps=10):
    """The NVFP4 cache format (E2M1 codes, E4M3 scale per 16 channels, b = 128): decode on
    the Qwen3-4B-shaped layer (a graph of 36 calls over 4 layer pools, as the plain-INT4
    line) and the 8 x 8192-token prefill append."""
    import torch

    import bit_paged_kv_diag_b200 as kvq
    peak, peak_kind = _peaks()
    res = {}
    w = workloads.WORKLOADS[WORKLOAD]
    L = np.asarray(w.context, np.int32)
    B, H, HQ, S, NL = w.batch, w.num_kv_heads, w.num_q_heads, w.page_size, 4
    cap = L + 1
    P = workloads.pool_pages(w, cap)
    mp = int((cap.max() + S - 1) // S)
    desc = kvq.Desc(NL, H, HQ, 128, w.block, S, P, B, mp, kvq.FORMAT_NVFP4)
    cache, pt = kvq.alloc_pages(desc, cap, None)
    ptd = torch.from_numpy(pt).to(dev)
    zeros = torch.zeros(B, dtype=torch.int32, device=dev)
    cu = torch.from_numpy(workloads.cu_seqlens(cap)).to(dev)
    for layer in range(NL):
        kp = workloads.kv_rows_torch(w, layer, 0, int(cap.sum()), stream=1, device=dev)
        vp = workloads.kv_rows_torch(w, layer, 1, int(cap.sum()), stream=1, device=dev)
        kvq.rotate_quant_append(cache, layer, kp, vp, cu, zeros, ptd)
        del kp, vp
    q = torch.stack([workloads.q_rows_torch(w, l, device=dev) for l in range(NL)])
    out = torch.empty_like(q)
    lens = torch.from_numpy(cap).to(dev)
    side = torch.cuda.Stream(device=dev)
    kvq.decode_attention(cache, 0, q[0], lens, ptd, out=out[0])
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for i in range(36):
            kvq.decode_attention(cache, i % NL, q[i % NL], lens, ptd, out=out[i % NL])
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    us = a.elapsed_time(b) * 1e3 / (reps * 36)
    nb = decode_bytes(cap, H, HQ, S, BYTES_PER_TOKEN_HEAD_NVFP4)
    gbs = nb / (us * 1e-6) / 1e9
    res["decode"] = {"us_per_launch": round(us, 3), "bytes_per_launch": nb, "gbs": round(gbs, 1),
                     "frac": round(gbs / peak, 4), "peak": peak, "peak_kind": peak_kind,
                     "traffic": _traffic("decode_nvfp4", nb),
                     "how": "graph of 36 decode calls over 4 layer pools of the qwen3_4b_decode "
                            "shape, b = 128, 144 B per (token, KV head)"}
    del g
    # The fused step on the NVFP4 cache: per layer one kvq_append_decode_attention (the
    # same token re-appended at position L every replay).
    kn = torch.stack([workloads.kv_rows_torch(w, l, 0, B, stream=2, device=dev) for l in range(NL)])
    vn = torch.stack([workloads.kv_rows_torch(w, l, 1, B, stream=2, device=dev) for l in range(NL)])
    before = torch.from_numpy(L).to(dev)
    kvq.append_decode_attention(cache, 0, kn[0], vn[0], q[0], before, ptd, out=out[0])
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for i in range(36):
            kvq.append_decode_attention(cache, i % NL, kn[i % NL], vn[i % NL], q[i % NL], before,
                                        ptd, out=out[i % NL])
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    step_b = 36 * (nb + B * H * 2 * 256 + B * H * BYTES_PER_TOKEN_HEAD_NVFP4)
    res["fused_step"] = {"ms_per_36_layers": round(ms, 5), "gbs": round(step_b / (ms * 1e-3) / 1e9, 1),
                         "how": "graph of 36 kvq_append_decode_attention calls over 4 layer pools"}
    assert kvq.get_device_status(cache) == 0
    del g
    cache.close()

    wa = workloads.WORKLOADS["prefill_append"]
    B, H, S, T = wa.batch, wa.num_kv_heads, wa.page_size, wa.batch * wa.new_tokens
    cap = np.full(B, wa.new_tokens, np.int32)
    P = workloads.pool_pages(wa, cap)
    mp = int((cap.max() + S - 1) // S)
    k = workloads.kv_rows_torch(wa, 0, 0, T, stream=1, device=dev)
    v = workloads.kv_rows_torch(wa, 0, 1, T, stream=1, device=dev)
    cu = torch.from_numpy(workloads.cu_seqlens(cap)).to(dev)
    z = torch.zeros(B, dtype=torch.int32, device=dev)
    desc = kvq.Desc(1, H, wa.num_q_heads, 128, 128, S, P, B, mp, kvq.FORMAT_NVFP4)
    cache, pt = kvq.alloc_pages(desc, cap, None)
    ptd = torch.from_numpy(pt).to(dev)
    for _ in range(3):
        kvq.rotate_quant_append(cache, 0, k, v, cu, z, ptd)
    torch.cuda.synchronize()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    us = _timed_calls(lambda: kvq.rotate_quant_append(cache, 0, k, v, cu, z, ptd), 20, flush) * 1e3
    gbs = append_bytes(T, H, BYTES_PER_TOKEN_HEAD_NVFP4) / (us * 1e-6) / 1e9
    res["append_b128"] = {"us_per_call": round(us, 2), "tok_s": round(T / (us * 1e-6), 1),
                          "gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
                          "workload": "prefill_append: 8 x 8192 tokens, 8 KV heads, page 16"}
    assert kvq.get_device_status(cache) == 0
    cache.close()
    res["prefill"] = run_prefill_bench(dev, fmt=1)
    return res


def _fill_cache(cache, w, lens, ptd, layers, dev):
    """Write lens[b] tokens of every sequence into each layer through the append kernel."""
    import torch

    import bit_paged_kv_diag_b200 as kvq
    zeros = torch.zeros(len(lens), dtype=torch.int32, device=dev)
    cu = torch.from_numpy(workloads.cu_seqlens(lens)).to(dev)
    for layer in range(layers):
        kp = workloads.kv_rows_torch(w, layer, 0, int(np.sum(lens)), stream=1, device=dev)
        vp = workloads.kv_rows_torch(w, layer, 1, int(np.sum(lens)), stream=1, device=dev)
        kvq.rotate_quant_append(cache, layer, kp, vp, cu, zeros, ptd)
        del kp, vp
    torch.cuda.synchronize()


def run_decode_config(dev, name, reps=5):
    """Decode throughput on one decode workload at its full size: plain decode attention
    (kvq_decode_attention) and the decode step (kvq_append_decode_attention: the step's
    token of every sequence appended, then attention over it), each as a graph of calls
    alternating over the workload's layer pools, mean device time per launch from events
    around the replays.  long_context keeps two layer pools (2 x 190 MB), ragged one
    (1.1 GB), both larger than the 126 MB L2."""
    import torch

    import bit_paged_kv_diag_b200 as kvq
    w = workloads.WORKLOADS[name]
    L = workloads.context_lengths(w)
    B, H, HQ, S = w.batch, w.num_kv_heads, w.num_q_heads, w.page_size
    NL = 2 if name == "long_context" else 1
    cap = L + 1
    P = workloads.pool_pages(w, cap)
    mp = int((cap.max() + S - 1) // S)
    desc = kvq.Desc(NL, H, HQ, 128, w.block, S, P, B, mp)
    cache, pt = kvq.alloc_pages(desc, cap, workloads.page_order(w, P))
    ptd = torch.from_numpy(pt).to(dev)
    _fill_cache(cache, w, L, ptd, NL, dev)
    q = torch.stack([workloads.q_rows_torch(w, l, device=dev) for l in range(NL)])
    kn = torch.stack([workloads.kv_rows_torch(w, l, 0, B, stream=2, device=dev) for l in range(NL)])
    vn = torch.stack([workloads.kv_rows_torch(w, l, 1, B, stream=2, device=dev) for l in range(NL)])
    out = torch.empty_like(q)
    before = torch.from_numpy(L).to(dev)
    after = torch.from_numpy(cap).to(dev)
    side = torch.cuda.Stream(device=dev)
    calls = 8
    peak, peak_kind = _peaks()
    dec_b = decode_bytes(cap, H, HQ, S)
    fused_b = dec_b + append_bytes(B, H)
    res = {"workload": f"{name}: batch {B}, {H} KV heads, {HQ} query heads, b = {w.block}, "
                       f"page {S}, {int(cap.sum())} cached tokens after the step's append"
                       + (", pages scattered through a 1.2x pool" if w.permute_pages else ""),
           "bytes_per_launch": dec_b, "peak": peak, "peak_kind": peak_kind}
    for key, fn, nb in (
            ("decode", lambda l: kvq.decode_attention(cache, l, q[l], after, ptd, out=out[l]), dec_b),
            ("fused", lambda l: kvq.append_decode_attention(cache, l, kn[l], vn[l], q[l], before, ptd,
                                                            out=out[l]), fused_b)):
        fn(0)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for i in range(calls):
                fn(i % NL)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        us = a.elapsed_time(b) * 1e3 / (reps * calls)
        gbs = nb / (us * 1e-6) / 1e9
        res[key] = {"us_per_launch": round(us, 3), "bytes_per_launch": nb, "gbs": round(gbs, 1),
                    "frac": round(gbs / peak, 4), "frac_of_nominal": round(gbs / NOMINAL_HBM_GBS, 4),
                    "traffic": _traffic(f"{key}_{name}", nb)}
        del g
    res["how"] = (f"graph of {calls} calls alternating over {NL} layer pool(s), events around "
                  f"{reps} replays; fused = the step's one-token append + decode in one launch")
    if name == "long_context":
        res["step_36_layers_ms_extrapolated"] = round(36 * res["fused"]["us_per_launch"] / 1e3, 4)
    assert kvq.get_device_status(cache) == 0
    cache.close()
    return res


def run_tiny_latency(dev, reps=200):
    """The tiny workload's decode step (one fused append + decode launch over 257 tokens):
    latency of one call alone (events around each eager call, median) and back to back in
    a graph (mean per launch)."""
    import torch

    import bit_paged_kv_diag_b200 as kvq
    w = workloads.WORKLOADS["tiny"]
    L = np.asarray(w.context, np.int32)
    B, H, HQ, S = w.batch, w.num_kv_heads, w.num_q_heads, w.page_size
    cap = L + 1
    P = workloads.pool_pages(w, cap)
    mp = int((cap.max() + S - 1) // S)
    desc = kvq.Desc(1, H, HQ, 128, w.block, S, P, B, mp)
    cache, pt = kvq.alloc_pages(desc, cap, None)
    ptd = torch.from_numpy(pt).to(dev)
    _fill_cache(cache, w, L, ptd, 1, dev)
    q = workloads.q_rows_torch(w, 0, device=dev)
    kn = workloads.kv_rows_torch(w, 0, 0, B, stream=2, device=dev)
    vn = workloads.kv_rows_torch(w, 0, 1, B, stream=2, device=dev)
    out = torch.empty_like(q)
    before = torch.from_numpy(L).to(dev)
    fn = lambda: kvq.append_decode_attention(cache, 0, kn, vn, q, before, ptd, out=out)  # noqa: E731
    for _ in range(10):
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(50)]
    for a, b in ev:
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
    alone = float(np.median([a.elapsed_time(b) for a, b in ev])) * 1e3
    side = torch.cuda.Stream(device=dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for _ in range(100):
            fn()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps // 100 + 1):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    per = a.elapsed_time(b) * 1e3 / ((reps // 100 + 1) * 100)
    assert kvq.get_device_status(cache) == 0
    del g
    cache.close()
    return {"workload": "tiny: 1 sequence, 2 KV heads, 8 query heads, b = 32, page 16, "
                        "256 cached tokens + the step's token",
            "us_per_call_alone": round(alone, 3), "us_per_call_graph": round(per, 3),
            "bytes_per_call": decode_bytes(cap, H, HQ, S) + append_bytes(B, H),
            "how": "fused append + decode; alone = median of 50 eager calls with events around "
                   "each; graph = mean over back-to-back launches in a graph of 100"}


def run_decode_configs(dev):
    res = {}
    for name in ("long_context", "ragged"):
        res[name] = run_decode_config(dev, name)
    res["tiny"] = run_tiny_latency(dev)
    return res


def prefill_flops(lengths_after, chunks, num_q_heads):
    """Algorithmic FLOPs of causal chunked prefill: 4 * 128 per (query row, visible token)
    (q.k and p.v, a multiply and an add per channel each)."""
    total = 0
    for L, C in zip(lengths_after, chunks):
        first = int(L) - int(C) + 1          # visible tokens of the chunk's first query
        total += (first + first + int(C) - 1) * int(C) // 2
    return total * num_q_heads * 4 * 128


def run_prefill_bench(dev, reps=5, fmt=0):
    """Chunked prefill (kvq_prefill_attention) on the chunked_prefill workload: 16 x 512
    chunk tokens over 3584 cached ones, alternating two layer pools; device time per call
    from events around a graph of the calls.  fmt 1: the NVFP4 cache."""
    import torch

    import bit_paged_kv_diag_b200 as kvq
    w = workloads.WORKLOADS["chunked_prefill"]
    L0 = np.asarray(w.context, np.int32)
    B, H, HQ, S, NL = w.batch, w.num_kv_heads, w.num_q_heads, w.page_size, w.num_layers
    chunk = np.full(B, w.new_tokens, np.int32)
    cap = L0 + chunk
    P = workloads.pool_pages(w, cap)
    mp = int((cap.max() + S - 1) // S)
    desc = kvq.Desc(NL, H, HQ, 128, w.block, S, P, B, mp, fmt)
    cache, pt = kvq.alloc_pages(desc, cap, None)
    ptd = torch.from_numpy(pt).to(dev)
    zeros = torch.zeros(B, dtype=torch.int32, device=dev)
    cu_all = torch.from_numpy(workloads.cu_seqlens(cap)).to(dev)
    for layer in range(NL):
        kp = workloads.kv_rows_torch(w, layer, 0, int(cap.sum()), stream=1, device=dev)
        vp = workloads.kv_rows_torch(w, layer, 1, int(cap.sum()), stream=1, device=dev)
        kvq.rotate_quant_append(cache, layer, kp, vp, cu_all, zeros, ptd)
        del kp, vp
    T = int(chunk.sum())
    q = torch.stack([torch.from_numpy(workloads.q_rows_chunk(w, layer, T)) for layer in range(NL)]).to(dev)
    out = torch.empty_like(q)
    cu_q = torch.from_numpy(workloads.cu_seqlens(chunk)).to(dev)
    lens = torch.from_numpy(cap).to(dev)
    calls = 4
    side = torch.cuda.Stream(device=dev)
    kvq.prefill_attention(cache, 0, q[0], cu_q, lens, ptd, out=out[0])
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for i in range(calls):
            kvq.prefill_attention(cache, i % NL, q[i % NL], cu_q, lens, ptd, out=out[i % NL])
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    us = a.elapsed_time(b) * 1e3 / (reps * calls)
    assert kvq.get_device_status(cache) == 0
    del g
    cache.close()
    fl = prefill_flops(cap, chunk, HQ)
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak = float(json.load(f)["bf16_tflops"])
        kind = "measured bf16 dense (burst)"
    except Exception:
        peak, kind = 1590.0, "fallback bf16 dense"
    tf = fl / (us * 1e-6) / 1e12
    return {"us_per_call": round(us, 2), "tflops": round(tf, 1), "peak_tflops": peak,
            "frac": round(tf / peak, 4), "peak_kind": kind, "flops_per_call": fl,
            "workload": "chunked_prefill: 16 sequences x 512-token chunk after 3584 cached "
                        "tokens, Qwen3-4B heads (8 KV / 32 q), b = 128, page 16",
            "note": "algorithmic FLOPs 4*128 per (query row, visible token); the kernel runs "
                    + ("QK^T (q~ fp16 hi + lo against K dequantised exactly to fp16) and PV (p as "
                       "fp16 hi + lo against V dequantised exactly to fp16) as tcgen05 MMAs (NVFP4 "
                       "cache), twice the algorithmic FLOPs on the tensor cores" if fmt else
                       "QK^T (q~ fp16 hi + lo against exact fp16 K codes) and PV (P' bf16 hi + lo "
                       "against exact bf16 V codes) as tcgen05 MMAs, so the tensor cores execute twice "
                       "the algorithmic FLOPs")}


# ------------------------------------------------------------- CPU oracle arm --
def oracle_sample(budget_s, n_units_max=None):
    """Time the CPU oracle on whole (sequence, KV head) units of one layer of the decode
    workload: its step append (one token per sequence, all heads) and decode attention of
    the unit's G query heads, fp64, one thread.  Returns (GB/s, description)."""
    import oracle
    w = workloads.WORKLOADS[WORKLOAD]
    G, H, S = w.group, w.num_kv_heads, w.page_size
    L = int(w.context[0])
    nseq = 1
    g = oracle.Geometry(1, H, w.num_q_heads, 128, w.block, S, nseq * ((L + 1 + S - 1) // S),
                        (L + 1 + S - 1) // S)
    cap = np.full(nseq, L + 1, np.int32)
    pt = oracle.assign_pages(cap, S, g.num_pages, g.max_pages_per_seq)
    pool = g.new_pool()
    kp, vp = workloads.kv_rows(w, 0, 0, L * nseq, 1), workloads.kv_rows(w, 0, 1, L * nseq, 1)
    oracle.rotate_quant_append(g, pool, 0, kp, vp, workloads.cu_seqlens([L] * nseq),
                               np.zeros(nseq, np.int32), pt)
    kn, vn = workloads.kv_rows(w, 0, 0, nseq, 2), workloads.kv_rows(w, 0, 1, nseq, 2)
    q = workloads.q_rows(w, 0)[:nseq]
    units, byt = 0, 0
    t0 = time.perf_counter()
    while True:
        oracle.rotate_quant_append(g, pool, 0, kn, vn, workloads.cu_seqlens([1] * nseq),
                                   np.full(nseq, L, np.int32), pt)
        byt += append_bytes(nseq, H)
        for h in range(H):
            for qi in range(G):
                oracle.decode_one(g, pool, 0, q, cap, pt, 0, h * G + qi)
            units += 1
            byt += (L + 1) * BYTES_PER_TOKEN_HEAD + 2 * G * 256
            if (time.perf_counter() - t0 >= budget_s) or (n_units_max and units >= n_units_max):
                el = time.perf_counter() - t0
                desc = (f"oracle (C, fp64 attention, 1 thread): step append of 1 token x {H} "
                        f"KV heads + decode of {units} (sequence, KV head) units x {G} query "
                        f"heads at {L + 1} tokens, one layer of {WORKLOAD}; {el:.2f} s")
                return byt / el / 1e9, desc


def oracle_sample_threads(budget_s, threads):
    """The same oracle decode on every host core: threads call the oracle's C decode of one
    (sequence, query head) at a time (the C call releases the interpreter lock) over the
    G query heads of the layer's units, on one cache written once.  Returns (GB/s,
    threads, description)."""
    import concurrent.futures
    import oracle
    w = workloads.WORKLOADS[WORKLOAD]
    G, H, S = w.group, w.num_kv_heads, w.page_size
    L = int(w.context[0])
    g = oracle.Geometry(1, H, w.num_q_heads, 128, w.block, S, (L + 1 + S - 1) // S,
                        (L + 1 + S - 1) // S)
    cap = np.full(1, L + 1, np.int32)
    pt = oracle.assign_pages(cap, S, g.num_pages, g.max_pages_per_seq)
    pool = g.new_pool()
    kp, vp = workloads.kv_rows(w, 0, 0, L + 1, 1), workloads.kv_rows(w, 0, 1, L + 1, 1)
    oracle.rotate_quant_append(g, pool, 0, kp, vp, workloads.cu_seqlens([L + 1]),
                               np.zeros(1, np.int32), pt)
    q = workloads.q_rows(w, 0)[:1]
    t0 = time.perf_counter()

    def work(tid):
        n = 0
        while time.perf_counter() - t0 < budget_s:
            oracle.decode_one(g, pool, 0, q, cap, pt, 0, (tid + n * threads) % (H * G))
            n += 1
        return n

    with concurrent.futures.ThreadPoolExecutor(max_workers=threads) as ex:
        calls = sum(ex.map(work, range(threads)))
    el = time.perf_counter() - t0
    byt = calls / G * ((L + 1) * BYTES_PER_TOKEN_HEAD + 2 * G * 256)
    desc = (f"oracle (C, fp64 attention, {threads} threads): decode of {calls} (sequence, query "
            f"head) rows at {L + 1} tokens, one layer of {WORKLOAD}; {el:.2f} s")
    return byt / el / 1e9, threads, desc


def cpu_model():
    """The host CPU's model name (first 'model name' line of /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def oracle_append_sample(budget_s, threads=1):
    """The oracle's rotate-quant-append on the prefill-append workload (b = 128, 8 KV heads,
    Student-t(3) rows): calls of 64 tokens, each thread appending into its own one-sequence
    pool (the C call releases the interpreter lock).  Returns (tokens/s, description)."""
    import concurrent.futures
    import oracle
    w = workloads.WORKLOADS["prefill_append"]
    H, S, n = w.num_kv_heads, w.page_size, 64
    g = oracle.Geometry(1, H, w.num_q_heads, 128, 128, S, n // S, n // S)
    pt = oracle.assign_pages(np.array([n], np.int32), S, n // S, n // S)
    k, v = workloads.kv_rows(w, 0, 0, n, 1), workloads.kv_rows(w, 0, 1, n, 1)
    cu, z = workloads.cu_seqlens([n]), np.zeros(1, np.int32)
    t0 = time.perf_counter()

    def work(tid):
        pool = g.new_pool()
        calls = 0
        while time.perf_counter() - t0 < budget_s:
            oracle.rotate_quant_append(g, pool, 0, k, v, cu, z, pt)
            calls += 1
        return calls

    with concurrent.futures.ThreadPoolExecutor(max_workers=threads) as ex:
        calls = sum(ex.map(work, range(threads)))
    el = time.perf_counter() - t0
    desc = (f"oracle (C, fp32 rotation, {threads} thread(s)): {calls} calls of {n} tokens x {H} "
            f"KV heads, b = 128, prefill_append rows; {el:.2f} s")
    return calls * n / el, desc


def workload_config(world):
    """The bench workload's shape keys, shared by both arms' JSON lines."""
    w = workloads.WORKLOADS[WORKLOAD]
    L = np.asarray(w.context, np.int32)
    return {"workload": WORKLOAD, "layers": w.num_layers, "batch": w.batch, "context": int(L[0]),
            "kv_heads": w.num_kv_heads, "q_heads": w.num_q_heads, "head_dim": 128,
            "hadamard_block": w.block, "page_size": w.page_size, "global_batch": w.batch * world,
            "seq_len": int(L[0]) + 1, "parallelism": f"replicas x{world}"}


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle as it stands, on host cores, same metric and
    workload; each step a bounded sample sized so the whole run ends in a few minutes."""
    if rank != 0:
        return None
    total = max(1, args.steps + args.warmup)
    per_step = max(0.02, min(2.0, 150.0 / total))
    for _ in range(args.warmup):
        oracle_sample(per_step, n_units_max=1)
    vals, descs = [], []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        v, d = oracle_sample(per_step)
        vals.append(v)
        descs.append(d)
    el = time.perf_counter() - t0
    val = float(np.mean(vals))
    return {
        "impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / max(1, args.steps) * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {**workload_config(world),
                   "sample": "bounded per step: the oracle on host cores"},
        "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": descs[-1] if descs else "", "cpu_model": cpu_model()},
        "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------ profiling cases --
def run_kernel_case(which, calls):
    """A small case of one kernel for ncu captures: ``decode`` = decode attention on one
    layer of the Qwen3-4B-shaped workload (69 MB of cache); ``fused`` = the same with the
    step's one-token append fused in; ``append`` = the prefill-append call (8 x 8192
    tokens, b = 128; 268 MB read, 69 MB written); ``prefill`` = chunked-prefill attention
    (16 x 128-token chunks after 896 cached tokens); ``decode_nvfp4``, ``fused_nvfp4``,
    ``append_nvfp4`` and ``prefill_nvfp4`` are the same cases on an NVFP4 cache;
    ``decode_long`` / ``fused_long`` and ``decode_ragged`` / ``fused_ragged`` are the decode
    and the fused step on one layer of the long-context (190 MB) and ragged (1.1 GB)
    workloads.  The kernel is launched ``calls`` times after the setup."""
    import torch

    import bit_paged_kv_diag_b200 as kvq
    dev = torch.device("cuda", 0)
    fmt = kvq.FORMAT_NVFP4 if which.endswith("_nvfp4") else kvq.FORMAT_INT4
    which = which.replace("_nvfp4", "")
    if which == "prefill":
        # 16 sequences, a 128-token chunk after 896 cached tokens (chunked_prefill's heads).
        w = workloads.WORKLOADS["chunked_prefill"]
        B, H, S = w.batch, w.num_kv_heads, w.page_size
        chunk = np.full(B, 128, np.int32)
        cap = np.full(B, 1024, np.int32)
        P = workloads.pool_pages(w, cap)
        desc = kvq.Desc(1, H, w.num_q_heads, 128, w.block, S, P, B, int((cap.max() + S - 1) // S),
                        fmt)
        cache, pt = kvq.alloc_pages(desc, cap, None)
        ptd = torch.from_numpy(pt).to(dev)
        k = workloads.kv_rows_torch(w, 0, 0, int(cap.sum()), stream=1, device=dev)
        v = workloads.kv_rows_torch(w, 0, 1, int(cap.sum()), stream=1, device=dev)
        kvq.rotate_quant_append(cache, 0, k, v, torch.from_numpy(workloads.cu_seqlens(cap)).to(dev),
                                torch.zeros(B, dtype=torch.int32, device=dev), ptd)
        cu_q = torch.from_numpy(workloads.cu_seqlens(chunk)).to(dev)
        q = torch.from_numpy(workloads.q_rows_chunk(w, 0, int(chunk.sum()))).to(dev)
        lens = torch.from_numpy(cap).to(dev)
        torch.cuda.synchronize()
        for _ in range(calls):
            kvq.prefill_attention(cache, 0, q, cu_q, lens, ptd)
        torch.cuda.synchronize()
        assert kvq.get_device_status(cache) == 0
        cache.close()
        print(json.dumps({"kernel_case": which, "calls": calls, "ok": True}))
        return
    if which == "append":
        w = workloads.WORKLOADS["prefill_append"]
        B, H, S, T = w.batch, w.num_kv_heads, w.page_size, w.batch * w.new_tokens
        cap = np.full(B, w.new_tokens, np.int32)
        P = workloads.pool_pages(w, cap)
        desc = kvq.Desc(1, H, w.num_q_heads, 128, w.block, S, P, B, int((cap.max() + S - 1) // S),
                        fmt)
        cache, pt = kvq.alloc_pages(desc, cap, None)
        ptd = torch.from_numpy(pt).to(dev)
        k = workloads.kv_rows_torch(w, 0, 0, T, stream=1, device=dev)
        v = workloads.kv_rows_torch(w, 0, 1, T, stream=1, device=dev)
        cu = torch.from_numpy(workloads.cu_seqlens(cap)).to(dev)
        z = torch.zeros(B, dtype=torch.int32, device=dev)
        torch.cuda.synchronize()
        for _ in range(calls):
            kvq.rotate_quant_append(cache, 0, k, v, cu, z, ptd)
    else:
        # decode / fused on the Qwen3-4B-shaped layer; decode_long / fused_long on the
        # long-context workload (one layer, 190 MB); decode_ragged / fused_ragged on the
        # ragged workload (1.1 GB).
        which, _, wl = which.partition("_")
        w = workloads.WORKLOADS[{"": WORKLOAD, "long": "long_context", "ragged": "ragged"}[wl]]
        L = workloads.context_lengths(w)
        B, H, S = w.batch, w.num_kv_heads, w.page_size
        cap = L + 1
        P = workloads.pool_pages(w, cap)
        desc = kvq.Desc(1, H, w.num_q_heads, 128, w.block, S, P, B, int((cap.max() + S - 1) // S),
                        fmt)
        cache, pt = kvq.alloc_pages(desc, cap, workloads.page_order(w, P))
        ptd = torch.from_numpy(pt).to(dev)
        _fill_cache(cache, w, cap, ptd, 1, dev)
        torch.cuda.empty_cache()
        q = workloads.q_rows_torch(w, 0, device=dev)
        lens = torch.from_numpy(cap).to(dev)
        kn = workloads.kv_rows_torch(w, 0, 0, B, stream=2, device=dev)
        vn = workloads.kv_rows_torch(w, 0, 1, B, stream=2, device=dev)
        lens_before = torch.from_numpy(L).to(dev)
        torch.cuda.synchronize()
        for _ in range(calls):
            if which == "fused":
                kvq.append_decode_attention(cache, 0, kn, vn, q, lens_before, ptd)
            else:
                kvq.decode_attention(cache, 0, q, lens, ptd)
    torch.cuda.synchronize()
    assert kvq.get_device_status(cache) == 0
    cache.close()
    print(json.dumps({"kernel_case": which, "calls": calls, "ok": True}))


# ----------------------------------------------------------------------- main --
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["kvq", "reference"], default="kvq")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel-case", choices=["decode", "fused", "append", "prefill", "decode_nvfp4",
                                              "fused_nvfp4", "append_nvfp4", "prefill_nvfp4",
                                              "decode_long", "fused_long", "decode_ragged",
                                              "fused_ragged"],
                    default=None,
                    help="run one small case of one kernel (for ncu captures) and exit")
    ap.add_argument("--calls", type=int, default=3)
    args = ap.parse_args()
    if args.kernel_case:
        run_kernel_case(args.kernel_case, args.calls)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_kvq(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                v, d = oracle_sample(10.0)
                model = cpu_model()
                line["cpu_baseline"] = {"value": round(v, 4), "unit": "GB/s", "cores": 1,
                                        "kind": "oracle", "sample": d, "cpu_model": model}
                ncpu = os.cpu_count() or 1
                v, n, d = oracle_sample_threads(6.0, ncpu)
                line["cpu_baseline_all_cores"] = {"value": round(v, 4), "unit": "GB/s", "cores": n,
                                                  "kind": "oracle", "sample": d, "cpu_model": model}
                a1, d1 = oracle_append_sample(4.0, 1)
                an, dn = oracle_append_sample(4.0, ncpu)
                line["cpu_baseline_append"] = {
                    "unit": "tok/s", "kind": "oracle", "cpu_model": model,
                    "one_core": {"value": round(a1, 1), "cores": 1, "sample": d1},
                    "all_cores": {"value": round(an, 1), "cores": ncpu, "sample": dn}}
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
