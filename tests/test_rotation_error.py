"""Rotation against naive INT4 on the workloads' distributions: relative reconstruction
error of the oracle's cache rows (a check of the method's premise, not of parity).

"KVキャッシュを4ビットへ — SAW-INT4とシステムを踏まえたINT4量子化", sections
"素朴なINT4はなぜ崩れるのか" (a few outlier channels set a token's scale and crush the
other channels) and "回転のトリック — ブロック対角アダマール" (a block Hadamard rotation
spreads each outlier over its block): K and V rows of layer 0 go through the oracle's
append (rotate, quantise, page), are read back dequantised, rotated back in fp64 and
compared with the fp16 input.  Error = sum of squared errors / sum of squares."""
import numpy as np
import pytest

import oracle
import workloads

W = workloads.WORKLOADS


def relative_error(w, block, fmt, n=128):
    H, S = w.num_kv_heads, 16
    k = workloads.kv_rows(w, 0, 0, n, stream=1)
    v = workloads.kv_rows(w, 0, 1, n, stream=1)
    mp = (n + S - 1) // S
    g = oracle.Geometry(1, H, 4 * H, 128, block, S, mp, mp, fmt=fmt)
    pt = oracle.assign_pages(np.array([n], np.int32), S, mp, mp)
    pool = g.new_pool()
    oracle.rotate_quant_append(g, pool, 0, k, v, np.array([0, n], np.int32),
                               np.zeros(1, np.int32), pt)
    num = den = 0.0
    for kv, x in ((0, k), (1, v)):
        for t in range(n):
            for h in range(H):
                y = oracle.read_row(g, pool, 0, int(pt[0, t // S]), h, t % S, kv).astype(np.float64)
                xh = oracle.fwht_f64(y, block) if block > 1 else y
                xt = x[t, h].astype(np.float64)
                num += float(((xh - xt) ** 2).sum())
                den += float((xt ** 2).sum())
    return num / den


@pytest.mark.parametrize("name", ["tiny", "qwen3_4b_decode", "prefill_append"])
def test_rotation_lowers_int4_error(name):
    """Every Hadamard block beats naive INT4 at least threefold (measured: 4-12x)."""
    naive = relative_error(W[name], 1, 0)
    for block in (32, 64, 128):
        assert relative_error(W[name], block, 0) < naive / 3, block


def test_round_trip_errors_are_small():
    """Sanity of the measurement: every format and block reconstructs within a few %."""
    for block in (1, 32, 64, 128):
        for fmt in (0, 1):
            assert relative_error(W["qwen3_4b_decode"], block, fmt, n=32) < 0.08


if __name__ == "__main__":  # the table reported in the design notes
    for name in ("tiny", "qwen3_4b_decode", "prefill_append"):
        for fmt, label in ((0, "INT4"), (1, "NVFP4")):
            errs = "  ".join(f"b={b}: {relative_error(W[name], b, fmt):.2e}" for b in (1, 32, 64, 128))
            print(f"{name:16s} {label:5s} {errs}")
