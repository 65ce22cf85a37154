"""The seeded input recipes (workloads/) against their stated distributions.

Determinism and independent streams, and the statistics each recipe plants: the numpy
draws that the oracle and the parity tests share, and the torch draws of the full-size
runs (drawn here on the CPU)."""
import numpy as np
import pytest
import scipy.stats

import workloads

W = workloads.WORKLOADS
N = 4096  # tokens per statistical check


def _rows(w, layer, kv, n, torch_draw):
    if torch_draw:
        return workloads.kv_rows_torch(w, layer, kv, n, device="cpu").numpy()
    return workloads.kv_rows(w, layer, kv, n)


def _channel_rms(x):
    return np.sqrt((x.astype(np.float64) ** 2).mean(0))  # [H][D]


def test_draws_are_deterministic_and_streams_independent():
    w = W["qwen3_4b_decode"]
    a = workloads.kv_rows(w, 0, 0, 64, stream=1)
    assert a.dtype == np.float16 and a.shape == (64, 8, 128) and np.isfinite(a).all()
    assert np.array_equal(a, workloads.kv_rows(w, 0, 0, 64, stream=1))
    for other in (workloads.kv_rows(w, 0, 0, 64, stream=2), workloads.kv_rows(w, 1, 0, 64, stream=1),
                  workloads.kv_rows(w, 0, 1, 64, stream=1)):
        assert not np.array_equal(a, other)
    q = workloads.q_rows(w, 0)
    assert q.shape == (16, 32, 128) and np.array_equal(q, workloads.q_rows(w, 0))
    assert not np.array_equal(q, workloads.q_rows(w, 1))
    lens = workloads.context_lengths(W["ragged"])
    assert np.array_equal(lens, workloads.context_lengths(W["ragged"]))
    assert lens.shape == (256,) and lens.min() >= 128 and lens.max() <= 8192
    assert np.array_equal(workloads.cu_seqlens([3, 0, 5]), [0, 3, 3, 8])


@pytest.mark.parametrize("torch_draw", [False, True])
def test_fixed_outliers(torch_draw):
    """tiny: per KV head 4 channels x 20, the same channels in every layer; N(0,1) else."""
    w = W["tiny"]
    sets = []
    for layer in (0, 1):
        rms = _channel_rms(_rows(w, layer, 0, N, torch_draw))
        for h in range(w.num_kv_heads):
            big = np.sort(np.argsort(rms[h])[-4:])
            assert np.all((rms[h, big] > 18.5) & (rms[h, big] < 21.5))
            assert np.all(np.abs(np.delete(rms[h], big) - 1.0) < 0.08)
            sets.append((layer, h, tuple(big)))
    assert [s[2] for s in sets if s[0] == 0] == [s[2] for s in sets if s[0] == 1]


@pytest.mark.parametrize("torch_draw", [False, True])
def test_lognormal_outliers(torch_draw):
    """qwen3_4b_decode: per (layer, KV head, K|V) one channel x exp(U[ln 10, ln 50]);
    each row x LogNormal(0, 0.5)."""
    w = W["qwen3_4b_decode"]
    for kv in (0, 1):
        x = _rows(w, 0, kv, N, torch_draw).astype(np.float64)
        rms = _channel_rms(x)
        for h in range(w.num_kv_heads):
            ratio = rms[h] / np.median(rms[h])
            big = np.nonzero(ratio > 5)[0]
            assert big.size == 1 and 9.0 < ratio[big[0]] < 55.0, ratio[big]
        # row scale: log RMS of a row's ordinary channels has the LogNormal's sigma 0.5
        mask = np.ones((w.num_kv_heads, 128), bool)
        for h in range(w.num_kv_heads):
            mask[h, np.argmax(rms[h])] = False
        row_rms = np.sqrt(np.stack([(x[:, h, mask[h]] ** 2).mean(1) for h in range(w.num_kv_heads)]))
        assert 0.46 < np.log(row_rms).std() < 0.55


@pytest.mark.parametrize("torch_draw", [False, True])
def test_student_t3(torch_draw):
    """prefill_append: iid Student-t(3): its median |x| and tail mass."""
    w = W["prefill_append"]
    x = np.abs(_rows(w, 0, 0, N, torch_draw).astype(np.float64)).ravel()
    t3 = scipy.stats.t(3)
    assert abs(np.median(x) - t3.ppf(0.75)) < 0.01
    tail = float((x > 5).mean())
    assert abs(tail - 2 * t3.sf(5)) < 0.001
