"""Pins of the oracle's NVFP4 cache format (fmt = 1) against things other than itself.

"BitDecoding-FP4:FP4 KVキャッシュのネイティブ復号" (sns.style), sections "背景と概要" and
"深掘り分析": NVFP4 is a 4-bit microscaling format with E4M3 block scales.  The readings
(E2M1 elements, 16 channels per block, scale = E4M3(amax / 6), codes = E2M1(y * (1/s)))
are stated in the oracle.  Pins:

* E4M3 decoding of every code and E4M3 rounding of many values, against torch's
  float8_e4m3fn (a library routine; torch rounds to nearest even and turns values past
  the top into NaN, so values are clamped to 448 first, the saturating reading);
* E2M1 values and rounding of hand-computed cases written from the format definition
  (sign, 2 exponent bits with bias 1, 1 mantissa bit; ties to the even code);
* lossless rows: values that are E2M1 values times an E4M3 scale, with the block maximum
  at 6 s, come back exactly; a zero block gives scale 0 and codes 0;
* the paged store: block size, and decode attention over a cache of lossless rows (b = 1)
  equal to plain fp64 attention on the original values.
"""
import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")


def test_e4m3_decode_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    for c in range(256):
        if np.isnan(ref[c]):
            continue
        assert oracle.e4m3_to_float(c) == ref[c], c


def test_e4m3_rounding_matches_torch():
    rng = np.random.default_rng(7)
    x = np.exp2(rng.uniform(-12, 10, 4000)).astype(np.float32)
    # every midpoint between neighbouring positive codes: exact ties
    vals = np.array([oracle.e4m3_to_float(c) for c in range(127)], np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, np.float32([0.0, 448.0, 460.0, 464.0, 1e6])])
    x = np.concatenate([x, -x])  # the sign is kept (-0 included)
    ref = torch.from_numpy(np.clip(x, -448.0, 448.0).astype(np.float32)).to(torch.float8_e4m3fn)
    ref = ref.view(torch.uint8).numpy()
    got = np.array([oracle.float_to_e4m3(float(v)) for v in x], np.uint8)
    assert np.array_equal(got, ref), np.nonzero(got != ref)[0][:10]


def test_e2m1_values_and_rounding():
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(16):
        assert oracle.e2m1_to_float(c) == (-1.0 if c & 8 else 1.0) * mags[c & 7]
    # exact values, midpoints (ties to the even code), saturation, signs
    cases = {0.0: 0, 0.5: 1, 6.0: 7, 0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6,
             5.0: 6, 0.3: 1, 0.74: 1, 2.6: 5, 4.9: 6, 5.1: 7, 7.0: 7, 1e9: 7,
             -0.1: 8, -0.3: 9, -2.5: 12, -5.1: 15, -100.0: 15}
    for x, c in cases.items():
        assert oracle.float_to_e2m1(x) == c, (x, c)


def test_quant_row_nvfp4_lossless_and_zero():
    rng = np.random.default_rng(8)
    mags = np.float32([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    for _ in range(50):
        y = np.zeros(128, np.float32)
        scales = rng.integers(8, 120, 8)   # normal E4M3 codes
        want_codes = np.zeros(128, np.uint8)
        for blk in range(8):
            s = oracle.e4m3_to_float(int(scales[blk]))
            idx = rng.integers(0, 8, 16)
            idx[rng.integers(0, 16)] = 7    # the block maximum is 6 s
            sign = rng.integers(0, 2, 16)
            idx = np.where(idx == 0, 0, idx)
            sign = np.where(idx == 0, 0, sign)
            y[16 * blk:16 * blk + 16] = np.where(sign, -1, 1) * mags[idx] * np.float32(s)
            want_codes[16 * blk:16 * blk + 16] = (sign << 3) | idx
        codes, sc = oracle.quant_row_nvfp4(y)
        assert np.array_equal(sc, scales.astype(np.uint8))
        assert np.array_equal(codes, want_codes)
    codes, sc = oracle.quant_row_nvfp4(np.zeros(128, np.float32))
    assert not codes.any() and not sc.any()


def test_quant_row_nvfp4_error_bound():
    """|y - code * s| is at most half the E2M1 spacing at |y / s| (times s), plus the
    saturation excess above 6 s."""
    rng = np.random.default_rng(9)
    for _ in range(40):
        y = (rng.standard_t(3, 128) * rng.choice([1e-3, 1.0, 40.0])).astype(np.float32)
        codes, sc = oracle.quant_row_nvfp4(y)
        for blk in range(8):
            s = oracle.e4m3_to_float(int(sc[blk]))
            if s == 0.0:  # amax / 6 rounds to zero: at most half the smallest E4M3 step
                amax = float(np.abs(y[16 * blk:16 * blk + 16]).max())
                assert amax / 6 <= 2.0 ** -10 and not codes[16 * blk:16 * blk + 16].any()
                continue
            for i in range(16 * blk, 16 * blk + 16):
                t = abs(float(y[i])) / s
                half = 0.25 if t <= 2 else (0.5 if t <= 4 else 1.0)
                err = abs(float(y[i]) - oracle.e2m1_to_float(int(codes[i])) * s)
                assert err <= (half + max(0.0, t - 6.0) + 1e-6) * s + 1e-30, (i, t, err)


def test_block_bytes_nvfp4():
    assert oracle.block_bytes(16, 128, 1) == 16 * 144
    assert oracle.block_bytes(64, 128, 1) == 64 * 144
    assert oracle.block_bytes(16, 128, 0) == 16 * 132


def test_nvfp4_decode_is_dense_attention_on_lossless_rows():
    """b = 1 (no rotation): rows that NVFP4 stores exactly give plain softmax attention."""
    rng = np.random.default_rng(10)
    H, G, S, L = 2, 4, 16, 37
    mags = np.float32([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])

    def lossless_rows(n):
        out = np.zeros((n, H, 128), np.float32)
        for t in range(n):
            for h in range(H):
                for blk in range(8):
                    s = oracle.e4m3_to_float(int(rng.integers(40, 64)))  # 1/16 .. 1/2: fp16-exact
                    idx = rng.integers(0, 8, 16)
                    idx[0] = 7
                    sign = np.where(rng.integers(0, 2, 16) == 1, -1.0, 1.0)
                    out[t, h, 16 * blk:16 * blk + 16] = sign * mags[idx] * s
        return out

    k = lossless_rows(L)
    v = lossless_rows(L)
    assert np.array_equal(k.astype(np.float16).astype(np.float32), k)
    P = 4
    g = oracle.Geometry(1, H, H * G, 128, 1, S, P, P, fmt=1)
    pool = g.new_pool()
    pt = oracle.assign_pages(np.array([L], np.int32), S, P, P)
    oracle.rotate_quant_append(g, pool, 0, k.astype(np.float16), v.astype(np.float16),
                               np.array([0, L], np.int32), np.array([0], np.int32), pt)
    for t in (0, 17, L - 1):
        for kv, src in ((0, k), (1, v)):
            row = oracle.read_row(g, pool, 0, int(pt[0, t // S]), 1, t % S, kv)
            assert np.array_equal(row, src[t, 1])
    q = rng.standard_normal((1, H * G, 128)).astype(np.float16)
    out = oracle.decode_attention(g, pool, 0, q, np.array([L], np.int32), pt)
    for hq in range(H * G):
        ref = oracle.attention_dense(q[0, hq].astype(np.float64), k[:, hq // G].astype(np.float64),
                                     v[:, hq // G].astype(np.float64), 1, 0)
        np.testing.assert_allclose(out[0, hq], ref, rtol=1e-12, atol=1e-12)


def test_nvfp4_pool_bytes_follow_the_documented_layout():
    """The oracle's NVFP4 append writes exactly what the header's pool layout says: an
    expected pool built here byte by byte -- block ((layer*P + page)*Hkv + head)*S*144,
    codes of slot s at kv*S*64 + s*64 (low nibble = even channel), the 8 E4M3 block scales
    at S*128 + kv*S*8 + s*8 -- from the row quantiser applied to the rotated rows, equals
    the oracle's pool (other layers and unused slots stay zero); and reading the bytes back
    with a table of E2M1 values and torch's E4M3 gives the oracle's dequantised rows."""
    rng = np.random.default_rng(11)
    L, H, Hq, b, S, P, mp, layer = 2, 2, 8, 32, 16, 8, 4, 1
    g = oracle.Geometry(L, H, Hq, 128, b, S, P, mp, fmt=1)
    cap = np.array([37, 5], np.int32)
    pt = oracle.assign_pages(cap, S, P, mp, rng.permutation(P).astype(np.int32))
    n = int(cap.sum())
    k = (rng.standard_t(3, (n, H, 128)) * 3).astype(np.float16)
    v = rng.standard_normal((n, H, 128)).astype(np.float16)
    cu = np.array([0, 37, 42], np.int32)
    pool = g.new_pool()
    oracle.rotate_quant_append(g, pool, layer, k, v, cu, np.zeros(2, np.int32), pt)

    want = np.zeros_like(pool)
    R = 144
    for seq in range(2):
        for pos in range(int(cap[seq])):
            page, slot = int(pt[seq, pos // S]), pos % S
            for h in range(H):
                base = ((layer * P + page) * H + h) * S * R
                for kv, src in ((0, k), (1, v)):
                    y = oracle.fwht_f32(src[cu[seq] + pos, h].astype(np.float32), b)
                    codes, sc = oracle.quant_row_nvfp4(y)
                    codes = codes.astype(np.uint8)
                    packed = (codes[0::2] & 0xF) | ((codes[1::2] & 0xF) << 4)
                    o = base + kv * S * 64 + slot * 64
                    want[o:o + 64] = packed
                    o = base + S * 128 + kv * S * 8 + slot * 8
                    want[o:o + 8] = sc
    assert np.array_equal(pool, want)

    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    for seq, pos, h, kv in ((0, 0, 0, 0), (0, 36, 1, 1), (1, 4, 1, 0), (0, 17, 0, 1)):
        page, slot = int(pt[seq, pos // S]), pos % S
        base = ((layer * P + page) * H + h) * S * R
        byt = pool[base + kv * S * 64 + slot * 64:][:64]
        c = np.empty(128, np.int64)
        c[0::2] = byt & 0xF
        c[1::2] = byt >> 4
        vals = np.where(c & 8, -1.0, 1.0) * mags[c & 7]
        sc = pool[base + S * 128 + kv * S * 8 + slot * 8:][:8].copy()
        s = torch.from_numpy(sc).view(torch.float8_e4m3fn).double().numpy()
        row = vals * np.repeat(s, 16)
        assert np.array_equal(row, oracle.read_row(g, pool, layer, page, h, slot, kv).astype(np.float64))
