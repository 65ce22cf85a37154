"""Pins of the CPU oracle against what the pages and mathematics fix (no GPU).

Each test ties an oracle function to something other than itself: the explicit
Sylvester-Hadamard matrix (scipy's construction), exact rational arithmetic, closed
forms, invariants of an orthogonal transform, numpy's own fp16 rounding, hand-worked
golden fixtures, and brute-force softmax.  A plausible mistake in the oracle -- a
dropped stage, a wrong sign or pairing, a transposed index, a wrong rounding mode, a
wrong nibble order -- fails at least one of them.

Sources: [P1] "KVキャッシュを4ビットへ — SAW-INT4とシステムを踏まえたINT4量子化"
(youngju.dev); [P2] "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World
LLM Serving" (gist.science).
"""
import os
from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import scipy.special

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BLOCKS = [2, 4, 8, 16, 32, 64, 128]


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


# ------------------------------------------------------------ rotation ------
@pytest.mark.parametrize("b", [32, 64, 128])
def test_hadamard_scale_is_nearest_fp32_to_inverse_sqrt(b):
    """c_b is the fp32 value nearest 1/sqrt(b), checked with exact arithmetic."""
    getcontext().prec = 80
    exact = Decimal(1) / Decimal(b).sqrt()
    c = oracle.hadamard_scale_f32(b)
    cands = [np.nextafter(c, np.float32(0)), c, np.nextafter(c, np.float32(1))]
    dist = [abs(Decimal(Fraction(float(x)).numerator) / Decimal(Fraction(float(x)).denominator)
                - exact) for x in cands]
    assert int(np.argmin(dist)) == 1


def _sign_matrix_from_oracle(b):
    """Columns of the oracle's transform on unit vectors, as +-1 integers.

    On a unit vector every butterfly output is +-1 or 0 exactly, so the fp32 result is
    exactly +-c_b: the sign matrix is the oracle's unnormalised Hadamard matrix."""
    c = oracle.hadamard_scale_f32(b)
    cols = []
    for j in range(b):
        e = np.zeros(b, np.float32)
        e[j] = 1.0
        y = oracle.fwht_f32(e, b)
        assert np.all(np.abs(y) == c), "unit-vector transform must be exactly +-c_b"
        cols.append(np.sign(y).astype(np.int64))
    return np.stack(cols, axis=1)


@pytest.mark.parametrize("b", BLOCKS)
def test_sylvester_matrix_orthogonality_exact(b):
    """H . H^T = b . I for the +-1 matrix, in exact integer arithmetic [P1, rotation is
    orthogonal], and H equals scipy's Sylvester construction (natural order)."""
    H = _sign_matrix_from_oracle(b)
    assert np.array_equal(H @ H.T, b * np.eye(b, dtype=np.int64))
    assert np.array_equal(H, scipy.linalg.hadamard(b).astype(np.int64))
    i = np.arange(b)
    pop = np.vectorize(lambda v: bin(int(v)).count("1"))(i[:, None] & i[None, :])
    assert np.array_equal(H, np.where(pop % 2 == 0, 1, -1))


def test_golden_fwht_e3_block32():
    rows = _golden("fwht_b32_e3.txt")
    x = np.zeros(32, np.float32)
    x[3] = 1
    y = oracle.fwht_f32(x, 32)
    c = oracle.hadamard_scale_f32(32)
    for idx, sign in rows:
        assert y[int(idx)] == np.float32(int(sign)) * c


@pytest.mark.parametrize("b", [32, 64, 128])
def test_fwht_equals_explicit_block_diagonal_matrix(b):
    """Block-diagonal transform of a 128-channel vector = explicit matrix-vector product
    with H_ij = (-1)^popcount(i&j)/sqrt(b) on each block (fp64 reference)."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal((16, 128)).astype(np.float32)
    Hn = scipy.linalg.hadamard(b) / np.sqrt(b)
    ref = np.concatenate([x[:, j:j + b].astype(np.float64) @ Hn.T for j in range(0, 128, b)], 1)
    y = oracle.fwht_f32(x, b)
    assert np.max(np.abs(y - ref)) < 4e-6
    y64 = oracle.fwht_f64(x, b)
    assert np.max(np.abs(y64 - ref)) < 1e-12


def test_fwht_blocks_are_independent():
    """Changing one block leaves the others untouched (block-diagonal, [P1])."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal(128).astype(np.float32)
    x2 = x.copy()
    x2[32:64] += 3.0
    y, y2 = oracle.fwht_f32(x, 32), oracle.fwht_f32(x2, 32)
    assert np.array_equal(y[:32], y2[:32]) and np.array_equal(y[64:], y2[64:])
    assert not np.array_equal(y[32:64], y2[32:64])


@pytest.mark.parametrize("b", [32, 64, 128])
def test_rotate_unrotate_round_trip(b):
    """The orthonormal Sylvester matrix is symmetric and its own inverse: applying the
    fp32 transform twice returns the input to 1e-6 for N(0,1) inputs [P1: exactly
    invertible]."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    back = oracle.fwht_f32(oracle.fwht_f32(x, b), b)
    assert np.max(np.abs(back - x)) <= 1e-6
    # outlier inputs: relative to the value scale
    x[:, 5] *= 50
    back = oracle.fwht_f32(oracle.fwht_f32(x, b), b)
    assert np.max(np.abs(back - x)) <= 1e-6 * np.max(np.abs(x))


@pytest.mark.parametrize("b", [32, 64, 128])
def test_inner_product_invariant(b):
    """(Hq).(Hk) = q.k: attention scores survive the rotation [P1]."""
    rng = np.random.default_rng(3)
    q = rng.standard_normal((32, 128))
    k = rng.standard_normal((32, 128))
    k[:, 9] *= 30
    lhs = np.sum(oracle.fwht_f64(q, b) * oracle.fwht_f64(k, b), -1)
    rhs = np.sum(q * k, -1)
    assert np.max(np.abs(lhs - rhs)) < 1e-10 * np.max(np.abs(rhs)) + 1e-12
    lhs32 = np.sum(oracle.fwht_f32(q.astype(np.float32), b).astype(np.float64)
                   * oracle.fwht_f32(k.astype(np.float32), b), -1)
    assert np.max(np.abs(lhs32 - rhs)) < 1e-4 * np.max(np.abs(rhs))


@pytest.mark.parametrize("b", [32, 64, 128])
def test_fwht_special_cases(b):
    """FWHT(e_0) = c_b on the whole first block; FWHT(ones on a block) = b*c_b*e_0."""
    c = oracle.hadamard_scale_f32(b)
    e = np.zeros(128, np.float32)
    e[0] = 1
    y = oracle.fwht_f32(e, b)
    assert np.all(y[:b] == c) and np.all(y[b:] == 0)
    ones = np.zeros(128, np.float32)
    ones[:b] = 1
    y = oracle.fwht_f32(ones, b)
    assert y[0] == np.float32(b) * c and np.all(y[1:] == 0)
    assert abs(float(y[0]) - np.sqrt(b)) < 1e-6 * np.sqrt(b)


def test_block_of_one_is_plain_int4():
    """b = 1 (the plain token-wise INT4 variant): the transform is the identity (no stage,
    c_1 = 1), so the appended codes are those of the unrotated row: every code is within
    s/2 of the raw value and the largest |value| maps to |code| = 7."""
    assert oracle.hadamard_scale_f32(1) == 1.0
    x = np.random.default_rng(11).standard_normal(128).astype(np.float32)
    assert np.array_equal(oracle.fwht_f32(x, 1), x)
    assert np.array_equal(oracle.fwht_f64(x.astype(np.float64), 1), x.astype(np.float64))
    x16 = x.astype(np.float16).astype(np.float32)
    bits, codes = oracle.quant_row(x16)
    s = float(np.array([bits], np.uint16).view(np.float16)[0])
    deq = codes.astype(np.float64) * s
    assert np.all(np.abs(x16 - deq) <= s / 2 + 1e-12)
    assert abs(int(codes[np.argmax(np.abs(x16))])) == 7


# ------------------------------------------------------------ fp16 -----------
def test_fp16_rounding_matches_numpy():
    """The oracle's float->fp16 is IEEE nearest-even (numpy's independent conversion),
    including ties, subnormals and overflow."""
    rng = np.random.default_rng(4)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-9, 5, 20000),
        # exact ties between fp16 neighbours: 1 + (2k+1)*2^-11
        (1.0 + (2 * np.arange(200) + 1) * 2.0 ** -11).astype(np.float32),
        np.float32([6.1e-5, 5.96e-8, 2.98e-8, 65504, 65519, 65520, -65520, 0.0, -0.0]),
    ]).astype(np.float32)
    ours = np.array([oracle.float_to_half(v) for v in vals], np.uint16)
    with np.errstate(over="ignore"):  # the overflow to +-inf is part of what is checked
        ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)
    back = np.array([oracle.half_to_float(h) for h in ref[:500]], np.float32)
    assert np.array_equal(back, ref[:500].view(np.float16).astype(np.float32))


# ------------------------------------------------------------ quantisation --
def test_golden_quant_ties():
    rows = _golden("quant_ties.txt")
    y = np.array([float(v) for v in rows[0]], np.float32)
    s, codes = oracle.quant_row(y)
    assert s == int(rows[1][0], 16)
    assert codes.tolist() == [int(v) for v in rows[2]]


def test_quant_bounds_on_random_rows():
    """|y - code*s| <= s/2, |code| <= 7 and some |code| = 7 on every non-zero row
    (invariants of the max|y|/7 scale with round-half-even) [P1, token-wise INT4]."""
    rng = np.random.default_rng(5)
    for trial in range(400):
        y = rng.standard_normal(128).astype(np.float32) * np.float32(10.0 ** rng.uniform(-3, 3))
        if trial % 3 == 0:
            y[rng.integers(128)] *= 40
        s_bits, codes = oracle.quant_row(y)
        s = np.float32(np.uint16(s_bits).view(np.float16))
        assert s > 0
        assert np.all(np.abs(codes) <= 7)
        assert np.max(np.abs(codes)) == 7
        err = np.abs(y.astype(np.float64) - codes.astype(np.float64) * float(s))
        assert np.all(err <= float(s) / 2 * (1 + 2.0 ** -20))
        # the stored scale is the fp16 rounding of max|y|/7 (numpy's fp16 rounding)
        assert s_bits == int(np.float16(np.max(np.abs(y)) / np.float32(7)).view(np.uint16))


def test_quant_degenerate_rows():
    """Zero row and a row whose scale underflows fp16 give scale 0 and all-zero codes;
    a scale above the fp16 range saturates to 65504 and codes clamp to [-8, 7]."""
    s, codes = oracle.quant_row(np.zeros(128, np.float32))
    assert s == 0 and not codes.any()
    y = np.full(128, 1e-8, np.float32)
    s, codes = oracle.quant_row(y)
    assert s == 0 and not codes.any()
    y = np.zeros(128, np.float32)
    y[0], y[1], y[2] = 540000.0, -540000.0, 65504.0
    s, codes = oracle.quant_row(y)
    assert s == 0x7BFF
    assert codes[0] == 7 and codes[1] == -8 and codes[2] == 1
    # subnormal fp16 scale still satisfies the error bound
    y = np.linspace(-1e-5, 1e-5, 128).astype(np.float32)
    s, codes = oracle.quant_row(y)
    sf = float(np.uint16(s).view(np.float16))
    assert 0 < sf < 6.1e-5
    assert np.all(np.abs(y - codes * sf) <= sf / 2 * (1 + 1e-6))


def test_quant_constant_row_closed_form():
    """y = a on every channel: m = a, s = fp16(a/7), every code = rint(a/s) = 7."""
    for a in [0.3, 1.0, 7.0, 123.4, 2000.0]:
        y = np.full(128, a, np.float32)
        s, codes = oracle.quant_row(y)
        assert np.all(codes == 7)
        assert s == int(np.float16(np.float32(a) / np.float32(7)).view(np.uint16))


def test_golden_pack_and_unpack():
    rows = _golden("pack_nibbles.txt")
    codes = np.array([int(v) for v in rows[0]], np.int8)
    packed = oracle.pack_codes(codes)
    assert packed.tolist() == [int(v, 16) for v in rows[1]]
    assert oracle.unpack_codes(packed, codes.size).tolist() == codes.tolist()
    every = np.arange(-8, 8, dtype=np.int8)
    allpairs = np.stack(np.meshgrid(every, every), -1).reshape(-1)
    assert np.array_equal(oracle.unpack_codes(oracle.pack_codes(allpairs), allpairs.size), allpairs)


# ------------------------------------------------------------ paging ---------
def test_golden_page_table():
    rows = _golden("page_table_small.txt")
    S, P, mp = (int(v) for v in rows[0])
    cap = [int(v) for v in rows[1]]
    order = [int(v) for v in rows[2]]
    pt = oracle.assign_pages(cap, S, P, mp, order)
    assert pt.tolist() == [[int(v) for v in r] for r in rows[3:]]


def test_page_assignment_properties():
    rng = np.random.default_rng(6)
    cap = rng.integers(0, 300, size=40)
    S = 16
    need = (cap + S - 1) // S
    P = int(need.sum()) + 5
    order = rng.permutation(P)
    pt = oracle.assign_pages(cap, S, P, int(need.max()), order)
    used = pt[pt >= 0]
    assert len(np.unique(used)) == used.size == need.sum()          # no page twice
    assert np.array_equal(used, order[:used.size])                  # handed out in order
    for b in range(40):
        assert np.all(pt[b, :need[b]] >= 0) and np.all(pt[b, need[b]:] == -1)
    with pytest.raises(oracle.OracleError):
        oracle.assign_pages(cap, S, int(need.sum()) - 1, int(need.max()), None)
    with pytest.raises(oracle.OracleError):
        oracle.assign_pages(cap, S, P, int(need.max()) - 1, None)


def _tiny_geometry(block=32, S=16, hkv=2, hq=8, P=12, mp=6, layers=2):
    return oracle.Geometry(layers, hkv, hq, 128, block, S, P, mp)


def test_append_index_round_trip_and_no_revisit():
    """Every appended (sequence, position) is found at page_table[b][pos/S], slot pos%S of
    its own (layer, page, head) block; rows decode back to the input within the
    quantisation bound; bytes of other tokens are never touched [P1: append without
    revisiting past tokens]."""
    g = _tiny_geometry()
    rng = np.random.default_rng(8)
    cap = np.array([40, 23, 0], np.int32)
    order = rng.permutation(g.num_pages).astype(np.int32)
    pt = oracle.assign_pages(cap, g.page_size, g.num_pages, g.max_pages_per_seq, order)
    pool = np.full(g.pool_bytes, 0xA5, np.uint8)

    lens = np.array([0, 0, 0], np.int32)
    counts = [[17, 9, 0], [23, 14, 0]]           # two appends per sequence
    written = {}
    for step, cnt in enumerate(counts):
        T = sum(cnt)
        k = (rng.standard_normal((T, 2, 128)) * 3).astype(np.float16)
        v = (rng.standard_normal((T, 2, 128))).astype(np.float16)
        k[:, :, 11] *= 25
        cu = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32)
        before = pool.copy()
        oracle.rotate_quant_append(g, pool, 1, k, v, cu, lens, pt)
        # bytes of previously written tokens unchanged
        changed = np.nonzero(before != pool)[0]
        for b in range(3):
            for i in range(cnt[b]):
                written[(b, int(lens[b]) + i)] = (k[cu[b] + i], v[cu[b] + i])
        blk = oracle.block_bytes(g.page_size, 128)
        allowed = set()
        for (b, pos) in written:
            if pos < lens[b]:
                continue
            page, slot = pt[b, pos // g.page_size], pos % g.page_size
            for h in range(2):
                base = ((1 * g.num_pages + page) * 2 + h) * blk
                for kv in range(2):
                    allowed.update(range(base + kv * 16 * 64 + slot * 64,
                                         base + kv * 16 * 64 + slot * 64 + 64))
                    allowed.update(range(base + 16 * 128 + kv * 32 + slot * 2,
                                         base + 16 * 128 + kv * 32 + slot * 2 + 2))
        assert set(changed.tolist()) <= allowed
        lens = lens + np.array(cnt, np.int32)

    for (b, pos), (kr, vr) in written.items():
        page, slot = pt[b, pos // g.page_size], pos % g.page_size
        for h in range(2):
            for kv, src in ((0, kr), (1, vr)):
                yhat = oracle.read_row(g, pool, 1, page, h, slot, kv).astype(np.float64)
                x = src[h].astype(np.float64)
                y = np.concatenate([x[j:j + 32] @ (scipy.linalg.hadamard(32) / np.sqrt(32)).T
                                    for j in range(0, 128, 32)])
                s = np.max(np.abs(y)) / 7
                # orthogonality: ||x - H^T yhat|| = ||y - yhat|| <= sqrt(D) * s/2 (+ fp16 slack)
                xback = np.concatenate([yhat[j:j + 32] @ (scipy.linalg.hadamard(32) / np.sqrt(32))
                                        for j in range(0, 128, 32)])
                assert np.linalg.norm(x - xback) <= np.sqrt(128) * s / 2 * 1.01
                assert np.max(np.abs(y - yhat)) <= s / 2 * 1.01
    # layer 0 never written
    assert np.all(pool[: g.pool_bytes // 2] == 0xA5)


def test_append_rejects_bad_page():
    g = _tiny_geometry()
    pool = g.new_pool()
    pt = np.full((1, g.max_pages_per_seq), -1, np.int32)
    pt[0, 0] = g.num_pages          # out of range
    k = np.zeros((1, 2, 128), np.float16)
    with pytest.raises(oracle.OracleError):
        oracle.rotate_quant_append(g, pool, 0, k, k, [0, 1], [0], pt)


# ------------------------------------------------------------ attention ------
def _brute_attention(q, K, V, scale):
    s = scale * (K @ q)
    p = scipy.special.softmax(s)
    return p @ V


def test_dense_attention_matches_brute_force():
    """Unquantised attention vs numpy/scipy softmax on tiny inputs (B=1, Hkv=1, G=2,
    L<=20) [P1: fused attention over the cache]."""
    rng = np.random.default_rng(9)
    for L in [1, 2, 7, 20]:
        for g in range(2):
            q = rng.standard_normal(128)
            K = rng.standard_normal((L, 128)) * 2
            V = rng.standard_normal((L, 128))
            ours = oracle.attention_dense(q, K, V, 32, rotate=0)
            ref = _brute_attention(q, K, V, 1 / np.sqrt(128))
            assert np.max(np.abs(ours - ref)) < 1e-12
            ours = oracle.attention_dense(q, K, V, 32, rotate=0, softmax_scale=0.3)
            assert np.max(np.abs(ours - _brute_attention(q, K, V, 0.3))) < 1e-12


@pytest.mark.parametrize("b", [32, 64, 128])
def test_rotated_domain_attention_equals_unrotated(b):
    """Attention with q rotated, K/V stored rotated and the output unrotated equals
    plain attention (orthogonality, [P1])."""
    rng = np.random.default_rng(10)
    L = 13
    q = rng.standard_normal(128)
    K = rng.standard_normal((L, 128))
    V = rng.standard_normal((L, 128))
    K[:, 3] *= 20
    Hn = scipy.linalg.block_diag(*[scipy.linalg.hadamard(b) / np.sqrt(b)] * (128 // b))
    ours = oracle.attention_dense(q, K @ Hn.T, V @ Hn.T, b, rotate=1)
    ref = _brute_attention(q, K, V, 1 / np.sqrt(128))
    assert np.max(np.abs(ours - ref)) < 1e-12


def test_attention_special_cases():
    """L = 1 -> out = v; equal scores (q = 0) -> mean of V; empty -> zeros."""
    rng = np.random.default_rng(11)
    v = rng.standard_normal((1, 128))
    out = oracle.attention_dense(rng.standard_normal(128), rng.standard_normal((1, 128)), v, 32, 0)
    assert np.allclose(out, v[0], atol=1e-14)
    V = rng.standard_normal((9, 128))
    out = oracle.attention_dense(np.zeros(128), rng.standard_normal((9, 128)), V, 32, 0)
    assert np.allclose(out, V.mean(0), atol=1e-14)
    out = oracle.attention_dense(np.ones(128), np.zeros((0, 128)), np.zeros((0, 128)), 32, 0)
    assert not out.any()


def test_cache_decode_equals_dense_attention_on_dequantised_rows():
    """The paged decode reads exactly the dequantised rows at page_table[b][t/S], slot t%S
    (GQA: query head hq uses KV head hq // G), and is the rotated-domain dense attention
    on them; L = 1 gives the unrotated dequantised v."""
    g = _tiny_geometry(block=64, S=16, hkv=2, hq=8, P=8, mp=4, layers=1)
    rng = np.random.default_rng(12)
    cap = np.array([50, 1], np.int32)
    pt = oracle.assign_pages(cap, 16, 8, 4, rng.permutation(8).astype(np.int32))
    pool = g.new_pool()
    k = rng.standard_normal((51, 2, 128)).astype(np.float16)
    v = rng.standard_normal((51, 2, 128)).astype(np.float16)
    oracle.rotate_quant_append(g, pool, 0, k, v, np.array([0, 50, 51], np.int32),
                               np.array([0, 0], np.int32), pt)
    lens = cap
    q = rng.standard_normal((2, 8, 128)).astype(np.float16)
    out = oracle.decode_attention(g, pool, 0, q, lens, pt)
    for b in range(2):
        for hq in range(8):
            h = hq // 4
            K = np.stack([oracle.read_row(g, pool, 0, pt[b, t // 16], h, t % 16, 0)
                          for t in range(lens[b])]).astype(np.float64)
            V = np.stack([oracle.read_row(g, pool, 0, pt[b, t // 16], h, t % 16, 1)
                          for t in range(lens[b])]).astype(np.float64)
            ref = oracle.attention_dense(q[b, hq].astype(np.float64), K, V, 64, rotate=1)
            assert np.max(np.abs(out[b, hq] - ref)) < 1e-12
    # L = 1: output is the unrotated dequantised value row
    vhat = oracle.read_row(g, pool, 0, pt[1, 0], 0, 0, 1).astype(np.float64)
    Hn = scipy.linalg.block_diag(*[scipy.linalg.hadamard(64) / 8.0] * 2)
    assert np.max(np.abs(out[1, 0] - Hn @ vhat)) < 1e-12


def _numpy_rows(pool, g, layer, page, head, slot, kv):
    """Dequantised cache row read straight from the pool bytes (independent of the oracle's
    reader): nibbles low = even channel, two's complement, times the fp16 scale."""
    S, D = g.page_size, g.head_dim
    blk = S * (D + 4)
    base = ((layer * g.num_pages + page) * g.num_kv_heads + head) * blk
    b = pool[base + kv * S * (D // 2) + slot * (D // 2):][:D // 2].astype(np.int16)
    codes = np.empty(D, np.int16)
    codes[0::2] = b & 0xF
    codes[1::2] = b >> 4
    codes = np.where(codes >= 8, codes - 16, codes)
    s = pool[base + S * D + kv * S * 2 + slot * 2:][:2].view(np.float16)[0]
    return codes.astype(np.float64) * float(s)


def test_prefill_attention_is_causal_attention_on_the_cache():
    """Chunked prefill: query i of sequence b's chunk (position L_b - C_b + i) attends
    exactly cache positions 0..p.  Brute force in numpy (rows read from the pool bytes,
    scipy's Hadamard, explicit softmax) on a tiny ragged case with a chunk of the whole
    sequence, a partial chunk, one query, and an empty chunk."""
    g = _tiny_geometry(block=32, S=16, hkv=2, hq=4, P=16, mp=4, layers=1)
    rng = np.random.default_rng(21)
    cap = np.array([37, 20, 9, 5], np.int32)
    pt = oracle.assign_pages(cap, 16, 16, 4, rng.permutation(16).astype(np.int32))
    pool = g.new_pool()
    n = int(cap.sum())
    k = rng.standard_normal((n, 2, 128)).astype(np.float16)
    v = rng.standard_normal((n, 2, 128)).astype(np.float16)
    oracle.rotate_quant_append(g, pool, 0, k, v, np.concatenate([[0], np.cumsum(cap)]).astype(np.int32),
                               np.zeros(4, np.int32), pt)
    chunks = np.array([37, 7, 1, 0], np.int32)
    cu = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    q = rng.standard_normal((int(cu[-1]), 4, 128)).astype(np.float16)
    out = oracle.prefill_attention(g, pool, 0, q, cu, cap, pt, softmax_scale=0.07)
    Hn = scipy.linalg.block_diag(*[scipy.linalg.hadamard(32) / np.sqrt(32.0)] * 4)
    for b in range(4):
        for i in range(chunks[b]):
            pos = cap[b] - chunks[b] + i
            for hq in range(4):
                h = hq // 2
                K = np.stack([_numpy_rows(pool, g, 0, pt[b, t // 16], h, t % 16, 0) for t in range(pos + 1)])
                V = np.stack([_numpy_rows(pool, g, 0, pt[b, t // 16], h, t % 16, 1) for t in range(pos + 1)])
                qr = Hn @ q[cu[b] + i, hq].astype(np.float64)
                sc = 0.07 * (K @ qr)
                p = np.exp(sc - sc.max())
                p /= p.sum()
                ref = Hn @ (p @ V)
                assert np.max(np.abs(out[cu[b] + i, hq] - ref)) < 1e-10, (b, i, hq)


def test_prefill_attention_reduces_to_decode():
    """A chunk of one query is decode over L_b; the last query of a longer chunk too."""
    g = _tiny_geometry(block=64, S=16, hkv=2, hq=8, P=8, mp=4, layers=1)
    rng = np.random.default_rng(22)
    cap = np.array([50, 3], np.int32)
    pt = oracle.assign_pages(cap, 16, 8, 4)
    pool = g.new_pool()
    k = rng.standard_normal((53, 2, 128)).astype(np.float16)
    v = rng.standard_normal((53, 2, 128)).astype(np.float16)
    oracle.rotate_quant_append(g, pool, 0, k, v, np.array([0, 50, 53], np.int32),
                               np.zeros(2, np.int32), pt)
    qd = rng.standard_normal((2, 8, 128)).astype(np.float16)
    dec = oracle.decode_attention(g, pool, 0, qd, cap, pt)
    one = oracle.prefill_attention(g, pool, 0, qd, np.array([0, 1, 2], np.int32), cap, pt)
    assert np.array_equal(one, dec)
    qc = rng.standard_normal((9, 8, 128)).astype(np.float16)
    qc[5] = qd[0]
    qc[8] = qd[1]
    chunk = oracle.prefill_attention(g, pool, 0, qc, np.array([0, 6, 9], np.int32), cap, pt)
    assert np.array_equal(chunk[5], dec[0]) and np.array_equal(chunk[8], dec[1])
