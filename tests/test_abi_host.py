"""C-ABI library checks that need no GPU: it loads, exports every symbol the header
declares, its host-only page allocator is bit-exact with the oracle's, and argument errors
are reported before any CUDA call."""
import ctypes
import os
import re

import numpy as np
import pytest

import bit_paged_kv_diag_b200 as kvq
import oracle
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(kvq_\w+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    L = kvq.lib()
    declared = _declared_symbols()
    assert declared, "no declarations found"
    assert declared == set(kvq.EXPORTED)
    for name in declared:
        assert hasattr(L, name), name


def _desc(**kw):
    base = dict(num_layers=2, num_kv_heads=8, num_q_heads=32, head_dim=128, hadamard_block=128,
                page_size=16, num_pages=100, max_batch=16, max_pages_per_seq=20)
    base.update(kw)
    return kvq.Desc(**base)


def test_pool_bytes_and_descriptor_validation():
    d = _desc()
    assert kvq.pool_bytes(d) == 2 * 100 * 8 * 16 * 132
    assert kvq.pool_bytes(_desc(hadamard_block=1)) == 2 * 100 * 8 * 16 * 132  # plain INT4
    # NVFP4: 64 B codes + 8 E4M3 scale bytes per K and per V row
    assert kvq.pool_bytes(_desc(kv_format=kvq.FORMAT_NVFP4)) == 2 * 100 * 8 * 16 * 144
    import oracle
    assert 144 * 16 == oracle.block_bytes(16, 128, 1)
    for bad in [dict(head_dim=64), dict(hadamard_block=16), dict(hadamard_block=2),
                dict(page_size=24), dict(kv_format=2), dict(kv_format=-1),
                dict(num_q_heads=24), dict(num_q_heads=48), dict(max_batch=5000),
                dict(num_layers=0), dict(num_pages=0)]:
        assert kvq.pool_bytes(_desc(**bad)) == 0, bad


@pytest.mark.parametrize("name", ["tiny", "qwen3_4b_decode", "long_context", "ragged",
                                  "prefill_append"])
def test_page_assignment_bit_exact_with_oracle(name):
    w = workloads.WORKLOADS[name]
    lens = workloads.context_lengths(w) + w.new_tokens
    P = workloads.pool_pages(w, lens)
    mp = int(((lens.astype(np.int64) + w.page_size - 1) // w.page_size).max())
    d = _desc(num_kv_heads=w.num_kv_heads, num_q_heads=w.num_q_heads, hadamard_block=w.block,
              page_size=w.page_size, num_pages=P, max_batch=w.batch, max_pages_per_seq=mp)
    order = workloads.page_order(w, P)
    ours = kvq.assign_pages(d, lens, order)
    ref = oracle.assign_pages(lens, w.page_size, P, mp, order)
    assert np.array_equal(ours, ref)


def test_page_assignment_random_and_errors():
    rng = np.random.default_rng(0)
    for trial in range(50):
        B = int(rng.integers(1, 40))
        S = int(rng.choice([16, 32, 64, 128, 256]))
        cap = rng.integers(0, 2000, size=B).astype(np.int32)
        need = (cap + S - 1) // S
        P = int(need.sum()) + int(rng.integers(0, 10))
        mp = int(need.max()) + int(rng.integers(0, 3))
        order = rng.permutation(max(P, 1)).astype(np.int32) if trial % 2 else None
        d = _desc(page_size=S, num_pages=max(P, 1), max_batch=B, max_pages_per_seq=max(mp, 1))
        ours = kvq.assign_pages(d, cap, order)
        ref = oracle.assign_pages(cap, S, max(P, 1), max(mp, 1), order)
        assert np.array_equal(ours, ref)
    d = _desc(num_pages=3, max_pages_per_seq=4, max_batch=2)
    with pytest.raises(kvq.KVQError) as e:
        kvq.assign_pages(d, [40, 40])                       # 3 + 3 pages > 3
    assert e.value.status == kvq.KVQ_ENOPAGES
    with pytest.raises(kvq.KVQError) as e:
        kvq.assign_pages(d, [65])                           # 5 pages > 4 per sequence
    assert e.value.status == kvq.KVQ_ENOPAGES
    with pytest.raises(kvq.KVQError) as e:
        kvq.assign_pages(d, [-1])
    assert e.value.status == kvq.KVQ_EINVAL


def test_calls_reject_bad_arguments_before_any_cuda_call():
    L = kvq.lib()
    d = _desc()
    h = ctypes.c_void_p()
    # unsupported descriptor, null out pointer, misaligned caller pool: host-side errors
    assert L.kvq_alloc_pages(ctypes.byref(_desc(head_dim=96)), None, 0, 0, None, None, None,
                             ctypes.byref(h)) == kvq.KVQ_EUNSUPPORTED
    assert L.kvq_alloc_pages(ctypes.byref(d), None, 0, 0, None, None, None, None) == kvq.KVQ_EINVAL
    assert L.kvq_alloc_pages(ctypes.byref(d), 0x1003, 1 << 40, 0, None, None, None,
                             ctypes.byref(h)) == kvq.KVQ_EINVAL
    assert L.kvq_rotate_quant_append(None, 0, None, None, None, None, None, 0, 0, None) == kvq.KVQ_EINVAL
    assert L.kvq_decode_attention(None, 0, None, None, None, 0, 0.0, None, None) == kvq.KVQ_EINVAL
    assert L.kvq_append_decode_attention(None, 0, None, None, None, None, None, 0, 0.0, None,
                                         None) == kvq.KVQ_EINVAL
    assert L.kvq_prefill_attention(None, 0, None, None, None, None, 0, 0, 0.0, None,
                                   None) == kvq.KVQ_EINVAL
    assert L.kvq_free(None) == kvq.KVQ_OK
    assert L.kvq_pool_ptr(None) is None
    assert kvq.status_string(kvq.KVQ_ENOPAGES) == "not enough pages"


def test_noalloc_decode_rejects_bad_arguments_before_any_cuda_call():
    """The allocation-free decode checks its descriptor, pool size, layer, batch, scale,
    pointers, alignment and the fixed scratch's unit limit before its first CUDA call."""
    L = kvq.lib()
    d = _desc()
    ok = 0x10000  # 16-byte aligned stand-ins; nothing is dereferenced on these paths
    need = kvq.pool_bytes(d)
    args = lambda **kw: dict(dict(d=ctypes.byref(d), pool=ok, nbytes=need, layer=0, q=ok,  # noqa: E731
                                  lens=ok, pt=ok, batch=4, scale=0.0, out=ok, st=None), **kw)

    def call(a):
        return L.kvq_decode_attention_noalloc(a["d"], a["pool"], a["nbytes"], a["layer"], a["q"],
                                              a["lens"], a["pt"], a["batch"], a["scale"], a["out"],
                                              a["st"], None)

    assert call(args(d=None)) == kvq.KVQ_EINVAL
    for bad in (dict(head_dim=96), dict(num_q_heads=24), dict(hadamard_block=16),
                dict(page_size=8), dict(kv_format=2), dict(max_batch=5000)):
        assert call(args(d=ctypes.byref(_desc(**bad)))) == kvq.KVQ_EUNSUPPORTED, bad
    assert call(args(d=ctypes.byref(_desc(num_layers=0)))) == kvq.KVQ_EINVAL
    assert call(args(layer=2)) == kvq.KVQ_EINVAL
    assert call(args(layer=-1)) == kvq.KVQ_EINVAL
    assert call(args(batch=17)) == kvq.KVQ_EINVAL
    assert call(args(batch=-1)) == kvq.KVQ_EINVAL
    assert call(args(scale=-1.0)) == kvq.KVQ_EINVAL
    assert call(args(scale=float("inf"))) == kvq.KVQ_EINVAL
    assert call(args(scale=float("nan"))) == kvq.KVQ_EINVAL
    assert call(args(batch=0, q=None)) == kvq.KVQ_OK  # nothing to do
    for name in ("pool", "q", "lens", "pt", "out"):
        assert call(args(**{name: None})) == kvq.KVQ_EINVAL, name
    for name in ("pool", "q", "out"):
        assert call(args(**{name: ok + 8})) == kvq.KVQ_EINVAL, name
    assert call(args(st=ok + 2)) == kvq.KVQ_EINVAL          # misaligned status word
    # a pool smaller than the descriptor's layers: rejected before the kernel could read
    # past its end
    assert call(args(nbytes=need - 1)) == kvq.KVQ_EINVAL
    assert call(args(nbytes=0)) == kvq.KVQ_EINVAL
    big = _desc(num_kv_heads=8, num_q_heads=8, max_batch=4096)
    assert call(args(d=ctypes.byref(big), nbytes=kvq.pool_bytes(big),
                     batch=513)) == kvq.KVQ_EUNSUPPORTED  # 513 * 8 units > the counter array
