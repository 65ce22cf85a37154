"""Seeded synthetic workloads for the rotated-INT4 paged KV cache.

This module holds only the INPUT recipes: shapes, seeds and value distributions.  It
contains none of the method's arithmetic (no rotation, quantisation, paging or
attention), so both the CUDA path and the CPU oracle may draw from it.

The five workloads follow the model shapes of the pages' setting (a Qwen3-4B-shaped
decoder, long-context and high-concurrency serving, and a prefill stress); no public
benchmark, evaluation suite or dataset is used -- these synthetic arrays stand in for
real K/V activations.  Values are drawn in fp64 by numpy's PCG64 generator, clamped to
the fp16 range and rounded to fp16 (nearest-even).

Recipe per distribution (per K and per V separately):

* ``fixed_outliers``  N(0,1); per KV head, 4 channels drawn once are multiplied by 20.
* ``lognormal_outliers``  N(0,1); per (layer, KV head, K|V), max(1, round(1% of D))
  channels are multiplied by exp(U[ln 10, ln 50]); each (token, KV head, K|V) row is
  multiplied by an RMS factor drawn from LogNormal(0, 0.5).
* ``student_t3``  iid Student-t with 3 degrees of freedom per element.

q is N(0,1) in every workload.
"""
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

HEAD_DIM = 128


@dataclass
class Workload:
    name: str
    num_layers: int
    batch: int
    num_kv_heads: int
    num_q_heads: int
    block: int                     # Hadamard block b
    page_size: int                 # S
    dist: str
    seed: int
    context: Optional[List[int]] = None     # tokens already in the cache (decode workloads)
    new_tokens: int = 1                     # tokens appended per sequence per step
    ragged: Optional[tuple] = None          # (lo, hi) inclusive uniform lengths
    pool_factor: float = 1.0                # pool pages = ceil(factor * pages needed)
    permute_pages: bool = False
    blocks_sweep: List[int] = field(default_factory=list)
    head_dim: int = HEAD_DIM

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


WORKLOADS = {
    # Tiny: latency and parity only.
    "tiny": Workload("tiny", num_layers=1, batch=1, num_kv_heads=2, num_q_heads=8, block=32,
                     page_size=16, dist="fixed_outliers", seed=0, context=[256], new_tokens=1),
    # Qwen3-4B-shaped decode: 36 layers, 16 sequences of 4096 tokens.
    "qwen3_4b_decode": Workload("qwen3_4b_decode", num_layers=36, batch=16, num_kv_heads=8,
                                num_q_heads=32, block=128, page_size=16,
                                dist="lognormal_outliers", seed=1, context=[4096] * 16,
                                new_tokens=1),
    # Long context: one layer of four sequences up to 128K tokens.
    "long_context": Workload("long_context", num_layers=1, batch=4, num_kv_heads=4,
                             num_q_heads=32, block=64, page_size=64,
                             dist="lognormal_outliers", seed=2,
                             context=[32768, 65536, 131072, 131072], new_tokens=1),
    # High concurrency, ragged lengths, pages scattered through a 1.2x pool.
    "ragged": Workload("ragged", num_layers=1, batch=256, num_kv_heads=8, num_q_heads=32,
                       block=128, page_size=16, dist="lognormal_outliers", seed=3,
                       ragged=(128, 8192), new_tokens=1, pool_factor=1.2, permute_pages=True),
    # Chunked prefill on the Qwen3-4B shape: 16 sequences, a 512-token chunk appended after
    # 3584 cached tokens, the chunk's queries attending causally.
    "chunked_prefill": Workload("chunked_prefill", num_layers=2, batch=16, num_kv_heads=8,
                                num_q_heads=32, block=128, page_size=16,
                                dist="lognormal_outliers", seed=5, context=[3584] * 16,
                                new_tokens=512),
    # Prefill-append stress: 8 x 8192 new tokens in one call, b swept over 32/64/128.
    "prefill_append": Workload("prefill_append", num_layers=1, batch=8, num_kv_heads=8,
                               num_q_heads=32, block=128, page_size=16, dist="student_t3",
                               seed=4, context=[0] * 8, new_tokens=8192,
                               blocks_sweep=[32, 64, 128]),
}


def rng_for(w: Workload, *stream) -> np.random.Generator:
    """Independent generator for a named stream of a workload (seed, then stream ids)."""
    return np.random.default_rng([w.seed, *[int(s) for s in stream]])


# Stream ids (fixed; changing them changes every input).
_S_LENGTHS, _S_PAGES, _S_CHANNELS, _S_KV, _S_Q = 1, 2, 3, 4, 5


def context_lengths(w: Workload) -> np.ndarray:
    """Tokens already cached per sequence before the step's append."""
    if w.ragged is not None:
        lo, hi = w.ragged
        return rng_for(w, _S_LENGTHS).integers(lo, hi + 1, size=w.batch).astype(np.int32)
    return np.asarray(w.context, np.int32)


def pages_needed(lengths, page_size: int) -> int:
    lengths = np.asarray(lengths, np.int64)
    return int(((lengths + page_size - 1) // page_size).sum())


def pool_pages(w: Workload, capacity) -> int:
    need = pages_needed(capacity, w.page_size)
    return int(np.ceil(w.pool_factor * need)) if w.pool_factor != 1.0 else need


def page_order(w: Workload, num_pages: int) -> Optional[np.ndarray]:
    """Order in which the allocator hands out pages (a seeded permutation, or None)."""
    if not w.permute_pages:
        return None
    return rng_for(w, _S_PAGES).permutation(num_pages).astype(np.int32)


def to_fp16(x: np.ndarray) -> np.ndarray:
    """Clamp to the fp16 range and round to fp16 (nearest-even)."""
    return np.clip(x, -65504.0, 65504.0).astype(np.float16)


def _outlier_channels(w: Workload, layer: int, kv: int):
    """(channels, factors) per KV head for one layer and K (kv=0) or V (kv=1)."""
    D = w.head_dim
    if w.dist == "fixed_outliers":
        r = rng_for(w, _S_CHANNELS, kv)            # drawn once, shared by all layers
        ch = np.stack([r.choice(D, 4, replace=False) for _ in range(w.num_kv_heads)])
        fac = np.full(ch.shape, 20.0)
        return ch, fac
    if w.dist == "lognormal_outliers":
        r = rng_for(w, _S_CHANNELS, layer, kv)
        n = max(1, int(round(0.01 * D)))
        ch = np.stack([r.choice(D, n, replace=False) for _ in range(w.num_kv_heads)])
        fac = np.exp(r.uniform(np.log(10.0), np.log(50.0), size=ch.shape))
        return ch, fac
    return None, None


def kv_rows(w: Workload, layer: int, kv: int, n_tokens: int, stream: int = 0) -> np.ndarray:
    """fp16 rows [n_tokens][Hkv][D] for K (kv=0) or V (kv=1) of one layer.

    ``stream`` separates independent batches of tokens (e.g. the prefill context of
    sequence b vs the token appended at a decode step)."""
    D, H = w.head_dim, w.num_kv_heads
    r = rng_for(w, _S_KV, layer, kv, stream)
    if w.dist == "student_t3":
        x = r.standard_t(3.0, size=(n_tokens, H, D))
        return to_fp16(x)
    x = r.standard_normal((n_tokens, H, D))
    ch, fac = _outlier_channels(w, layer, kv)
    for h in range(H):
        x[:, h, ch[h]] *= fac[h]
    if w.dist == "lognormal_outliers":
        x *= r.lognormal(0.0, 0.5, size=(n_tokens, H, 1))
    return to_fp16(x)


def q_rows(w: Workload, layer: int, stream: int = 0) -> np.ndarray:
    """fp16 queries [batch][Hq][D], N(0,1)."""
    r = rng_for(w, _S_Q, layer, stream)
    return to_fp16(r.standard_normal((w.batch, w.num_q_heads, w.head_dim)))


def q_rows_chunk(w: Workload, layer: int, n_tokens: int, stream: int = 0) -> np.ndarray:
    """q of n_tokens query tokens (chunks of several sequences concatenated), N(0,1), fp16
    [n_tokens][Hq][D]."""
    rng = rng_for(w, _S_Q, layer, 100 + stream)
    return to_fp16(rng.standard_normal((n_tokens, w.num_q_heads, w.head_dim)))


def cu_seqlens(counts) -> np.ndarray:
    counts = np.asarray(counts, np.int64)
    out = np.zeros(len(counts) + 1, np.int32)
    out[1:] = np.cumsum(counts)
    return out


def scale_down(w: Workload, max_tokens: int, batch: Optional[int] = None) -> Workload:
    """A smaller case of the same recipe (same heads, block, page size, distribution):
    lengths capped at ``max_tokens`` and optionally fewer sequences -- for parity tests
    the oracle finishes in seconds."""
    import dataclasses
    v = dataclasses.replace(w)
    if batch is not None:
        v.batch = batch
    if v.ragged is not None:
        lo, hi = v.ragged
        v.ragged = (min(lo, max_tokens), max_tokens)
    elif v.context is not None:
        v.context = [min(c, max_tokens) for c in v.context][: v.batch]
        while len(v.context) < v.batch:
            v.context.append(v.context[-1] if v.context else max_tokens)
    v.num_layers = min(v.num_layers, 1)
    return v


# ---------------------------------------------------------------- on-device ---
# The same recipes drawn with torch's generator on a CUDA device, for workloads too
# large to generate on the host (full-size benchmarks and sampled parity checks, which
# copy back only the rows they check).  Values differ from the numpy draws above (a
# different generator) but follow the same distributions.
def kv_rows_torch(w: Workload, layer: int, kv: int, n_tokens: int, stream: int = 0,
                  device="cuda"):
    import torch
    D, H = w.head_dim, w.num_kv_heads
    gen = torch.Generator(device=device)
    gen.manual_seed(int(np.random.SeedSequence([w.seed, _S_KV, layer, kv, stream]).generate_state(1)[0]))
    if w.dist == "student_t3":
        # t(3) = N(0,1) / sqrt(chi2(3)/3), chi2(3) = sum of 3 squared normals
        z = torch.randn((n_tokens, H, D), generator=gen, device=device, dtype=torch.float32)
        c = torch.randn((3, n_tokens, H, D), generator=gen, device=device, dtype=torch.float32)
        x = z / torch.sqrt((c * c).sum(0) / 3.0)
        return x.clamp_(-65504.0, 65504.0).to(torch.float16)
    x = torch.randn((n_tokens, H, D), generator=gen, device=device, dtype=torch.float32)
    ch, fac = _outlier_channels(w, layer, kv)
    for h in range(H):
        x[:, h, torch.as_tensor(ch[h], device=device)] *= torch.as_tensor(
            fac[h], device=device, dtype=torch.float32)
    if w.dist == "lognormal_outliers":
        x *= torch.exp(0.5 * torch.randn((n_tokens, H, 1), generator=gen, device=device))
    return x.clamp_(-65504.0, 65504.0).to(torch.float16)


def q_rows_torch(w: Workload, layer: int, stream: int = 0, device="cuda"):
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(int(np.random.SeedSequence([w.seed, _S_Q, layer, stream]).generate_state(1)[0]))
    x = torch.randn((w.batch, w.num_q_heads, w.head_dim), generator=gen, device=device)
    return x.to(torch.float16)
