"""Seeded synthetic inputs for the ReSA decode hot path.

This module is the only code shared by the CPU oracle and the CUDA path. It
draws random numbers and rounds them to the storage type; it holds none of the
method's arithmetic (no descriptors, scores, selection or attention).

Distribution (the workloads of the five benchmark configurations, all
synthetic, no dataset):

* keys and values: N(0, 1) per element plus a mean vector per (batch, KV head,
  16-token block) drawn from N(0, 0.5^2) per channel; K and V use independent
  draws;
* queries: N(0, 1) / sqrt(head_dim), i.e. the 1/sqrt(d) softmax scale is
  folded into q and the attention calls take softmax_scale = 1;
* decode tokens (k_new, v_new) follow the cache distribution, with the mean of
  the block their position falls in;
* rectify K/V: either fresh N(0, 1) draws (the tiny fp32 configuration) or the
  same block-mean structure (the batched sweep);
* optional "needle" blocks: per (batch, KV head) a unit vector q_dir and a set
  of seeded block positions whose keys are shifted by shift * q_dir.

Every draw is keyed by (seed, stream, index) through numpy's SeedSequence, so
any decode step or rectify call can be regenerated on its own.

bf16 data is produced by round-to-nearest-even of the fp32 draw; the returned
fp32 arrays then hold exactly the bf16 values, so both sides see identical
numbers.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

BLOCK = 16

# stream ids for SeedSequence keys
_S_CACHE_K, _S_CACHE_V, _S_MEAN_K, _S_MEAN_V = 1, 2, 3, 4
_S_Q, _S_KNEW, _S_VNEW = 5, 6, 7
_S_RQ, _S_RK, _S_RV = 8, 9, 10
_S_NEEDLE = 11
_S_LENS = 12
_S_PQ = 13


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the uint16 patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    u = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (u >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Return x as fp32 values representable in `dtype` ('f32' or 'bf16')."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        return bf16_to_f32(bf16_bits(x))
    if dtype == "f32":
        return x
    raise ValueError(dtype)


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *key])))


@dataclasses.dataclass
class Spec:
    """One synthetic workload.

    len0 tokens are in the cache before the first decode step; decode step s
    (0-based) appends the token at position len0 + s, so after it the cache
    holds len0 + s + 1 valid tokens.
    """
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    len0: int
    steps: int
    dtype: str = "bf16"          # 'f32' or 'bf16'
    r: float = 0.1
    n_min: int = 16
    f: int = 32
    seed: int = 20260602
    needles: int = 0             # needle blocks per (batch, KV head)
    needle_shift: float = 2.0
    rect_block_mean: bool = True  # rectify K/V carry the block means
    max_len: int = 0             # cache capacity; 0 -> len0 + steps rounded up to 16

    def __post_init__(self):
        if self.max_len == 0:
            need = self.len0 + self.steps
            self.max_len = ((need + BLOCK - 1) // BLOCK) * BLOCK
        assert self.max_len % BLOCK == 0 and self.max_len >= self.len0 + self.steps
        assert self.n_q_heads % self.n_kv_heads == 0

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def max_blocks(self) -> int:
        return self.max_len // BLOCK


def block_means(spec: Spec, which: str) -> np.ndarray:
    """Per-(b, h, block) mean vectors [B, Hkv, max_blocks, d], N(0, 0.5^2)."""
    stream = _S_MEAN_K if which == "k" else _S_MEAN_V
    g = _rng(spec.seed, stream)
    shape = (spec.batch, spec.n_kv_heads, spec.max_blocks, spec.head_dim)
    return (0.5 * g.standard_normal(shape, dtype=np.float32)).astype(np.float32)


def needle_layout(spec: Spec):
    """(q_dir [B,Hkv,d] unit vectors, positions [B,Hkv,needles] block ids)."""
    g = _rng(spec.seed, _S_NEEDLE)
    qd = g.standard_normal((spec.batch, spec.n_kv_heads, spec.head_dim)).astype(np.float64)
    qd /= np.linalg.norm(qd, axis=-1, keepdims=True)
    m0 = spec.len0 // BLOCK  # full blocks of the prefilled context
    pos = np.zeros((spec.batch, spec.n_kv_heads, spec.needles), dtype=np.int64)
    if spec.needles:
        assert m0 > spec.needles
        for b in range(spec.batch):
            for h in range(spec.n_kv_heads):
                pos[b, h] = np.sort(g.choice(m0, size=spec.needles, replace=False))
    return qd.astype(np.float32), pos


def make_cache(spec: Spec):
    """Prefilled caches K, V as fp32 arrays [B, Hkv, max_len, d].

    Slots [0, len0) hold data; slots beyond are zero. Values are rounded to
    spec.dtype.
    """
    B, H, L, d = spec.batch, spec.n_kv_heads, spec.max_len, spec.head_dim
    out = []
    for which, s_cache in (("k", _S_CACHE_K), ("v", _S_CACHE_V)):
        mean = block_means(spec, which)
        arr = np.zeros((B, H, L, d), dtype=np.float32)
        g = _rng(spec.seed, s_cache)
        for b in range(B):
            for h in range(H):
                x = g.standard_normal((spec.len0, d), dtype=np.float32)
                nb = (spec.len0 + BLOCK - 1) // BLOCK
                x += np.repeat(mean[b, h, :nb], BLOCK, axis=0)[: spec.len0]
                arr[b, h, : spec.len0] = x
        out.append(arr)
    K, V = out
    if spec.needles:
        qd, pos = needle_layout(spec)
        for b in range(B):
            for h in range(H):
                for j in pos[b, h]:
                    K[b, h, j * BLOCK:(j + 1) * BLOCK] += spec.needle_shift * qd[b, h]
    return round_to(K, spec.dtype), round_to(V, spec.dtype)


def prefill_queries(spec: Spec) -> np.ndarray:
    """Queries of every prompt position: [B, len0, Hq, d], N(0, 1) / sqrt(d),
    rounded to spec.dtype (the prompt's keys and values are make_cache's)."""
    q = _rng(spec.seed, _S_PQ).standard_normal(
        (spec.batch, spec.len0, spec.n_q_heads, spec.head_dim), dtype=np.float32)
    q /= np.float32(math.sqrt(spec.head_dim))
    return round_to(q, spec.dtype)


def length_mix(spec: Spec, min_len: int, salt: int = 0) -> np.ndarray:
    """Per-row prompt lengths for a ragged batch: int32 [B] drawn uniformly
    from [min_len, spec.len0]; the longest row is set to spec.len0 so that
    spec.len0 stays the bound."""
    g = _rng(spec.seed, _S_LENS, salt)
    lens = g.integers(min_len, spec.len0 + 1, size=spec.batch).astype(np.int32)
    lens[int(g.integers(0, spec.batch))] = spec.len0
    return lens


def ragged(K: np.ndarray, V: np.ndarray, lens0) -> tuple[np.ndarray, np.ndarray]:
    """Copies of K, V [B, Hkv, L, d] with row b's slots at or past lens0[b]
    cleared, as a cache filled to those lengths would be."""
    K, V = K.copy(), V.copy()
    for b, n in enumerate(lens0):
        K[b, :, int(n):] = 0.0
        V[b, :, int(n):] = 0.0
    return K, V


def decode_inputs(spec: Spec, step: int):
    """Inputs of decode step `step`: q [B,Hq,d], k_new, v_new [B,Hkv,d]."""
    B, Hq, H, d = spec.batch, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
    pos = spec.len0 + step
    q = _rng(spec.seed, _S_Q, step).standard_normal((B, Hq, d), dtype=np.float32)
    q /= np.float32(math.sqrt(d))
    kn = _rng(spec.seed, _S_KNEW, step).standard_normal((B, H, d), dtype=np.float32)
    vn = _rng(spec.seed, _S_VNEW, step).standard_normal((B, H, d), dtype=np.float32)
    j = pos // BLOCK
    kn += _block_mean_row(spec, "k", j)
    vn += _block_mean_row(spec, "v", j)
    return round_to(q, spec.dtype), round_to(kn, spec.dtype), round_to(vn, spec.dtype)


_MEAN_CACHE: dict = {}


def _block_mean_row(spec: Spec, which: str, j: int) -> np.ndarray:
    key = (spec.seed, spec.batch, spec.n_kv_heads, spec.max_blocks, spec.head_dim, which)
    if key not in _MEAN_CACHE:
        if len(_MEAN_CACHE) > 8:
            _MEAN_CACHE.clear()
        _MEAN_CACHE[key] = block_means(spec, which)
    return _MEAN_CACHE[key][:, :, j, :]


def rectify_inputs(spec: Spec, call: int, length: int, f: int | None = None):
    """Inputs of rectify call `call` over positions [length - f, length).

    Returns q_f [B, f, Hq, d], k_f, v_f [B, f, Hkv, d].
    """
    f = spec.f if f is None else f
    B, Hq, H, d = spec.batch, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
    q = _rng(spec.seed, _S_RQ, call).standard_normal((B, f, Hq, d), dtype=np.float32)
    q /= np.float32(math.sqrt(d))
    k = _rng(spec.seed, _S_RK, call).standard_normal((B, f, H, d), dtype=np.float32)
    v = _rng(spec.seed, _S_RV, call).standard_normal((B, f, H, d), dtype=np.float32)
    if spec.rect_block_mean:
        blocks = (length - f + np.arange(f)) // BLOCK
        for which, arr in (("k", k), ("v", v)):
            rows = np.stack([_block_mean_row(spec, which, int(j)) for j in blocks], axis=1)
            arr += rows
    return round_to(q, spec.dtype), round_to(k, spec.dtype), round_to(v, spec.dtype)


# The five benchmark workloads. Sizes follow the configuration list the
# method's evaluation is reproduced on (all synthetic).
def config(idx: int, **over) -> Spec:
    if idx == 0:   # tiny fp32 step
        s = dict(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=64, len0=2048, steps=64,
                 dtype="f32", r=0.1, n_min=4, f=32, rect_block_mean=False)
    elif idx == 1:  # Llama-3-8B-shaped layer at 32K, batch 4, needles
        s = dict(batch=4, n_q_heads=32, n_kv_heads=8, head_dim=128, len0=32768, steps=256,
                 dtype="bf16", r=0.1, n_min=16, f=32, needles=8)
    elif idx == 2:  # 128K, batch 1
        s = dict(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, len0=131072, steps=512,
                 dtype="bf16", r=0.1, n_min=16, f=32)
    elif idx == 3:  # 256K, batch 1
        s = dict(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, len0=262144, steps=512,
                 dtype="bf16", r=0.1, n_min=16, f=32)
    elif idx == 4:  # batched rectify-heavy sweep at 64K
        s = dict(batch=16, n_q_heads=32, n_kv_heads=8, head_dim=128, len0=65536, steps=64,
                 dtype="bf16", r=0.1, n_min=16, f=32)
    else:
        raise ValueError(idx)
    s.update(over)
    return Spec(**s)
