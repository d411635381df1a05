"""Bit-exact top-n selection at the benchmark's row sizes.

With the synthetic N(0, 1) keys, 8192 or 16384 block scores per group lie so
close together that the n-th and (n+1)-th oracle scores are within the 1e-4
near-tie band in most groups, so those runs can only check the band rules.
Here the keys are built so that fp32 evaluates every group score exactly, in
any summation order: the query heads of a group put powers of two on two
channels each (zero elsewhere), and the keys are small integers on those
channels, so every product and partial sum is an integer below 2^24. The
GPU's scores then equal the oracle's, and its block list must equal the
oracle's bit for bit, ties (many exact ones) broken by the lower index, as
the group score and tie rule define ("Rectified Sparse Attention", section
"What carries the argument"; Eq. 5 for n).

Channels the queries do not use hold the usual N(0, 1) + block-mean keys, so
the attention outputs still see ordinary data; they are compared with the
oracle at the bf16 tolerance.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from workload import Spec, decode_inputs, make_cache, round_to

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import __graft_entry__
    __graft_entry__.build()
    from tests.pair import Pair, close, to_dev


def integer_score_inputs(spec: Spec, seed: int):
    """Cache and query of one decode step whose group scores are integers.

    Head i of group g weights channels 2i and 2i+1 by +-2^e (e in 0..4); the
    keys' per-block minimum and maximum on those channels are integers drawn
    in [-60, 59] (the first two tokens of a block attain them, the others
    lie between), every other channel is the workload's usual draw."""
    rng = np.random.default_rng(seed)
    K, V = make_cache(spec)
    B, H, _, d = K.shape
    G = spec.group
    C = 2 * G
    m0 = spec.len0 // 16
    lo = rng.integers(-60, 30, size=(B, H, m0, C))
    hi = lo + rng.integers(0, 31, size=(B, H, m0, C))
    mid = rng.integers(0, 1 << 30, size=(B, H, m0, 16, C)) % (hi - lo + 1)[:, :, :, None, :]
    tok = lo[:, :, :, None, :] + mid
    tok[:, :, :, 0, :] = lo
    tok[:, :, :, 1, :] = hi
    K[:, :, : m0 * 16, :C] = tok.reshape(B, H, m0 * 16, C).astype(np.float32)
    q = np.zeros((B, spec.n_q_heads, d), dtype=np.float32)
    w = (2.0 ** rng.integers(0, 5, size=(B, spec.n_q_heads, 2))) * rng.choice([-1.0, 1.0],
                                                                             size=(B, spec.n_q_heads, 2))
    for h in range(spec.n_q_heads):
        i = h % G
        q[:, h, 2 * i] = w[:, h, 0]
        q[:, h, 2 * i + 1] = w[:, h, 1]
    return round_to(K, "bf16"), V, round_to(q, "bf16")


@pytest.mark.parametrize("len0,r", [(131072, 0.1), (262144, 0.1)])
def test_selection_bit_exact_at_benchmark_sizes(len0, r):
    """128K (8193 blocks after the step: keys in registers, 8 per thread) and
    256K (16385 blocks: 16 per thread), at the benchmark's head shape."""
    spec = Spec(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, len0=len0, steps=1,
                dtype="bf16", r=r, n_min=16)
    K, V, q = integer_score_inputs(spec, seed=len0 + int(r * 100))
    p = Pair(spec, cache=(K, V))
    _, kn, vn = decode_inputs(spec, 0)
    length = spec.len0 + 1
    n = p.resa.num_selected(length, r, spec.n_min)
    out = torch.empty(1, 32, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(1, 32, dtype=torch.float32, device="cuda")
    sel = torch.empty(1, 8, n, dtype=torch.int32, device="cuda")
    scale = 1.0 / 1024.0
    p.resa.decode_sparse(to_dev(q, "bf16"), to_dev(kn, "bf16"), to_dev(vn, "bf16"), p.k, p.v,
                         p.desc, length, r, spec.n_min, scale, out, p.ws, lse=lse, sel=sel)
    assert p.resa.workspace_status(p.ws) == p.resa.RESA_OK
    ref = p.st.decode(q, kn, vn, r, spec.n_min, scale)
    assert ref["n"] == n
    scores = ref["scores"]
    # the scores are integers (exact in fp32), and the threshold really ties
    assert np.array_equal(scores[:, :, :-1], np.round(scores[:, :, :-1]))
    M = orc.num_blocks(length)
    tied = 0
    for g in range(8):
        s = scores[0, g, : M - 1]
        order = np.lexsort((np.arange(M - 1), -s))
        tied += int(s[order[n - 2]] == s[order[n - 1]])
    assert tied >= 1, "the construction should put exact ties at the threshold"
    assert np.array_equal(sel.cpu().numpy(), ref["sel"]), "block lists differ"
    close(out.float().cpu().numpy(), ref["out"], "bf16", f"decode at {length}")
    close(lse.cpu().numpy(), ref["lse"], "bf16", f"lse at {length}")
    assert p.desc_matches()
