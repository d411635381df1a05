"""Prefill (causal attention of every prompt position, descriptors from the
same pass) against the oracle's prefill."""
import numpy as np
import pytest
import torch

import oracle as orc
from pair import close, tdt, to_dev
from workload import Spec, make_cache, prefill_queries

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def resa():
    import __graft_entry__
    __graft_entry__.build()
    import block_sparse_attention_quest_b200 as m
    return m


def _run(resa, spec, scale=1.0):
    K, V = make_cache(spec)
    q = prefill_queries(spec)
    k, v = to_dev(K, spec.dtype), to_dev(V, spec.dtype)
    desc = torch.zeros(spec.batch, spec.n_kv_heads, spec.max_blocks, 2, spec.head_dim,
                       dtype=tdt(spec.dtype), device="cuda")
    out = torch.full((spec.batch, spec.len0, spec.n_q_heads, spec.head_dim), 7.0,
                     dtype=tdt(spec.dtype), device="cuda")
    dims = resa.dims_for(k, spec.n_q_heads)
    ws = resa.alloc_workspace(dims, spec.max_len, 0)
    resa.prefill(to_dev(q, spec.dtype), k, v, desc, spec.len0, scale, out, ws)
    assert resa.workspace_status(ws) == resa.RESA_OK
    return K, V, q, out.float().cpu().numpy(), desc.float().cpu().numpy()


def _desc_exact(K, spec, desc):
    lo, hi = orc.build_desc(K, spec.len0)
    M = orc.num_blocks(spec.len0)
    assert np.array_equal(desc[:, :, :M, 0], lo) and np.array_equal(desc[:, :, :M, 1], hi)
    assert not desc[:, :, M:].any(), "blocks past the prompt were written"


@pytest.mark.parametrize("G,d,length", [(4, 128, 1), (4, 128, 16), (4, 128, 100), (4, 128, 777),
                                        (1, 64, 300), (2, 128, 257), (8, 64, 500)])
def test_prefill_matches_oracle(resa, G, d, length):
    spec = Spec(batch=2, n_q_heads=2 * G, n_kv_heads=2, head_dim=d, len0=length, steps=0)
    K, V, q, out, desc = _run(resa, spec, scale=0.9)
    O, lo, hi = orc.prefill(q, K, V, length, 0.9, spec.group)
    close(out, O, "bf16", f"prefill G={G} d={d} len={length}")
    _desc_exact(K, spec, desc)


def test_prefill_long_prompt_sampled_rows(resa):
    """32 query heads / 8 KV heads, 8197 positions: descriptors bit-exact,
    sampled rows against dense decodes of the oracle."""
    spec = Spec(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, len0=8197, steps=0)
    K, V, q, out, desc = _run(resa, spec)
    _desc_exact(K, spec, desc)
    for i in (0, 31, 32, 127, 128, 4095, 4096, 8000, 8191, 8196):
        st = orc.State(K, V, i + 1, spec.group)
        Od, _ = st.dense(q[:, i], 1.0)
        close(out[:, i], Od, "bf16", f"row {i}")


def test_prefill_descriptors_equal_build_desc(resa):
    """The fused descriptors are the ones the standalone build writes."""
    spec = Spec(batch=2, n_q_heads=32, n_kv_heads=8, head_dim=128, len0=3001, steps=0)
    K, V, q, out, desc = _run(resa, spec)
    k = to_dev(K, "bf16")
    d2 = torch.zeros(2, 8, spec.max_blocks, 2, 128, dtype=torch.bfloat16, device="cuda")
    resa.build_desc(k, spec.len0, d2, 32)
    assert np.array_equal(desc, d2.float().cpu().numpy())
