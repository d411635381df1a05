"""Failure detection on the GPU without a fault: a bounded device wait on a
flag that nothing sets runs out, reports RESA_ERR_TIMEOUT through the
workspace, and the context stays usable for the next calls."""
import time

import pytest
import torch

from workload import Spec

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def resa():
    import __graft_entry__
    __graft_entry__.build()
    import block_sparse_attention_quest_b200 as m
    return m


def test_stuck_wait_times_out_and_is_reported(resa):
    dims = resa.Dims(1, 8, 2, 128, 16, resa.RESA_BF16, 1024)
    ws = resa.alloc_workspace(dims, 1024, 32)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")       # nothing sets it
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    resa.wait_check(flag, 1, 50_000, ws)                           # 50 ms limit
    assert resa.workspace_status(ws) == resa.RESA_ERR_TIMEOUT
    elapsed = time.perf_counter() - t0
    assert 0.04 < elapsed < 5.0, elapsed
    assert resa.workspace_status(ws) == resa.RESA_OK               # the flag was cleared
    # a flag that is already set: no time-out
    flag.fill_(3)
    resa.wait_check(flag, 2, 50_000, ws)
    assert resa.workspace_status(ws) == resa.RESA_OK


def test_context_usable_after_a_time_out(resa):
    """Decode steps after the timed-out wait, on the same workspace, match the
    oracle."""
    from pair import Pair
    spec = Spec(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, len0=3000, steps=2)
    p = Pair(spec)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    resa.wait_check(flag, 1, 20_000, p.ws)
    assert resa.workspace_status(p.ws) == resa.RESA_ERR_TIMEOUT
    for step in range(spec.steps):
        p.decode(step)                # checks the workspace status and the oracle
    assert p.desc_matches()
