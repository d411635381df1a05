"""The allocation-free decode entry point, against the oracle and against the
workspace entry point.

Some callers cannot allocate device memory: code inside a framework whose
caching allocator owns the GPU (a private cudaMalloc there can fail once the
pool has reserved the memory, and bypasses its accounting), decode loops
captured into CUDA graphs that must not allocate between captures, and plugin
hosts that hand a kernel only its input and output pointers.
resa_decode_sparse_noalloc serves them with scratch in a fixed array inside
the library, and resa_noalloc_status reports the device-side errors raised
there. This file is collected last so that a failure here never hides the
other GPU tests; it also runs on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as orc
from workload import Spec, decode_inputs, make_cache

pytestmark = pytest.mark.gpu

TOL = (5e-3, 2e-2)   # bf16: rel-L2, max-abs (the tolerance of the parity tests)


def _close(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    rel = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)
    assert rel <= TOL[0] and np.abs(a - b).max() <= TOL[1], rel


def test_noalloc_matches_oracle_and_workspace_entry_point_on_two_calls():
    import __graft_entry__
    __graft_entry__.build()
    import block_sparse_attention_quest_b200 as resa
    from tests.pair import check_selection, fp32_score_error

    spec = Spec(batch=2, n_q_heads=32, n_kv_heads=8, head_dim=128, len0=5000, steps=2,
                dtype="bf16", r=0.1, n_min=16)
    K, V = make_cache(spec)
    st = orc.State(K, V, spec.len0, spec.group)

    def dev(x):
        return torch.from_numpy(np.ascontiguousarray(x)).cuda().to(torch.bfloat16)

    # two identical caches: one driven through each entry point
    ka, va = dev(K), dev(V)
    kb, vb = ka.clone(), va.clone()
    da = torch.zeros(2, 8, spec.max_blocks, 2, 128, dtype=torch.bfloat16, device="cuda")
    db = torch.zeros_like(da)
    resa.build_desc(ka, spec.len0, da, 32)
    resa.build_desc(kb, spec.len0, db, 32)
    dims = resa.dims_for(ka, 32)
    ws = resa.alloc_workspace(dims, spec.max_len)
    stream = torch.cuda.current_stream().cuda_stream
    for step in range(2):                       # two calls in a row
        length = spec.len0 + step + 1
        q_h, kn_h, vn_h = decode_inputs(spec, step)
        q, kn, vn = dev(q_h), dev(kn_h), dev(vn_h)
        n = resa.num_selected(length, spec.r, spec.n_min)
        out_a = torch.empty(2, 32, 128, dtype=torch.bfloat16, device="cuda")
        out_b = torch.empty_like(out_a)
        lse_a = torch.empty(2, 32, dtype=torch.float32, device="cuda")
        lse_b = torch.empty_like(lse_a)
        sel_a = torch.empty(2, 8, n, dtype=torch.int32, device="cuda")
        sel_b = torch.empty_like(sel_a)
        resa.decode_sparse(q, kn, vn, ka, va, da, length, spec.r, spec.n_min, 1.0, out_a, ws,
                           lse=lse_a, sel=sel_a)
        rc = resa._lib.resa_decode_sparse_noalloc(
            ctypes.byref(dims), q.data_ptr(), kn.data_ptr(), vn.data_ptr(), kb.data_ptr(),
            vb.data_ptr(), db.data_ptr(), length, spec.r, spec.n_min, 1.0, out_b.data_ptr(),
            lse_b.data_ptr(), sel_b.data_ptr(), stream)
        assert rc == resa.RESA_OK, resa.status_string(rc)
        assert resa._lib.resa_noalloc_status(stream) == resa.RESA_OK
        assert resa.workspace_status(ws) == resa.RESA_OK
        # against the oracle (selection by the parity rule, outputs within tolerance)
        ref = st.decode(q_h, kn_h, vn_h, spec.r, spec.n_min, 1.0)
        gsel = sel_b.cpu().numpy()
        err = fp32_score_error(q_h, st.lo, st.hi, ref["scores"].shape[-1])
        exact = all(check_selection(gsel[b, g], ref["scores"][b, g], n, err[b, g])
                    for b in range(2) for g in range(8))
        O, L = (ref["out"], ref["lse"]) if exact else st.attend_with(q_h, gsel, 1.0)
        _close(out_b.float().cpu().numpy(), O)
        _close(lse_b.cpu().numpy(), L)
        # against the workspace entry point on the same inputs
        _close(out_b.float().cpu().numpy(), out_a.float().cpu().numpy())
        assert torch.allclose(lse_b, lse_a, rtol=0, atol=1e-4)
        assert torch.equal(sel_b, sel_a)
        assert torch.equal(kb, ka) and torch.equal(vb, va) and torch.equal(db, da)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import block_sparse_attention_quest_b200 as resa
    # 64 x 8 groups at 1M tokens: scores alone need 128 MiB, far above 16 MiB
    dims = resa.Dims(64, 64, 8, 128, 16, resa.RESA_BF16, 1 << 20)
    fake = 0x10000
    rc = resa._lib.resa_decode_sparse_noalloc(ctypes.byref(dims), fake, None, None, fake, fake,
                                              fake, 1 << 20, 0.1, 16, 1.0, fake, None, None, None)
    assert rc == resa.RESA_ERR_WORKSPACE
