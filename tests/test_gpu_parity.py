"""GPU (sm_100a) vs CPU oracle parity through the C ABI.

Tolerances: bf16 K/V rel-L2 <= 5e-3 and max-abs <= 2e-2 on outputs; fp32 both
<= 1e-5. Descriptors are bit-exact (min/max). Selected blocks are bit-exact
wherever the oracle's gap between the n-th and (n+1)-th score exceeds 1e-4
relative; inside a near-tie band the GPU's choice is checked for validity and
the output is compared with the oracle evaluated on that choice.
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc
from workload import Spec, config, make_cache, round_to

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import __graft_entry__
    __graft_entry__.build()
    from tests.pair import Pair, check_selection, close, fp32_score_error, to_dev, tdt
    from workload import decode_inputs


# ------------------------------------------------------------------ descriptors
@pytest.mark.parametrize("dtype,d,length", [("f32", 64, 2047), ("bf16", 128, 4001),
                                            ("bf16", 64, 33), ("f32", 128, 16),
                                            ("bf16", 128, 1)])
def test_build_desc_bitexact(dtype, d, length):
    import block_sparse_attention_quest_b200 as resa
    spec = Spec(batch=2, n_q_heads=8, n_kv_heads=2, head_dim=d, len0=length, steps=16, dtype=dtype)
    K, _ = make_cache(spec)
    k = to_dev(K, dtype)
    desc = torch.full((2, 2, spec.max_blocks, 2, d), 7.0, dtype=tdt(dtype), device="cuda")
    resa.build_desc(k, length, desc, 8)
    lo, hi = orc.build_desc(K, length)
    M = orc.num_blocks(length)
    got = desc.float().cpu().numpy()
    assert np.array_equal(got[:, :, :M, 0], lo) and np.array_equal(got[:, :, :M, 1], hi)
    assert np.all(got[:, :, M:] == 7.0)   # blocks past len untouched


# ------------------------------------------------------------- full decode runs
def test_tiny_fp32_workload_every_step():
    """64 decode steps with rectification after steps 32 and 64 (f = 32)."""
    spec = config(0)
    p = Pair(spec)
    for step in range(spec.steps):
        p.decode(step)
        assert p.desc_matches()
        if (step + 1) % spec.f == 0:
            p.rectify()
            assert p.desc_matches()


def test_bf16_midsize_run_with_rectify():
    spec = Spec(batch=2, n_q_heads=32, n_kv_heads=8, head_dim=128, len0=5000, steps=40,
                dtype="bf16", r=0.1, n_min=16, f=32)
    p = Pair(spec)
    for step in range(spec.steps):
        p.decode(step)
        if (step + 1) % spec.f == 0:
            p.rectify()
    assert p.desc_matches()


def test_stage_calls_match_oracle():
    """resa_select_blocks + resa_attend_blocks (the three-kernel path)."""
    spec = Spec(batch=2, n_q_heads=32, n_kv_heads=8, head_dim=128, len0=9000, steps=3,
                dtype="bf16", r=0.1, n_min=16)
    p = Pair(spec)
    for step in range(spec.steps):
        q, kn, vn = decode_inputs(spec, step)
        p.length += 1
        n = p.resa.num_selected(p.length, spec.r, spec.n_min)
        sel = torch.empty(2, 8, n, dtype=torch.int32, device="cuda")
        out = torch.empty(2, 32, 128, dtype=torch.bfloat16, device="cuda")
        qd = to_dev(q, "bf16")
        p.resa.select_blocks(qd, to_dev(kn, "bf16"), to_dev(vn, "bf16"), p.k, p.v, p.desc, p.length,
                             spec.r, spec.n_min, sel, p.ws)
        p.resa.attend_blocks(qd, p.k, p.v, p.length, sel, 1.0, out, p.ws)
        ref = p.st.decode(q, kn, vn, spec.r, spec.n_min, 1.0)
        gsel = sel.cpu().numpy()
        err = fp32_score_error(q, p.st.lo, p.st.hi, ref["scores"].shape[-1])
        exact = all(check_selection(gsel[b, g], ref["scores"][b, g], n, err[b, g])
                    for b in range(2) for g in range(8))
        if not exact:
            ref["out"], _ = p.st.attend_with(q, gsel, 1.0)
        close(out.float().cpu().numpy(), ref["out"], "bf16", f"staged step {step}")
    assert p.desc_matches()


def test_dense_decode_arm():
    spec = Spec(batch=2, n_q_heads=32, n_kv_heads=8, head_dim=128, len0=3000, steps=4,
                dtype="bf16")
    p = Pair(spec)
    for step in range(spec.steps):
        p.decode(step, dense=True)
    assert p.desc_matches()


# ------------------------------------------------------------------ edge cases
@pytest.mark.parametrize("dtype,d,G,len0,r,n_min", [
    ("bf16", 128, 4, 1023, 0.1, 4),     # first step lands on len % 16 == 0
    ("bf16", 128, 4, 1024, 0.1, 4),     # len % 16 == 1: a new local block
    ("bf16", 128, 4, 1038, 0.1, 4),     # len % 16 == 15
    ("bf16", 64, 4, 700, 0.2, 2),       # head_dim 64
    ("f32", 128, 4, 900, 0.1, 3),       # fp32, head_dim 128
    ("bf16", 128, 1, 800, 0.1, 4),      # group of 1
    ("bf16", 128, 8, 800, 0.1, 4),      # group of 8
    ("f32", 64, 2, 600, 0.1, 4),
    ("bf16", 128, 4, 100, 0.1, 16),     # M <= n_min: the step is dense
    ("bf16", 128, 4, 500, 1.0, 1),      # r = 1 selects every block
    ("bf16", 128, 4, 5, 0.1, 1),        # a single partial block
])
def test_decode_edge_cases(dtype, d, G, len0, r, n_min):
    spec = Spec(batch=2, n_q_heads=2 * G, n_kv_heads=2, head_dim=d, len0=len0, steps=20,
                dtype=dtype, r=r, n_min=n_min, f=16)
    p = Pair(spec)
    for step in range(spec.steps):
        p.decode(step)
    assert p.desc_matches()


def test_all_tied_scores_take_lowest_indices():
    spec = Spec(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, len0=640, steps=2,
                dtype="bf16", r=0.1, n_min=4)
    K, V = make_cache(spec)
    K[:] = round_to(np.full_like(K, 0.5), "bf16")       # every block identical
    p = Pair(spec, cache=(K, V))
    for step in range(spec.steps):
        res = p.decode(step)
        n = res["n"]
        M = orc.num_blocks(p.length)
        assert list(res["sel"][0, 0]) == list(range(n - 1)) + [M - 1]
        assert np.array_equal(res["gpu_sel"], res["sel"])


def test_crowded_ties_take_lowest_indices():
    """Blocks drawn from three constant patterns: scores take three values, so
    the threshold is a crowded exact tie broken by block index."""
    spec = Spec(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, len0=16 * 3000, steps=2,
                dtype="bf16", r=0.1, n_min=4)
    K, V = make_cache(spec)
    rng = np.random.default_rng(99)
    pats = round_to(rng.standard_normal((3, 128)).astype(np.float32), "bf16")
    which = rng.integers(0, 3, size=(1, 2, 3000))
    K[:, :, :spec.len0] = np.repeat(pats[which], 16, axis=2)
    p = Pair(spec, cache=(K, V))
    for step in range(spec.steps):
        res = p.decode(step)
        assert np.array_equal(res["gpu_sel"], res["sel"])


@pytest.mark.parametrize("extra", [0, 5, 700, 1500])
def test_two_score_levels(extra):
    """Blocks whose tokens alternate +a and -a in every channel have lo = -a,
    hi = +a and the pooled bound a * sum_c (P_c - N_c) >= 0, so two amplitudes
    give exactly two scores. With need + extra blocks at the higher one the
    threshold bin is taken whole (0), resolved by ranking its members by index
    (5, 700) or, with more members than the ranked path holds, by the radix
    passes (1500). Either way the lowest-index high blocks are kept."""
    spec = Spec(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, len0=16 * 3000, steps=1,
                dtype="bf16", r=0.1, n_min=4)
    K, V = make_cache(spec)
    M = orc.num_blocks(spec.len0 + 1)
    need = orc.num_selected(M, spec.r, spec.n_min) - 1
    rng = np.random.default_rng(7)
    amp = np.full((2, 3000), 0.5, dtype=np.float32)
    for h in range(2):
        amp[h, rng.choice(3000, need + extra, replace=False)] = 1.0
    sign = np.where(np.arange(16) % 2 == 0, 1.0, -1.0).astype(np.float32)
    blocks = amp[:, :, None, None] * sign[None, None, :, None] * np.ones(128, np.float32)
    K[0, :, :spec.len0] = blocks.reshape(2, spec.len0, 128)
    p = Pair(spec, cache=(K, V))
    res = p.decode(0)
    for h in range(2):
        high = np.sort(np.nonzero(amp[h] == 1.0)[0])[:need]
        assert list(res["gpu_sel"][0, h]) == list(high) + [M - 1]
    assert np.array_equal(res["gpu_sel"], res["sel"])


@pytest.mark.parametrize("len0", [16 * 2000 + 5, 16 * 6000, 16 * 12000 + 3, 16 * 30000])
def test_select_row_sizes(len0):
    """Rows of 2000 to 30000 blocks: the register selection with 8 and 16 keys
    per thread and the shared-memory one."""
    spec = Spec(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=64, len0=len0, steps=3,
                dtype="bf16", r=0.1, n_min=16)
    p = Pair(spec)
    for step in range(spec.steps):
        p.decode(step)
    assert p.desc_matches()


@pytest.mark.parametrize("r,n_min", [(1.0, 16), (1e-4, 1)])
def test_select_every_block_and_local_only(r, n_min):
    """n = M (every block kept) and n = 1 (only the local block) on a row of
    3000 blocks."""
    spec = Spec(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=64, len0=16 * 3000 + 7, steps=2,
                dtype="bf16", r=r, n_min=n_min)
    p = Pair(spec)
    for step in range(spec.steps):
        res = p.decode(step)
        M = orc.num_blocks(p.length)
        expect = list(range(M)) if res["n"] == M else [M - 1]
        assert res["n"] in (1, M)
        assert [list(x) for x in res["gpu_sel"][0]] == [expect, expect]


def test_all_tied_scores_on_a_long_row():
    """Every block identical at 3000 blocks: the whole row ties, the lowest
    indices are kept."""
    spec = Spec(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, len0=16 * 3000, steps=2,
                dtype="bf16", r=0.1, n_min=4)
    K, V = make_cache(spec)
    K[:] = round_to(np.full_like(K, 0.5), "bf16")
    p = Pair(spec, cache=(K, V))
    for step in range(spec.steps):
        res = p.decode(step)
        n, M = res["n"], orc.num_blocks(p.length)
        assert list(res["gpu_sel"][0, 0]) == list(range(n - 1)) + [M - 1]


def test_select_beyond_shared_memory_keys():
    """More blocks than the selection keeps in shared memory (M > 40960)."""
    spec = Spec(batch=1, n_q_heads=4, n_kv_heads=1, head_dim=64, len0=700_001, steps=2,
                dtype="bf16", r=0.05, n_min=16)
    p = Pair(spec)
    for step in range(spec.steps):
        p.decode(step)


def test_select_at_the_block_limit():
    """262144 blocks (4,194,299 tokens after the step), the largest row the
    selection accepts: keys re-read from L2 by the general radix kernel."""
    spec = Spec(batch=1, n_q_heads=4, n_kv_heads=1, head_dim=64, len0=16 * 262144 - 6, steps=1,
                dtype="bf16", r=0.05, n_min=16)
    p = Pair(spec)
    res = p.decode(0)
    assert orc.num_blocks(p.length) == 262144 and res["n"] == 13108


@pytest.mark.parametrize("length,f", [(100, 32), (64, 16), (48, 48), (1000, 7), (1000, 64)])
def test_rectify_shapes(length, f):
    for dtype in ("bf16", "f32"):
        spec = Spec(batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, len0=length, steps=0,
                    dtype=dtype, f=f, max_len=((length + 15) // 16) * 16 + 32)
        p = Pair(spec)
        p.rectify(f)
        assert p.desc_matches()


def test_rectify_fallback_group_of_three():
    """bf16 with a group size the tensor-core tile does not take (3)."""
    spec = Spec(batch=2, n_q_heads=6, n_kv_heads=2, head_dim=128, len0=700, steps=8,
                dtype="bf16", f=32)
    p = Pair(spec)
    for step in range(spec.steps):
        p.decode(step)
    p.rectify(32)
    assert p.desc_matches()


def test_stale_cache_slots_do_not_leak():
    """Slots at or past len hold NaN bit patterns; outputs must not see them."""
    for dtype in ("bf16", "f32"):
        spec = Spec(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, len0=1000, steps=6,
                    dtype=dtype, r=0.1, n_min=4, f=16)
        p = Pair(spec)
        p.k[:, :, spec.len0:] = float("nan")
        p.v[:, :, spec.len0:] = float("nan")
        for step in range(spec.steps):
            p.decode(step)
        p.rectify(16)


def test_rectify_softmax_scale_argument():
    spec = Spec(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, len0=300, steps=4,
                dtype="bf16", f=16)
    p = Pair(spec)
    p.decode(0, scale=1 / math.sqrt(128))
    p.rectify(16, scale=1 / math.sqrt(128))


def test_needle_blocks_are_selected():
    spec = Spec(batch=2, n_q_heads=32, n_kv_heads=8, head_dim=128, len0=8192, steps=1,
                dtype="bf16", r=0.1, n_min=16, needles=8, needle_shift=12.0)
    p = Pair(spec)
    from workload import needle_layout
    qd, pos = needle_layout(spec)
    # queries aligned with each group's needle direction
    q = np.repeat(qd, 4, axis=1) * 0.5
    q = round_to(q, "bf16")
    n = p.resa.num_selected(spec.len0, spec.r, spec.n_min)
    out = torch.empty(2, 32, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(2, 8, n, dtype=torch.int32, device="cuda")
    p.resa.decode_sparse(to_dev(q, "bf16"), None, None, p.k, p.v, p.desc, spec.len0, spec.r,
                         spec.n_min, 1.0, out, p.ws, sel=sel)
    gsel = sel.cpu().numpy()
    for b in range(2):
        for g in range(8):
            assert set(pos[b, g].tolist()) <= set(gsel[b, g].tolist())
    ref = p.st.decode(q, None, None, spec.r, spec.n_min, 1.0)
    close(out.float().cpu().numpy(), ref["out"], "bf16", "needle decode")


# ------------------------------------------------------- workload configurations
def _run_sampled(spec, steps, rect_f=(), r=None, rows=None):
    import tests.pair as tp
    before = dict(tp.SELECTION_STATS)
    p = Pair(spec, r=r, rows=rows)
    for step in range(steps):
        p.decode(step)
    for f in rect_f:
        p.rectify(f)
    print(f"{spec.len0} x batch {spec.batch}: selection "
          f"{tp.SELECTION_STATS['exact'] - before['exact']} exact, "
          f"{tp.SELECTION_STATS['near_tie'] - before['near_tie']} near-tied (step, group) decisions")
    return p


def test_config_32k_batch4_needles():
    _run_sampled(config(1), steps=3, rect_f=(32,))


def test_config_128k():
    # f = 64: 256 query rows per KV head, two m-tiles
    _run_sampled(config(2), steps=3, rect_f=(32, 64))


@pytest.mark.parametrize("r", [0.1, 0.05])
def test_config_256k(r):
    _run_sampled(config(3, r=r), steps=2, rect_f=(32,) if r == 0.1 else ())


@pytest.mark.parametrize("r", [0.05, 0.1, 0.2])
def test_config_64k_batch16(r):
    spec = config(4, r=r, steps=2)
    _run_sampled(spec, steps=2, rect_f=(16, 32, 64) if r == 0.1 else (), rows=[0, 7, 15])


@pytest.mark.parametrize("len0,batch", [(20000, 2), (131072, 1)])
def test_one_launch_decode_path(len0, batch):
    """The one-launch decode kernel (RESA_DECODE_ONE_LAUNCH=1: the CTAs of each
    KV group score their slices, agree on the exact cut through the
    workspace and attend to equal shares), run in a child process so that the
    choice does not leak into other tests; also rows where every block is
    kept and where only the newest one is."""
    import subprocess
    import sys
    code = (
        "import sys; sys.path.insert(0, '.');"
        "from tests.pair import Pair;"
        "from workload import Spec;"
        f"spec = Spec(batch={batch}, n_q_heads=32, n_kv_heads=8, head_dim=128, len0={len0}, steps=4,"
        "            dtype='bf16', r=0.1, n_min=16);"
        "p = Pair(spec);"
        "[p.decode(s) for s in range(spec.steps)];"
        "assert p.desc_matches();"
        "spec2 = Spec(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, len0=640, steps=2,"
        "             dtype='bf16', r=0.1, n_min=4);"
        "p2 = Pair(spec2); [p2.decode(s) for s in range(2)];"
        "p3 = Pair(spec2, r=1.0); [p3.decode(s) for s in range(2)];"
        "p4 = Pair(spec2, r=1e-4, n_min=1); [p4.decode(s) for s in range(2)];"
        "spec5 = Spec(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=64, len0=16 * 3000, steps=2,"
        "             dtype='bf16', r=0.1, n_min=4);"
        "p5 = Pair(spec5); [p5.decode(s) for s in range(2)];"
        "print('one-launch ok')")
    import os
    env = dict(os.environ, RESA_DECODE_ONE_LAUNCH="1")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0 and "one-launch ok" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]


def test_one_launch_ties_and_crowded_bins():
    """The one-launch kernel on rows whose threshold is an exact tie: every
    block identical (one key), and three constant patterns (a crowded
    threshold bin resolved by the radix passes)."""
    import subprocess
    import sys
    code = (
        "import sys; sys.path.insert(0, '.');"
        "import numpy as np;"
        "from tests.pair import Pair;"
        "from workload import Spec, make_cache, round_to;"
        "spec = Spec(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, len0=16 * 3000, steps=2,"
        "            dtype='bf16', r=0.1, n_min=4);"
        "K, V = make_cache(spec); K[:] = round_to(np.full_like(K, 0.5), 'bf16');"
        "p = Pair(spec, cache=(K, V)); res = [p.decode(s) for s in range(2)];"
        "assert all(np.array_equal(r['gpu_sel'], r['sel']) for r in res);"
        "K, V = make_cache(spec); rng = np.random.default_rng(99);"
        "pats = round_to(rng.standard_normal((3, 128)).astype(np.float32), 'bf16');"
        "which = rng.integers(0, 3, size=(1, 2, 3000));"
        "K[:, :, :spec.len0] = np.repeat(pats[which], 16, axis=2);"
        "p = Pair(spec, cache=(K, V)); res = [p.decode(s) for s in range(2)];"
        "assert all(np.array_equal(r['gpu_sel'], r['sel']) for r in res);"
        "print('ties ok')")
    import os
    env = dict(os.environ, RESA_DECODE_ONE_LAUNCH="1")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], cwd=root, env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0 and "ties ok" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]


def test_back_to_back_calls_without_host_sync():
    """Decode calls on two layer caches issued back to back (each call's score
    kernel may launch while the previous call's attention kernel runs), every
    output kept, all compared with the oracle at the end."""
    import block_sparse_attention_quest_b200 as resa
    from pair import check_selection, close, fp32_score_error, to_dev
    from workload import decode_inputs
    spec = Spec(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, len0=20000, steps=6)
    K, V = make_cache(spec)
    layers = []
    for li in range(2):
        k, v = to_dev(K, "bf16"), to_dev(V, "bf16")
        desc = torch.zeros(1, 8, spec.max_blocks, 2, 128, dtype=torch.bfloat16, device="cuda")
        resa.build_desc(k, spec.len0, desc, 32)
        ws = resa.alloc_workspace(resa.dims_for(k, 32), spec.max_len, 32)
        layers.append((k, v, desc, ws, orc.State(K, V, spec.len0, spec.group)))
    outs = torch.empty(spec.steps, 2, 1, 32, 128, dtype=torch.bfloat16, device="cuda")
    sels = [[torch.full((1, 8, resa.num_selected(spec.len0 + t + 1, spec.r, spec.n_min)), -1,
                        dtype=torch.int32, device="cuda") for _ in range(2)]
            for t in range(spec.steps)]
    inputs = [tuple(to_dev(x, "bf16") for x in decode_inputs(spec, t)) for t in range(spec.steps)]
    torch.cuda.synchronize()
    for t in range(spec.steps):
        for li, (k, v, desc, ws, _) in enumerate(layers):
            resa.decode_sparse(*inputs[t], k, v, desc, spec.len0 + t + 1, spec.r, spec.n_min, 1.0,
                               outs[t, li], ws, sel=sels[t][li])
    torch.cuda.synchronize()
    for _, _, _, ws, _ in layers:
        assert resa.workspace_status(ws) == resa.RESA_OK
    got = outs.float().cpu().numpy()
    for t in range(spec.steps):
        q, kn, vn = decode_inputs(spec, t)
        for li, (_, _, _, _, st) in enumerate(layers):
            res = st.decode(q, kn, vn, spec.r, spec.n_min, 1.0)
            n, gsel = res["n"], sels[t][li].cpu().numpy()
            assert gsel.shape[-1] == n
            err = fp32_score_error(q, st.lo, st.hi, res["scores"].shape[-1])
            exact = all([check_selection(gsel[0, g], res["scores"][0, g], n, err[0, g])
                         for g in range(8)])
            O = res["out"] if exact else st.attend_with(q, gsel, 1.0)[0]
            close(got[t, li], O, "bf16", f"step {t} layer {li}")
