"""Pins for the CPU oracle, independent of the oracle itself.

Each test checks the oracle against something it does not share code with:
hand-worked fixtures (tests/golden), invariants that hold for any input,
special cases with a closed form, brute force on tiny inputs, and library
routines that compute the same textbook operation (torch's
scaled_dot_product_attention in float64, scipy's logsumexp).
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from scipy.special import logsumexp

import oracle as orc
from workload import Spec, decode_inputs, make_cache, rectify_inputs, round_to

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#")[0].strip()
            if line:
                yield line.split()


# --------------------------------------------------------------------- Eq. 5
def test_num_selected_golden():
    n = 0
    for M, r, n_min, exp in _rows("eq5_budget.txt"):
        assert orc.num_selected(int(M), float(r), int(n_min)) == int(exp), (M, r, n_min)
        n += 1
    assert n >= 10


def test_num_blocks_counts_partial_block():
    assert [orc.num_blocks(x) for x in (1, 15, 16, 17, 32, 33)] == [1, 1, 1, 2, 2, 3]


# --------------------------------------------------------------- descriptors
def test_desc_bounds_and_attained():
    rng = np.random.default_rng(1)
    K = rng.standard_normal((2, 3, 80, 5)).astype(np.float32)
    length = 71
    K[:, :, length:] = 1e6  # slots past len must not leak into descriptors
    lo, hi = orc.build_desc(K, length)
    assert lo.shape == (2, 3, 5, 5)
    for j in range(5):
        seg = K[:, :, j * 16:min(j * 16 + 16, length)]
        assert np.all(seg >= lo[:, :, j:j + 1]) and np.all(seg <= hi[:, :, j:j + 1])
        # attained: every lo/hi entry equals some token's value in that channel
        assert np.all(np.any(seg == lo[:, :, j:j + 1], axis=2))
        assert np.all(np.any(seg == hi[:, :, j:j + 1], axis=2))


def test_append_matches_rebuild():
    rng = np.random.default_rng(2)
    K = np.zeros((1, 2, 64, 4), np.float32)
    V = np.zeros_like(K)
    K[:, :, :13] = rng.standard_normal((1, 2, 13, 4))
    st = orc.State(K, V, 13, group=2)
    for _ in range(30):   # crosses the block boundaries at 16 and 32
        st.append(rng.standard_normal((1, 2, 4)).astype(np.float32),
                  rng.standard_normal((1, 2, 4)).astype(np.float32))
    lo, hi = orc.build_desc(st.K, st.length)
    M = orc.num_blocks(st.length)
    assert np.array_equal(st.lo[:, :, :M], lo) and np.array_equal(st.hi[:, :, :M], hi)


# ---------------------------------------------------------------- Quest bound
def test_quest_bound_hand_example():
    rows = {r[0]: [float(x) for x in r[1:]] for r in _rows("quest_bound_example.txt")}
    q = np.array([[rows["q0"], rows["q1"]]], np.float32)            # [1, 2, 2]
    lo = np.array(rows["lo"], np.float32).reshape(1, 1, 1, 2)
    hi = np.array(rows["hi"], np.float32).reshape(1, 1, 1, 2)
    # two blocks so that block 0 is not the (forced) local block
    lo2 = np.concatenate([lo, lo], axis=2)
    hi2 = np.concatenate([hi, hi], axis=2)
    s = orc.group_scores(q, lo2, hi2, 32, group=2)
    assert s[0, 0, 0] == rows["s"][0]
    assert s[0, 0, 1] == np.inf


def _true_block_max(q, K, length, group):
    """max over tokens t of block j of sum_h q_h . k_t, by direct dot products."""
    B, Hq, d = q.shape
    M = orc.num_blocks(length)
    out = np.empty((B, Hq // group, M))
    for b in range(B):
        for g in range(Hq // group):
            qsum = q[b, g * group:(g + 1) * group].astype(np.float64).sum(axis=0)
            dots = K[b, g, :length].astype(np.float64) @ qsum
            for j in range(M):
                out[b, g, j] = dots[j * 16:min(j * 16 + 16, length)].max()
    return out


def test_quest_bound_is_upper_bound():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((2, 8, 16)).astype(np.float32)
    K = rng.standard_normal((2, 2, 100, 16)).astype(np.float32)
    length = 97
    lo, hi = orc.build_desc(K, length)
    s = orc.group_scores(q, lo, hi, length, group=4)
    tmax = _true_block_max(q, K, length, 4)
    M = orc.num_blocks(length)
    assert np.all(s[:, :, :M - 1] >= tmax[:, :, :M - 1] - 1e-12)


def test_quest_bound_tight_when_d1_g1():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 3, 1)).astype(np.float32)
    K = rng.standard_normal((1, 3, 64, 1)).astype(np.float32)
    lo, hi = orc.build_desc(K, 64)
    s = orc.group_scores(q, lo, hi, 64, group=1)
    tmax = _true_block_max(q, K, 64, 1)
    assert np.allclose(s[:, :, :3], tmax[:, :, :3], rtol=0, atol=1e-12)


def test_quest_bound_tight_for_constant_blocks():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 4, 8)).astype(np.float32)
    rowvals = rng.standard_normal((1, 1, 4, 8)).astype(np.float32)
    K = np.repeat(rowvals, 16, axis=2)          # every block holds 16 copies of one key
    lo, hi = orc.build_desc(K, 64)
    s = orc.group_scores(q, lo, hi, 64, group=4)
    exact = (rowvals[0, 0].astype(np.float64) @ q[0].astype(np.float64).sum(0))
    assert np.allclose(s[0, 0, :3], exact[:3], rtol=0, atol=1e-12)


# ------------------------------------------------------------------- select
def _brute_select(s, n):
    """Repeated extraction of the best remaining block (lowest index on ties)."""
    M = len(s)
    left = list(range(M - 1))
    picked = [M - 1]
    for _ in range(min(n, M) - 1):
        best = left[0]
        for j in left[1:]:
            if s[j] > s[best]:
                best = j
        picked.append(best)
        left.remove(best)
    return sorted(picked)


@pytest.mark.parametrize("seed", range(6))
def test_select_matches_bruteforce_with_ties(seed):
    rng = np.random.default_rng(10 + seed)
    M = int(rng.integers(2, 60))
    s = rng.integers(-3, 4, size=M).astype(np.float64)   # many exact ties
    s[M - 1] = np.inf
    for n in (1, 2, 5, M // 2 + 1, M):
        assert list(orc.select_blocks(s, n)) == _brute_select(list(s), n)


def test_select_all_tied_takes_lowest():
    s = np.zeros(40)
    s[-1] = np.inf
    assert list(orc.select_blocks(s, 6)) == [0, 1, 2, 3, 4, 39]


def test_local_block_kept_even_if_lowest():
    rng = np.random.default_rng(6)
    K = rng.standard_normal((1, 1, 64, 8)).astype(np.float32)
    V = rng.standard_normal((1, 1, 64, 8)).astype(np.float32)
    K[0, 0, 48:] = -50.0     # last block would score lowest
    q = np.abs(rng.standard_normal((1, 1, 8))).astype(np.float32)
    st = orc.State(K, V, 63, group=1)
    res = st.decode(q, K[:, :, 63] * 0 - 50.0, V[:, :, 63], r=0.5, n_min=1, scale=1.0)
    s = res["scores"][0, 0]
    assert res["n"] == 2 and 3 in list(res["sel"][0, 0])
    # the local block's keys give the lowest true bound of all blocks
    lo, hi = orc.build_desc(st.K, 64)
    raw = orc.group_scores(q, lo, hi, 64, 1)[0, 0]   # local forced to +inf here too
    assert s[3] == np.inf and raw[3] == np.inf
    assert (q[0, 0].astype(np.float64) @ np.full(8, -50.0)) < min(s[:3])


# ---------------------------------------------------------------- attention
def _sdpa(q, K, V, scale, mask=None):
    """Library softmax attention in float64 (GQA by head // group)."""
    qt = torch.from_numpy(np.asarray(q, np.float64))
    kt = torch.from_numpy(np.asarray(K, np.float64))
    vt = torch.from_numpy(np.asarray(V, np.float64))
    m = None if mask is None else torch.from_numpy(mask)
    return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale,
                                          enable_gqa=True).numpy()


def _tiny_state(seed, B=1, Hq=4, Hkv=2, d=8, L=96, len0=70):
    rng = np.random.default_rng(seed)
    K = np.zeros((B, Hkv, L, d), np.float32)
    V = np.zeros_like(K)
    K[:, :, :len0] = rng.standard_normal((B, Hkv, len0, d))
    V[:, :, :len0] = rng.standard_normal((B, Hkv, len0, d))
    return rng, orc.State(K, V, len0, group=Hq // Hkv)


def test_dense_decode_equals_sdpa():
    rng, st = _tiny_state(7)
    q = rng.standard_normal((1, 4, 8)).astype(np.float32)
    O, _ = st.dense(q, 0.3)
    ref = _sdpa(q[:, :, None], st.K[:, :, :st.length], st.V[:, :, :st.length], 0.3)[:, :, 0]
    assert np.allclose(O, ref, rtol=0, atol=1e-12)


def test_r1_decode_equals_sdpa_including_new_token():
    rng, st = _tiny_state(8)
    q = rng.standard_normal((1, 4, 8)).astype(np.float32)
    kn = rng.standard_normal((1, 2, 8)).astype(np.float32)
    vn = rng.standard_normal((1, 2, 8)).astype(np.float32)
    res = st.decode(q, kn, vn, r=1.0, n_min=1, scale=0.5)
    assert st.length == 71 and res["n"] == orc.num_blocks(71)
    ref = _sdpa(q[:, :, None], st.K[:, :, :71], st.V[:, :, :71], 0.5)[:, :, 0]
    assert np.allclose(res["out"], ref, rtol=0, atol=1e-12)


def test_small_context_is_dense():
    rng, st = _tiny_state(9, len0=40)
    q = rng.standard_normal((1, 4, 8)).astype(np.float32)
    res = st.decode(q, None, None, r=0.1, n_min=16, scale=1.0)   # M = 3 <= n_min
    ref = _sdpa(q[:, :, None], st.K[:, :, :40], st.V[:, :, :40], 1.0)[:, :, 0]
    assert np.allclose(res["out"], ref, rtol=0, atol=1e-12)


def test_sparse_decode_equals_block_masked_sdpa():
    rng, st = _tiny_state(11, Hq=8, Hkv=2, d=16, L=400, len0=333)
    q = rng.standard_normal((1, 8, 16)).astype(np.float32)
    res = st.decode(q, None, None, r=0.2, n_min=2, scale=0.25)
    L = st.length
    # Eq. 2: token k of head h is visible iff its block floor(k/16) is selected
    mask = np.zeros((1, 8, 1, L), bool)
    for h in range(8):
        for j in res["sel"][0, h // 4]:
            mask[0, h, 0, j * 16:min(j * 16 + 16, L)] = True
    ref = _sdpa(q[:, :, None], st.K[:, :, :L], st.V[:, :, :L], 0.25, mask)[:, :, 0]
    assert np.allclose(res["out"], ref, rtol=0, atol=1e-12)
    # LSE against scipy on the visible logits
    for h in range(8):
        z = 0.25 * (st.K[0, h // 4, :L].astype(np.float64) @ q[0, h].astype(np.float64))
        assert abs(res["lse"][0, h] - logsumexp(z[mask[0, h, 0]])) < 1e-12


def test_sparse_selection_prefers_high_bound_blocks():
    """Blocks planted to align with the query must be selected."""
    rng, st0 = _tiny_state(12, Hq=4, Hkv=1, d=16, L=512, len0=480)
    qd = rng.standard_normal(16)
    qd /= np.linalg.norm(qd)
    K = st0.K.copy()
    for j in (3, 10, 20):
        K[0, 0, j * 16:(j + 1) * 16] += (8 * qd).astype(np.float32)
    st = orc.State(K, st0.V, st0.length, 4)
    q = np.tile(qd.astype(np.float32), (1, 4, 1))
    res = st.decode(q, None, None, r=0.1, n_min=4, scale=1.0)
    assert {3, 10, 20} <= set(res["sel"][0, 0].tolist())


# ------------------------------------------------------------------- rectify
def _rect_mask(length, f):
    pos = length - f + np.arange(f)
    return np.arange(length)[None, :] <= pos[:, None]


@pytest.mark.parametrize("length,f", [(70, 32), (64, 16), (33, 33), (100, 7)])
def test_rectify_equals_causal_sdpa(length, f):
    rng, st = _tiny_state(13, L=112, len0=length)
    q_f = rng.standard_normal((1, f, 4, 8)).astype(np.float32)
    k_f = rng.standard_normal((1, f, 2, 8)).astype(np.float32)
    v_f = rng.standard_normal((1, f, 2, 8)).astype(np.float32)
    O = st.rectify(q_f, k_f, v_f, f, 0.7)
    assert np.array_equal(st.K[0, :, length - f:length], np.transpose(k_f, (0, 2, 1, 3))[0])
    qt = np.transpose(q_f, (0, 2, 1, 3))
    ref = _sdpa(qt, st.K[:, :, :length], st.V[:, :, :length], 0.7,
                np.broadcast_to(_rect_mask(length, f), (1, 4, f, length)).copy())
    assert np.allclose(np.transpose(O, (0, 2, 1, 3)), ref, rtol=0, atol=1e-12)
    lo, hi = orc.build_desc(st.K, length)
    M = orc.num_blocks(length)
    assert np.array_equal(st.lo[:, :, :M], lo) and np.array_equal(st.hi[:, :, :M], hi)


def test_rectify_whole_sequence_is_causal_attention():
    rng, st = _tiny_state(14, len0=48)
    f = 48
    q_f = rng.standard_normal((1, f, 4, 8)).astype(np.float32)
    k_f = rng.standard_normal((1, f, 2, 8)).astype(np.float32)
    v_f = rng.standard_normal((1, f, 2, 8)).astype(np.float32)
    O = st.rectify(q_f, k_f, v_f, f, 1.0)
    qt = torch.from_numpy(np.transpose(q_f, (0, 2, 1, 3)).astype(np.float64))
    kt = torch.from_numpy(np.transpose(k_f, (0, 2, 1, 3)).astype(np.float64))
    vt = torch.from_numpy(np.transpose(v_f, (0, 2, 1, 3)).astype(np.float64))
    ref = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=1.0,
                                         enable_gqa=True).numpy()
    assert np.allclose(np.transpose(O, (0, 2, 1, 3)), ref, rtol=0, atol=1e-12)


# ------------------------------------------------------------------- prefill
def _prefill_case(seed, B=2, Hq=4, Hkv=2, d=8, L=80, length=53):
    rng = np.random.default_rng(seed)
    K = np.zeros((B, Hkv, L, d), np.float32)
    V = np.zeros_like(K)
    K[:, :, :length] = rng.standard_normal((B, Hkv, length, d))
    V[:, :, :length] = rng.standard_normal((B, Hkv, length, d))
    q = rng.standard_normal((B, length, Hq, d)).astype(np.float32)
    return q, K, V


@pytest.mark.parametrize("length", [1, 16, 53])
def test_prefill_equals_causal_sdpa(length):
    q, K, V = _prefill_case(21, length=length)
    O, lo, hi = orc.prefill(q, K, V, length, 0.6, group=2)
    qt = torch.from_numpy(np.transpose(q, (0, 2, 1, 3)).astype(np.float64))
    kt = torch.from_numpy(K[:, :, :length].astype(np.float64))
    vt = torch.from_numpy(V[:, :, :length].astype(np.float64))
    ref = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=0.6,
                                         enable_gqa=True).numpy()
    assert np.allclose(np.transpose(O, (0, 2, 1, 3)), ref, rtol=0, atol=1e-12)
    # the descriptors are the per-block min/max of the prompt's keys
    for j in range(orc.num_blocks(length)):
        blk = K[:, :, 16 * j:min(16 * j + 16, length)]
        assert np.array_equal(lo[:, :, j], blk.min(axis=2))
        assert np.array_equal(hi[:, :, j], blk.max(axis=2))


def test_prefill_rows_are_dense_decodes():
    """Row i of the prefill is a dense decode of query i over the first i + 1
    tokens (another code path of the oracle)."""
    q, K, V = _prefill_case(22, B=1, length=40)
    O, _, _ = orc.prefill(q, K, V, 40, 0.9, group=2)
    for i in (0, 15, 16, 39):
        st = orc.State(K, V, i + 1, group=2)
        Od, _ = st.dense(q[:, i], 0.9)
        assert np.allclose(O[:, i], Od, rtol=0, atol=1e-12)


def test_prefill_tail_is_the_rectification():
    """The last f rows equal a rectification of the same f tokens."""
    q, K, V = _prefill_case(23, B=1, length=50)
    O, _, _ = orc.prefill(q, K, V, 50, 1.0, group=2)
    st = orc.State(K, V, 50, group=2)
    f = 18
    k_f = np.transpose(K[:, :, 32:50], (0, 2, 1, 3)).copy()
    v_f = np.transpose(V[:, :, 32:50], (0, 2, 1, 3)).copy()
    Of = st.rectify(q[:, 32:50], k_f, v_f, f, 1.0)
    assert np.allclose(O[:, 32:50], Of, rtol=0, atol=1e-12)


# ------------------------------------------------------------ workload generator
def test_workload_bf16_rounding_is_exact_and_nearest():
    x = np.array([1.0, 1.00390625, 1.005859375, -3.14159, 1e-3], np.float32)
    y = round_to(x, "bf16")
    assert np.array_equal(round_to(y, "bf16"), y)                    # idempotent
    assert np.all(np.abs(y - x) <= np.abs(x) * 2.0 ** -8)            # nearest
    assert y[1] == 1.0                                               # tie -> even
    t = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(t, y)


def test_workload_steps_are_independent_of_history():
    spec = Spec(batch=1, n_q_heads=4, n_kv_heads=2, head_dim=8, len0=40, steps=8, dtype="f32")
    a = decode_inputs(spec, 5)
    decode_inputs(spec, 1)
    b = decode_inputs(spec, 5)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    K, V = make_cache(spec)
    assert K.shape == (1, 2, 48, 8) and np.all(K[:, :, 40:] == 0)
    q_f, k_f, v_f = rectify_inputs(spec, 0, 48, 16)
    assert q_f.shape == (1, 16, 4, 8) and k_f.shape == (1, 16, 2, 8)


# ------------------------------------------------- planted mistakes are caught
def _fails(fn):
    try:
        fn()
    except AssertionError:
        return True
    return False


def test_planted_mistakes_fail_a_pin(monkeypatch):
    """Plausible slips in the oracle (planted here, on the CPU) must trip a pin."""
    real_select, real_scores, real_attend = orc.select_blocks, orc.group_scores, orc.attend
    real_budget = orc.num_selected

    def select_ties_high(s_row, n):        # ties to the higher index
        M = s_row.shape[0]
        others = np.arange(M - 1)
        order = np.lexsort((-others, -s_row[: M - 1]))
        return np.sort(np.concatenate([others[order[: n - 1]], [M - 1]])).astype(np.int32)

    def select_drop_local(s_row, n):       # local block not forced
        s = s_row.copy()
        s[-1] = -np.inf
        M = s.shape[0]
        order = np.lexsort((np.arange(M), -s))
        return np.sort(order[:n]).astype(np.int32)

    def scores_max_over_heads(q, lo, hi, length, group):   # pooled by max, not sum
        s = real_scores(q, lo, hi, length, group)
        M = orc.num_blocks(length)
        B, Hq, d = q.shape
        for b in range(B):
            for g in range(Hq // group):
                qg = q[b, g * group:(g + 1) * group].astype(np.float64)
                L, U = lo[b, g, :M].astype(np.float64), hi[b, g, :M].astype(np.float64)
                t = np.maximum(qg[:, None] * L[None], qg[:, None] * U[None]).sum(2)
                s[b, g, :M - 1] = t.max(0)[:M - 1]
        return s

    def scores_wrong_sign(q, lo, hi, length, group):   # min instead of max
        return real_scores(-q, lo, hi, length, group) * -1.0 + 0.0

    def budget_no_guard(M, r, n_min):
        return int(min(M, max(n_min, math.ceil(M * r))))

    def attend_drops_last_token(q, K, V, sel, length, scale, group):
        return real_attend(q, K, V, sel, length - 1, scale, group)

    real_prefill = orc.prefill

    def prefill_sees_next_token(q, K, V, length, scale, group):   # mask t <= i + 1
        O, lo, hi = real_prefill(q, K, V, length, scale, group)
        B, L, Hq, d = q.shape
        vis = np.arange(L)[None, :] <= np.arange(L)[:, None] + 1
        for b in range(B):
            for h in range(Hq):
                k = K[b, h // group, :L].astype(np.float64)
                v = V[b, h // group, :L].astype(np.float64)
                z = np.where(vis, scale * (q[b, :, h].astype(np.float64) @ k.T), -np.inf)
                p = np.exp(z - z.max(axis=1, keepdims=True))
                O[b, :, h] = (p @ v) / p.sum(axis=1, keepdims=True)
        return O, lo, hi

    cases = [
        ("select_blocks", select_ties_high, test_select_all_tied_takes_lowest),
        ("select_blocks", select_drop_local, lambda: test_local_block_kept_even_if_lowest()),
        ("group_scores", scores_max_over_heads, test_quest_bound_hand_example),
        ("group_scores", scores_wrong_sign, test_quest_bound_is_upper_bound),
        ("num_selected", budget_no_guard, test_num_selected_golden),
        ("attend", attend_drops_last_token, test_r1_decode_equals_sdpa_including_new_token),
        ("prefill", prefill_sees_next_token, lambda: test_prefill_equals_causal_sdpa(53)),
    ]
    for name, bad, pin in cases:
        with monkeypatch.context() as mp:
            mp.setattr(orc, name, bad)
            mp.setattr(orc.resa_oracle, name, bad)   # the name State's methods resolve
            assert _fails(pin), f"planted mistake in {name} ({bad.__name__}) went unnoticed"
    assert orc.select_blocks is real_select and orc.num_selected is real_budget
