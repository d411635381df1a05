"""The selection parity rule itself (tests/pair.py::check_selection), on the
CPU: the near-tie branch must reject lists that drop a clearly better block,
take a block below the band or leave a better block out by more than the
band, and accept every valid choice inside it."""
import numpy as np
import pytest

from tests.pair import GAP, check_selection

INF = np.inf


def test_dropping_the_best_block_is_rejected_inside_a_near_tie():
    # blocks 1..3 tie within the band; block 0 (score 10) is clearly above it
    scores = np.array([10.0, 5.0, 5.0000001, 5.0000002, INF])
    with pytest.raises(AssertionError):
        check_selection(np.array([1, 2, 4]), scores, 3)


def test_valid_choices_inside_a_near_tie_are_accepted():
    scores = np.array([10.0, 5.0, 5.0000001, 5.0000002, INF])
    for pick in (1, 2, 3):
        assert check_selection(np.array(sorted([0, pick]) + [4]), scores, 3) is False


def test_a_block_below_the_band_is_rejected():
    scores = np.array([10.0, 5.0, 5.0000001, 1.0, INF])
    # n = 3: the oracle keeps 0 and 2; 1 and 2 are near-tied; 3 lies far below
    with pytest.raises(AssertionError):
        check_selection(np.array([0, 3, 4]), scores, 3)
    assert check_selection(np.array([0, 1, 4]), scores, 3) is False


def test_clear_gap_requires_the_oracle_set():
    scores = np.array([3.0, 9.0, 1.0, 7.0, 2.0, INF])
    assert check_selection(np.array([1, 3, 5]), scores, 3) is True
    with pytest.raises(AssertionError):
        check_selection(np.array([0, 1, 5]), scores, 3)


def test_structure_checks():
    scores = np.array([3.0, 9.0, 1.0, 7.0, 2.0, INF])
    for bad in ([3, 1, 5], [1, 1, 5], [1, 3, 4], [1, 5]):
        with pytest.raises(AssertionError):
            check_selection(np.array(bad), scores, 3)


def test_exchange_rule_inside_the_band():
    # s_(n) = s and s_(n+1) = s - d/2 tie within the band [s - 1.5 d, s + d];
    # block 3 lies inside the band too, but taking it over block 1 would let an
    # unselected block beat a selected one by 1.4 d
    s = 1e6
    d = GAP * s
    scores = np.array([s + 5 * d, s, s - 0.5 * d, s - 1.4 * d, INF])
    assert check_selection(np.array([0, 1, 4]), scores, 3) is False
    assert check_selection(np.array([0, 2, 4]), scores, 3) is False
    with pytest.raises(AssertionError):
        check_selection(np.array([0, 3, 4]), scores, 3)


def _fp32_scores(q, lo, hi, order):
    """The group score evaluated in float32 the way the kernel folds it
    (N_c, P_c per channel, then the 2d products summed in float32 in the
    given channel order)."""
    q32 = q.astype(np.float32)
    N = np.minimum(q32, 0).sum(axis=0, dtype=np.float32)
    P = np.maximum(q32, 0).sum(axis=0, dtype=np.float32)
    terms = np.concatenate([N[None, :] * lo, P[None, :] * hi], axis=1).astype(np.float32)
    terms = terms[:, order]
    acc = np.zeros(terms.shape[0], dtype=np.float32)
    for i in range(terms.shape[1]):
        acc = (acc + terms[:, i]).astype(np.float32)
    return acc


def test_fp32_score_error_bound_covers_fp32_evaluations():
    import oracle as orc
    from tests.pair import fp32_score_error
    from workload import round_to
    rng = np.random.default_rng(3)
    G, d, M = 4, 64, 300
    q = round_to(rng.standard_normal((1, G, d)).astype(np.float32) / 8, "bf16")
    K = round_to(rng.standard_normal((1, 1, M * 16, d)).astype(np.float32) * 3, "bf16")
    lo, hi = orc.build_desc(K, M * 16)
    exact = orc.group_scores(q, lo, hi, M * 16, G)[0, 0, : M - 1]
    err = fp32_score_error(q, lo, hi, M)[0, 0, : M - 1]
    worst = 0.0
    for order in (np.arange(2 * d), np.arange(2 * d)[::-1], rng.permutation(2 * d)):
        got = _fp32_scores(q[0], lo[0, 0, : M - 1], hi[0, 0, : M - 1], order).astype(np.float64)
        dev = np.abs(got - exact)
        assert np.all(dev <= err)
        worst = max(worst, float((dev / err).max()))
    assert worst > 1e-3   # the bound is not vacuous


def test_error_bound_makes_a_separated_near_tie_exact():
    # relative gap 5e-5 (inside the 1e-4 band) but error bounds of 1e-6
    scores = np.array([1.0, 1.0 - 5e-5, 0.5, INF])
    err = np.full(4, 1e-6)
    assert check_selection(np.array([0, 3]), scores, 2, err) is True
    with pytest.raises(AssertionError):
        check_selection(np.array([1, 3]), scores, 2, err)
    # without the bound block 1 is an admissible near-tie choice
    assert check_selection(np.array([1, 3]), scores, 2) is False
