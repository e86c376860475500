"""Pins of the oracle's near-tie machinery.

Every GPU parity test excuses a disagreement only where the oracle reports a near-tie
(a decision within 1e-6 of its threshold, a greedy top-2 gap within 1e-6*max(1,|z|), or a
scheduler objective within 1e-12 relative) and then lets the oracle follow the GPU's branch.
These checks pin that machinery on both sides of each window, with thresholds computed here
from closed forms (logistic two-token probabilities, uniform CDFs, exact Θ values), so a window
that is too wide, too narrow or applied to the wrong quantity fails one of them:
  * a decision just inside the window is reported as a tie, one just outside is not;
  * forcing an outcome that is not valid within the window raises.
"""

import numpy as np
import pytest
from scipy.special import expit

import oracle as O

W = O.NEAR_TIE
IN, OUT = 0.9, 1.1   # fractions of the window: just inside, just outside


# --------------------------------------------------------------------------- inverse CDF (draft, residual, bonus)

@pytest.mark.parametrize("side", [+1, -1])
def test_inverse_cdf_window_edges(side):
    p = np.full(4, 0.25)            # boundaries at F = 0.25, 0.5, 0.75
    v, alts = O.inverse_cdf(p, 0.5 + side * IN * W)
    assert alts == [1, 2] and v == (2 if side > 0 else 1)
    v, alts = O.inverse_cdf(p, 0.5 + side * OUT * W)
    assert alts == [v] and v == (2 if side > 0 else 1)


def test_inverse_cdf_window_scales_with_argument():
    p = np.full(4, 0.25)
    assert O.inverse_cdf(p, 0.5 + 5e-6, near=1e-5)[1] == [1, 2]
    assert O.inverse_cdf(p, 0.5 + 5e-6, near=1e-6)[1] == [2]


def test_inverse_cdf_window_skips_zero_mass_neighbours():
    p = np.array([0.5, 0.0, 0.5])
    # u just above F_0 = 0.5: token 2 is drawn, token 0 is the near-tie alternative, the
    # zero-mass token 1 is never valid
    assert O.inverse_cdf(p, 0.5 + IN * W)[1] == [0, 2]


# --------------------------------------------------------------------------- acceptance (T > 0)

def _two_token_position(a, b):
    """One drafted position over a two-token vocabulary, drafted token 1, T = 1:
    p_d(1) = expit(a), p_t(1) = expit(b) (closed form, independent of the oracle's softmax)."""
    ld = np.array([[0.0, a]], dtype=np.float32)
    lt = np.array([[0.0, b], [0.0, 0.0]], dtype=np.float32)
    x = np.array([1], dtype=np.int32)
    ratio = expit(np.float64(np.float32(b))) / expit(np.float64(np.float32(a)))
    return ld, lt, x, float(ratio)


@pytest.mark.parametrize("frac,tie", [(IN, True), (OUT, False)])
@pytest.mark.parametrize("side", [-1, +1])
def test_acceptance_window_edges(frac, tie, side):
    ld, lt, x, ratio = _two_token_position(1.5, 0.25)   # p_t/p_d ≈ 0.69
    u = ratio + side * frac * W
    r = O.verify_request(ld, lt, x, 1, np.array([u]), 0.3, 1.0)
    assert r["n"] == (1 if side < 0 else 0)              # strict test u * p_d < p_t
    assert (r["accept_ties"] == [0]) == tie


def test_forcing_an_acceptance_outside_the_window_raises():
    ld, lt, x, ratio = _two_token_position(1.5, 0.25)
    u_in, u_out = ratio + IN * W, ratio + OUT * W        # both reject
    r = O.verify_request(ld, lt, x, 1, np.array([u_in]), 0.3, 1.0, force_accept={0: True})
    assert r["n"] == 1                                   # the near-tie may go either way
    with pytest.raises(ValueError):
        O.verify_request(ld, lt, x, 1, np.array([u_out]), 0.3, 1.0, force_accept={0: True})
    # forcing the outcome the oracle reached anyway is always allowed
    assert O.verify_request(ld, lt, x, 1, np.array([u_out]), 0.3, 1.0, force_accept={0: False})["n"] == 0


# --------------------------------------------------------------------------- residual / bonus sample

def test_bonus_sample_window_and_forced_token():
    # bonus row uniform over 4 tokens (zero logits): F = 0.25, 0.5, 0.75
    ld = np.zeros((1, 4), dtype=np.float32)
    lt = np.zeros((2, 4), dtype=np.float32)
    x = np.array([2], dtype=np.int32)
    u_acc = np.array([0.0])                               # u p_d < p_t: accepted, then the bonus
    r = O.verify_request(ld, lt, x, 1, u_acc, 0.75 - IN * W, 1.0)
    assert r["kind"] == "bonus" and r["y"][1] == 2 and r["sample_alts"] == [2, 3]
    assert O.verify_request(ld, lt, x, 1, u_acc, 0.75 - IN * W, 1.0, force_token=3)["y"][1] == 3
    r = O.verify_request(ld, lt, x, 1, u_acc, 0.75 - OUT * W, 1.0)
    assert r["sample_alts"] == [2]
    with pytest.raises(ValueError):
        O.verify_request(ld, lt, x, 1, u_acc, 0.75 - OUT * W, 1.0, force_token=3)


def test_residual_sample_window():
    # p_d one-hot on token 0, p_t uniform over tokens 1..4 after a certain rejection:
    # residual q = p_t, F = 0.25, 0.5, 0.75 over tokens 1..4
    ld = np.array([[0.0, -1e4, -1e4, -1e4, -1e4]], dtype=np.float32)
    lt = np.array([[-1e4, 0, 0, 0, 0], [0, 0, 0, 0, 0]], dtype=np.float32)
    x = np.array([0], dtype=np.int32)
    r = O.verify_request(ld, lt, x, 1, np.array([0.5]), 0.25 + IN * W, 1.0)
    assert r["n"] == 0 and r["kind"] == "residual" and r["sample_alts"] == [1, 2]
    assert r["residual_mass"] == pytest.approx(1.0, abs=1e-12)
    r = O.verify_request(ld, lt, x, 1, np.array([0.5]), 0.25 + OUT * W, 1.0)
    assert r["sample_alts"] == [2]


# --------------------------------------------------------------------------- greedy gap rule

@pytest.mark.parametrize("top", [0.5, -0.25, 100.0, -3000.0])
def test_greedy_gap_window_scales_with_magnitude(top):
    gap = W * max(1.0, abs(top))
    for frac, tie in ((0.8, True), (1.2, False)):
        z = np.array([top - 10 * gap, top, top - frac * gap], dtype=np.float32)
        # the fp32 values must straddle the window for the check to mean anything
        d = float(np.float64(z[1]) - np.float64(z[2]))
        assert (d <= gap) == tie
        x, alts = O.greedy_choice(z)
        assert x == 1 and alts == ([1, 2] if tie else [1])


def test_greedy_acceptance_tie_only_when_draft_is_among_the_tied():
    top = 2.0
    lt = np.array([[0.0, top, top - 0.5 * W * top, -5.0], [0.0, 0.0, 0.0, 1.0]], dtype=np.float32)
    ld = np.zeros((1, 4), dtype=np.float32)
    # drafted the runner-up inside the gap: rejected (not the argmax), but reported as a tie
    r = O.verify_request(ld, lt, np.array([2], dtype=np.int32), 1, np.zeros(1), 0.0, 0.0)
    assert r["n"] == 0 and r["accept_ties"] == [0]
    assert O.verify_request(ld, lt, np.array([2], dtype=np.int32), 1, np.zeros(1), 0.0, 0.0,
                            force_accept={0: True})["n"] == 1
    # drafted a token far below: a plain rejection, forcing acceptance raises
    r = O.verify_request(ld, lt, np.array([3], dtype=np.int32), 1, np.zeros(1), 0.0, 0.0)
    assert r["n"] == 0 and r["accept_ties"] == []
    with pytest.raises(ValueError):
        O.verify_request(ld, lt, np.array([3], dtype=np.int32), 1, np.zeros(1), 0.0, 0.0, force_accept={0: True})


def test_markov_draft_follow_rejects_tokens_outside_the_window():
    V = 4
    U = np.zeros((1, 1, V), dtype=np.float32)            # uniform: F = 0.25, 0.5, 0.75
    W1 = np.zeros((V, 2), dtype=np.float32)
    W2 = np.zeros((2, V), dtype=np.float32)
    x0 = np.array([0], dtype=np.int32)
    x, _, alts = O.markov_draft(U, W1, W2, x0, np.array([[0.5 + IN * W]]), 1.0, follow={(0, 0): 1})
    assert x[0, 0] == 1 and alts[(0, 0)] == [1, 2]
    with pytest.raises(ValueError):
        O.markov_draft(U, W1, W2, x0, np.array([[0.5 + OUT * W]]), 1.0, follow={(0, 0): 1})


# --------------------------------------------------------------------------- scheduler Θ window

def _one_item(delta, c=0.5):
    """B = 1, γ = 1: Θ(0) = sps[0] = 1 and Θ(1) = (1 + a)·sps[1] = 1 + delta (to fp64 rounding)."""
    cc = np.array([[c]], dtype=np.float32)
    a = float(np.float32(c))
    sps = np.array([1.0, (1.0 + delta) / (1.0 + a)])
    return cc, sps


@pytest.mark.parametrize("mode", [O.SCHED_ARGMAX, O.SCHED_EARLY_STOP])
def test_scheduler_theta_window_edges(mode):
    for delta, tie in ((0.5e-12, True), (2e-12, False), (-0.5e-12, True), (-2e-12, False)):
        c, sps = _one_item(delta)
        r = O.prefix_schedule(c, sps, 1, mode)
        assert r["near_tie"] == tie, (delta, mode)
        assert r["D"] == (1 if delta > 0 else 0)


def test_scheduler_window_argument():
    c, sps = _one_item(5e-12)
    assert not O.prefix_schedule(c, sps, 1)["near_tie"]
    assert O.prefix_schedule(c, sps, 1, near=1e-11)["near_tie"]
