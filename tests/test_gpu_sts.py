"""Sequential temperature scaling and ECE on the GPU against the oracle."""

import numpy as np
import pytest
import torch

import oracle as O
from speculative_decoding_04_b200 import dspark as D
from speculative_decoding_04_b200 import inputs
from tests.parity import dev, host

pytestmark = pytest.mark.gpu
GRID = np.exp(np.linspace(np.log(0.25), np.log(4.0), 81))


def fit_both(c, n, grid, n_bins=15):
    g = D.sts_fit(dev(c), dev(n.astype(np.int32)), dev(grid), n_bins, want_curve=True)
    torch.cuda.synchronize()
    g = {k: (host(v) if v is not None else None) for k, v in g.items()}
    # the oracle follows the device's choice wherever that choice is within 1e-12 of its own
    # minimum (the fp64 sums differ in order); anything else raises
    r = O.sts_fit(c, n, grid, n_bins, near=1e-12, follow=g["index"])
    return g, r


def check(g, r):
    assert np.array_equal(g["tau"], np.asarray(r["tau"]))
    assert np.allclose(g["ece_raw"], r["ece_raw"], rtol=1e-12, atol=1e-15)
    assert np.allclose(g["ece_cal"], r["ece_cal"], rtol=1e-12, atol=1e-15)
    assert np.allclose(g["curve"], r["curves"], rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("N,G", [(1, 3), (777, 5), (50_000, 8)])
def test_fit_matches_oracle_on_the_validation_set(N, G):
    c, n = inputs.calibration_set(N, G, seed=N + G)
    g, r = fit_both(c, n, GRID)
    check(g, r)
    if N >= 50_000:
        assert np.all(g["ece_cal"] < g["ece_raw"]) and np.all(g["ece_cal"] < 0.02)


def test_fit_recovers_known_temperatures():
    from scipy.special import expit, logit
    rng = np.random.default_rng(63)
    N, scales = 100_000, np.array([2.0, 0.5, 1.5, 3.0])
    q = rng.beta(4, 2, size=(N, scales.size))
    n = np.cumprod(rng.random(q.shape) < q, axis=1).sum(axis=1).astype(np.int32)
    c = expit(logit(q) * scales[None, :]).astype(np.float32)
    g, r = fit_both(c, n, GRID)
    check(g, r)
    assert np.all(np.abs(np.log(g["tau"]) - np.log(scales)) < 0.1)


def test_fit_edge_values_and_bins():
    # confidences at 0, 1, NaN and outside [0, 1]; a coarse grid; 4 bins and 1 bin
    rng = np.random.default_rng(64)
    c = rng.random((3000, 4)).astype(np.float32)
    c[::7, 0] = 0.0
    c[::11, 1] = 1.0
    c[::13, 2] = np.nan
    c[::17, 3] = 1.5
    c[::19, 3] = -0.5
    n = rng.integers(0, 5, 3000).astype(np.int32)
    for bins in (4, 1):
        g, r = fit_both(c, n, np.array([0.5, 1.0, 2.0]), n_bins=bins)
        check(g, r)


def test_apply_matches_oracle_and_keeps_order():
    wl = inputs.SCHEDULED_STEP
    c = inputs.confidences(wl)
    c[0, :3] = [0.0, 1.0, np.nan]
    tau = np.linspace(0.7, 2.5, wl.gamma)
    out = host(D.sts_apply(dev(c), dev(tau)))
    want = np.stack([O.sts_scale(c[:, k], tau[k]) for k in range(wl.gamma)], axis=1).astype(np.float32)
    # both sides scale in fp64 and round once to fp32: equal but for a rare double rounding
    ulp = np.abs(out.view(np.int32).astype(np.int64) - want.view(np.int32).astype(np.int64))
    assert ulp.max() <= 1 and (ulp > 0).mean() < 1e-3
    for k in range(wl.gamma):   # order preserved per position (ties allowed after rounding)
        o = np.argsort(np.nan_to_num(c[:, k], nan=0.0), kind="stable")
        assert np.all(np.diff(out[o, k]) >= 0)


def test_calibrated_confidences_feed_the_scheduler():
    # STS fitted on a validation set, applied to a round, then the scheduler: the device's
    # calibrated confidences and schedule against the oracle's
    c_val, n_val = inputs.calibration_set(20_000, 5, seed=71)
    g = D.sts_fit(dev(c_val), dev(n_val), dev(GRID))
    wl = inputs.SCHEDULED_STEP
    c = inputs.confidences(wl.with_(conf_a=9.0, conf_b=1.5))
    cc = D.sts_apply(dev(c), g["tau"])
    L, a, th, fl = D.prefix_schedule(cc, dev(inputs.sps_table(wl)), wl.D_max)
    torch.cuda.synchronize()
    r = O.sts_fit(c_val, n_val, GRID, follow=host(g["index"]))
    cal = np.stack([O.sts_scale(c[:, k], r["tau"][k]) for k in range(wl.gamma)], axis=1).astype(np.float32)
    got = host(cc)
    assert np.abs(got.view(np.int32).astype(np.int64) - cal.view(np.int32).astype(np.int64)).max() <= 1
    s = O.prefix_schedule(cal, inputs.sps_table(wl), wl.D_max)
    if np.array_equal(got, cal):   # the usual case: the schedule is then exact
        assert np.array_equal(host(a), s["a"])
        if not (s["near_tie"] or host(fl)[0] & D.FLAG_SCHED_NEAR_TIE):
            assert np.array_equal(host(L), s["L"])
    else:
        assert np.allclose(host(a), s["a"], rtol=1e-5, atol=0)
