"""Prefix survival and the prefix scheduler on the GPU against the oracle and exhaustive search."""

import numpy as np
import pytest
import torch

import oracle as O
from speculative_decoding_04_b200 import dspark as D
from speculative_decoding_04_b200 import inputs
from tests.parity import dev, host

pytestmark = pytest.mark.gpu


def run(c, sps, D_max, mode=0):
    L, a, th, fl = D.prefix_schedule(dev(c), dev(np.asarray(sps, dtype=np.float64)), D_max, mode)
    torch.cuda.synchronize()
    return host(L), host(a), float(host(th)[0]), host(fl)


def check(c, sps, D_max, mode=0):
    L, a, th, fl = run(c, sps, D_max, mode)
    r = O.prefix_schedule(c, sps, D_max, mode)
    assert np.array_equal(a, r["a"]), "prefix survival must be bit-exact (fp32 left-to-right products)"
    # the near-tie bit against the oracle with a 4x margin on each side of the 1e-12 window
    flagged = bool(fl[0] & D.FLAG_SCHED_NEAR_TIE)
    if O.prefix_schedule(c, sps, D_max, mode, near=0.25 * O.THETA_NEAR_TIE)["near_tie"]:
        assert flagged, "the oracle finds a scheduler near-tie the device did not flag"
    if flagged:
        assert O.prefix_schedule(c, sps, D_max, mode, near=4 * O.THETA_NEAR_TIE)["near_tie"]
    near = flagged or r["near_tie"]
    if not near:
        assert np.array_equal(L, r["L"])
        assert th == pytest.approx(r["theta"], rel=1e-12)
    else:
        assert th == pytest.approx(r["theta"], rel=1e-11)
    assert L.sum() <= D_max and np.all(L <= c.shape[1]) and np.all(L >= 0)
    return L, th, r


def staircase(n_max, B):
    n = B + np.arange(n_max + 1)
    return 1000.0 / (1.0 + np.ceil(n / 8.0))


@pytest.mark.parametrize("seed", range(20))
def test_tiny_matches_exhaustive_search(seed):
    rng = np.random.default_rng(seed)
    B, G = int(rng.integers(1, 5)), int(rng.integers(1, 5))
    c = rng.beta(4, 2, size=(B, G)).astype(np.float32)
    D_max = int(rng.integers(0, B * G + 1))
    for sps in (1.0 / (0.005 + 0.0004 * (B + np.arange(B * G + 1))), staircase(B * G, B),
                100.0 * (1.0 - (B + np.arange(B * G + 1)) / (2.0 * B * (G + 1)))):
        for mode in (O.SCHED_ARGMAX, O.SCHED_EARLY_STOP):
            L, th, r = check(c, sps, D_max, mode)
            if mode == O.SCHED_ARGMAX and B <= 3:
                best, arg = O.exhaustive_schedule(c, sps, D_max)
                assert th == pytest.approx(best, rel=1e-12)
                assert tuple(L.tolist()) in arg


@pytest.mark.parametrize("wl", [inputs.TINY, inputs.SCHEDULED_STEP], ids=lambda w: w.name)
@pytest.mark.parametrize("mode", [0, 1])
def test_workload_sizes(wl, mode):
    c = inputs.confidences(wl)
    check(c, inputs.sps_table(wl), wl.D_max, mode)
    check(c, inputs.sps_table(wl), wl.D_max // 3, mode)


def test_largest_batch_and_ties():
    rng = np.random.default_rng(1)
    B, G = 1024, 16
    c = rng.beta(6, 2, size=(B, G)).astype(np.float32)
    c[::7] = 0.5                                     # many identical survivals: the tie-break decides
    sps = 1.0 / (0.005 + 0.00004 * (B + np.arange(B * G + 1)))
    check(c, sps, B * G)
    check(c, sps, 5000)


def test_staircase_early_stop_vs_global():
    c = np.full((4, 4), 0.97, dtype=np.float32)
    sps = np.array([10.0, 6.0] + [5.9] * 15)
    Le, the, _ = check(c, sps, 16, 1)
    Lg, thg, _ = check(c, sps, 16, 0)
    assert Le.sum() == 0 and Lg.sum() == 16 and the < thg


def test_confidence_out_of_range_is_flagged():
    c = np.array([[0.5, 1.5], [0.2, 0.3], [-0.1, 0.9]], dtype=np.float32)
    L, a, th, fl = run(c, np.ones(7), 6)
    assert [bool(f & D.FLAG_CONF_RANGE) for f in fl] == [True, False, True]


@pytest.mark.parametrize("B,G", [(512, 16), (300, 7), (1, 9)])
def test_merged_runs_with_ties(B, G):
    # every confidence in [0, 1]: the kernel merges the requests' sorted runs (up to 8192 keys);
    # identical rows and exact 1.0 / 0.0 confidences make equal survivals across requests
    rng = np.random.default_rng(B + G)
    c = rng.beta(5, 2, size=(B, G)).astype(np.float32)
    c[::5] = 0.75
    c[1::9, 0] = 1.0
    c[2::11, G // 2] = 0.0
    sps = 1.0 / (0.005 + 0.00004 * (B + np.arange(B * G + 1)))
    check(c, sps, B * G)
    check(c, sps, (B * G) // 4, 1)


def test_unsorted_runs_take_the_bitonic_sort():
    # confidences above 1 make survivals rise along a request: the order must still be the
    # oracle's (survival descending, then request, then position)
    rng = np.random.default_rng(9)
    B, G = 64, 16
    c = rng.uniform(0.2, 1.3, size=(B, G)).astype(np.float32)
    sps = 1.0 / (0.005 + 0.00004 * (B + np.arange(B * G + 1)))
    L, th, r = check(c, sps, B * G)
    fl = run(c, sps, B * G)[3]
    assert np.any(fl & D.FLAG_CONF_RANGE)
