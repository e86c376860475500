"""The five workloads at full size, in the launch configuration the benchmark times,
checked against the oracle (all requests where the oracle finishes in seconds,
sampled requests on the vocabulary sweep)."""

import json
import os

import numpy as np
import pytest
import torch

import oracle as O
from speculative_decoding_04_b200 import dspark as D
from speculative_decoding_04_b200 import inputs
from tests.parity import check_draft, check_labels, check_verify, dev, dev_weights, host, host_rm, pm

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def gpu_round(d, wl, L=None, want_c=True):
    W1, W2 = dev_weights(d["W1"], d["W2"], wl.w_dtype)
    x, ld, fl = D.markov_draft(pm(d["U"]), W1, W2, dev(d["x0"]), dev(d["u_draft"]), wl.T)
    n, y, c, fl = D.verify(ld, dev(d["lt"]), x, None if L is None else dev(L), dev(d["u_acc"]), dev(d["u_res"]),
                           wl.T, want_c_star=want_c, flags=fl)
    torch.cuda.synchronize()
    return host(x), host_rm(ld), host(n), host(y), (host(c) if c is not None else None), host(fl)


def test_tiny_round_matches_golden_fixture():
    wl = inputs.TINY
    d = inputs.full_inputs(wl)
    x, ld, n, y, c, fl = gpu_round(d, wl)
    with open(os.path.join(HERE, "golden", "tiny_round.json")) as f:
        g = json.load(f)
    if not fl.any():
        assert x.tolist() == g["x"] and n.tolist() == g["n_acc"] and y.tolist() == g["y"]
    np.testing.assert_allclose(c, g["c_star"], rtol=1e-5, atol=1e-9)
    check_draft(d["U"], d["W1"], d["W2"], d["x0"], d["u_draft"], wl.T, x, ld, fl)
    check_verify(ld, d["lt"], x, None, d["u_acc"], d["u_res"], wl.T, n, y, flags_gpu=fl)


@pytest.mark.parametrize("wl", [inputs.SINGLE_USER, inputs.SINGLE_USER_GREEDY], ids=lambda w: w.name)
def test_single_user(wl):
    d = inputs.full_inputs(wl)
    x, ld, n, y, c, fl = gpu_round(d, wl)
    check_draft(d["U"], d["W1"], d["W2"], d["x0"], d["u_draft"], wl.T, x, ld, fl)
    check_verify(ld, d["lt"], x, None, d["u_acc"], d["u_res"], wl.T, n, y, flags_gpu=fl)
    check_labels(ld, d["lt"], wl.T, c)


def test_high_concurrency_all_requests():
    wl = inputs.HIGH_CONCURRENCY
    d = inputs.full_inputs(wl)
    x, ld, n, y, c, fl = gpu_round(d, wl)
    check_draft(d["U"], d["W1"], d["W2"], d["x0"], d["u_draft"], wl.T, x, ld, fl)
    check_verify(ld, d["lt"], x, None, d["u_acc"], d["u_res"], wl.T, n, y, flags_gpu=fl)
    check_labels(ld, d["lt"], wl.T, c)
    # suffix decay of the synthetic target: later positions agree less
    assert c[:, :4].mean() > c[:, -4:].mean()


def test_scheduled_step():
    wl = inputs.SCHEDULED_STEP
    d = inputs.full_inputs(wl)
    Lg, a, th, sfl = D.prefix_schedule(dev(d["c"]), dev(d["sps"]), wl.D_max, D.SCHED_ARGMAX)
    Lg = host(Lg)
    r = O.prefix_schedule(d["c"], d["sps"], wl.D_max)
    if not (r["near_tie"] or host(sfl)[0] & D.FLAG_SCHED_NEAR_TIE):
        assert np.array_equal(Lg, r["L"])
    assert float(host(th)[0]) == pytest.approx(r["theta"], rel=1e-12)
    for want_c in (False, True):   # labels of every position are computed whatever L is
        x, ld, n, y, c, fl = gpu_round(d, wl, L=Lg, want_c=want_c)
        check_draft(d["U"], d["W1"], d["W2"], d["x0"], d["u_draft"], wl.T, x, ld, fl)
        check_verify(ld, d["lt"], x, Lg, d["u_acc"], d["u_res"], wl.T, n, y, flags_gpu=fl)
        assert np.all(n <= Lg)
        if want_c:
            check_labels(ld, d["lt"], wl.T, c)


@pytest.mark.parametrize("B", inputs.SWEEP_B)
@pytest.mark.parametrize("gamma", inputs.SWEEP_GAMMA)
def test_vocabulary_sweep(B, gamma):
    wl = inputs.sweep_point(B, gamma)
    U, lt = inputs.device_logits(wl, "cuda")
    W1h, W2h = inputs.weights(wl)
    W1, W2 = dev_weights(W1h, W2h, "bf16")
    x0 = inputs.tokens(wl)
    u_draft, u_acc, u_res = inputs.uniforms(wl)
    x, ld, fl = D.markov_draft(U, W1, W2, dev(x0), dev(u_draft), wl.T)
    n, y, c, fl = D.verify(ld, lt, x, None, dev(u_acc), dev(u_res), wl.T, want_c_star=True, flags=fl)
    torch.cuda.synchronize()
    xh, nh, yh = host(x), host(n), host(y)
    assert xh.min() >= 0 and xh.max() < wl.V and np.all(nh <= gamma)
    for b in range(B):
        assert np.array_equal(yh[b, :nh[b]], xh[b, :nh[b]]) and np.all(yh[b, nh[b] + 1:] == -1)
    # oracle on sampled requests (the requests are independent)
    reqs = sorted({0, B - 1, B // 2})
    Uh, lth, ldh = host_rm(U[:, reqs]), host(lt[reqs]), host_rm(ld[:, reqs])
    sub = dict(U=Uh, x0=x0[reqs], u=u_draft[reqs])
    flh = host(fl)[reqs]
    check_draft(sub["U"], W1h, W2h, sub["x0"], sub["u"], wl.T, xh[reqs], ldh, flh)
    check_verify(ldh, lth, xh[reqs], None, u_acc[reqs], u_res[reqs], wl.T, nh[reqs], yh[reqs], flags_gpu=flh)
    check_labels(ldh, lth, wl.T, host(c)[reqs])
    del U, lt, ld
    torch.cuda.empty_cache()
