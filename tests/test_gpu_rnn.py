"""The recurrent (RNN) draft head on the GPU against the oracle."""

import numpy as np
import pytest
import torch

import oracle as O
from speculative_decoding_04_b200 import dspark as D
from speculative_decoding_04_b200 import inputs
from tests.parity import LD_TOL, check_draft_flags, dev, dev_weights, host, host_rm, pm

pytestmark = pytest.mark.gpu


def rnn_case(B, G, V, r, T, w_dtype, seed):
    wl = inputs.SINGLE_USER.with_(name="rnn", B=B, gamma=G, V=V, r=r, T=T, seed=seed, w_sigma=0.05, w_dtype=w_dtype)
    d = inputs.full_inputs(wl)
    Wh = np.random.default_rng(seed).normal(0, 1.0 / np.sqrt(r), (r, r)).astype(np.float32)
    if w_dtype == "bf16":
        Wh = inputs.round_to_bf16(Wh)
    return wl, d, Wh


def check_rnn(d, Wh, T, x, ld, h, fl):
    follow = {(b, k): int(x[b, k]) for b in range(x.shape[0]) for k in range(x.shape[1])}
    x_o, ld_o, _, h_o = O.rnn_draft(d["U"], d["W1"], d["W2"], Wh, d["x0"], d["u_draft"], T, follow=follow)
    assert np.array_equal(x_o, x)
    err = np.abs(ld.astype(np.float64) - ld_o) / np.maximum(1.0, np.abs(ld_o.astype(np.float64)))
    assert err.max() <= LD_TOL, f"l_d max scaled error {err.max():.3e}"
    if h is not None:
        assert np.abs(h - h_o).max() <= 1e-5
    check_draft_flags(ld_o, x_o, d["u_draft"], T, fl, list(range(x.shape[0])))


@pytest.mark.parametrize("w_dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,r", [(3, 64), (40, 256), (9, 100)])
@pytest.mark.parametrize("T", [1.0, 0.0])
def test_rnn_draft_matches_oracle(w_dtype, B, r, T):
    G, V = 4, 4104
    wl, d, Wh = rnn_case(B, G, V, r, T, w_dtype, seed=500 + B + r)
    W1, W2 = dev_weights(d["W1"], d["W2"], w_dtype)
    Whd = dev(Wh, torch.bfloat16 if w_dtype == "bf16" else torch.float32)
    x, ld, h, fl = D.rnn_draft(pm(d["U"]), W1, W2, Whd, dev(d["x0"]), dev(d["u_draft"]), T, want_h=True)
    torch.cuda.synchronize()
    check_rnn(d, Wh, T, host(x), host_rm(ld), host(h), host(fl))


def test_rnn_draft_request_major_and_prefix_dependence():
    # request-major U; and two requests that draft the same first token after different x0
    B, G, V, r, T = 2, 3, 4096, 64, 1.0
    wl, d, Wh = rnn_case(B, G, V, r, T, "bf16", seed=555)
    d["U"][:, 0, 7] = 60.0
    d["x0"][:] = [3, 11]
    W1, W2 = dev_weights(d["W1"], d["W2"], "bf16")
    x, ld, h, fl = D.rnn_draft(dev(d["U"]), W1, W2, dev(Wh, torch.bfloat16), dev(d["x0"]), dev(d["u_draft"]), T,
                               layout="request", want_h=True)
    torch.cuda.synchronize()
    x, ld = host(x), host(ld)
    assert x[0, 0] == x[1, 0] == 7
    check_rnn(d, Wh, T, x, ld, host(h), host(fl))
    # the state still carries x0: position 1's bias differs although x_0 agrees
    bias1 = ld[:, 1].astype(np.float64) - d["U"][:, 1]
    assert not np.allclose(bias1[0], bias1[1])


def test_rnn_draft_rejects_bad_arguments():
    U = torch.zeros((2, 3, 64), device="cuda")
    W1 = torch.zeros((64, 8), device="cuda")
    W2 = torch.zeros((8, 64), device="cuda")
    with pytest.raises(ValueError):
        D.rnn_draft(U, W1, W2, torch.zeros((8, 4), device="cuda"), torch.zeros(3, dtype=torch.int32, device="cuda"),
                    torch.zeros((3, 2), device="cuda"), 1.0)
    big = torch.zeros((64, 1025), device="cuda")
    ws = D.workspace(D.WS_RNN_DRAFT, 3, 2, 64, 1025)
    st = D.lib.dspark_rnn_draft(D._p(U), D._p(big), D._p(big), D._p(big), D.F32,
                                D._p(torch.zeros(3, dtype=torch.int32, device="cuda")), None, 3, 2, 64, 1025, 0.0, 0,
                                D._p(torch.empty((3, 2), dtype=torch.int32, device="cuda")), D._p(torch.empty_like(U)),
                                None, D._p(torch.zeros(3, dtype=torch.int32, device="cuda")), D._p(ws), ws.numel(), None)
    assert st == D.EINVAL and "1024" in D.last_error()
