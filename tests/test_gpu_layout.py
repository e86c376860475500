"""Request-major draft logits ([B, gamma, V], as a backbone that emits a request's positions
together writes them) on every path, against the oracle and against the position-major call."""

import numpy as np
import pytest
import torch

from speculative_decoding_04_b200 import dspark as D
from speculative_decoding_04_b200 import inputs
from tests.parity import check_draft, check_labels, check_verify, dev, dev_weights, draw_tokens, host, pm

pytestmark = pytest.mark.gpu


def small(B, G, V, r, T, seed):
    wl = inputs.SINGLE_USER.with_(name="layout", B=B, gamma=G, V=V, r=r, T=T, seed=seed, w_sigma=0.05)
    return wl, inputs.full_inputs(wl)


@pytest.mark.parametrize("path,fused", [(2, 1), (2, 0), (1, 1)])
@pytest.mark.parametrize("B", [5, 40, 100])
@pytest.mark.parametrize("T", [1.0, 0.0])
def test_draft_request_major(path, fused, B, T):
    # V = 4104: ragged last tile; B = 100 takes two request groups on the tensor-core path
    wl, d = small(B, 4, 4104, 64, T, seed=600 + B + path + fused)
    W1, W2 = dev_weights(d["W1"], d["W2"], "bf16")
    D.set_option("draft_path", path)
    D.set_option("draft_fused", fused)
    x, ld, fl = D.markov_draft(dev(d["U"]), W1, W2, dev(d["x0"]), dev(d["u_draft"]), wl.T, layout="request")
    torch.cuda.synchronize()
    assert tuple(ld.shape) == (B, 4, wl.V)
    x, ld, fl = host(x), host(ld), host(fl)
    check_draft(d["U"], d["W1"], d["W2"], d["x0"], d["u_draft"], wl.T, x, ld, fl)
    # the same tokens and logits as the position-major call
    x2, ld2, _ = D.markov_draft(pm(d["U"]), W1, W2, dev(d["x0"]), dev(d["u_draft"]), wl.T)
    torch.cuda.synchronize()
    near = (fl & D.FLAG_DRAFT_NEAR_TIE) != 0
    assert np.array_equal(host(x2)[~near], x[~near])
    assert np.array_equal(host(ld2).transpose(1, 0, 2)[~near], ld[~near])


@pytest.mark.parametrize("impl", ["stream", "sliced", "rows", "noalloc"])
@pytest.mark.parametrize("T", [0.9, 0.0])
def test_verify_request_major(impl, T):
    wl = inputs.SINGLE_USER.with_(name="layout_v", B=12, gamma=5, V=20000, T=T, seed=610)
    ld, lt = inputs.logits(wl)
    u_draft, u_acc, u_res = inputs.uniforms(wl)
    x = draw_tokens(ld, u_draft, T)
    L = (np.arange(wl.B) * 5 % (wl.gamma + 1)).astype(np.int32)
    D.set_option("verify_impl", {"stream": 0, "sliced": 1, "rows": 2, "noalloc": 0}[impl])
    for Lc in (None, L):
        args = (dev(ld), dev(lt), dev(x), None if Lc is None else dev(Lc), dev(u_acc), dev(u_res), T)
        if impl == "noalloc":
            n, y, c, fl = D.verify_noalloc(*args, want_c_star=True, ld_layout="request")
        else:
            n, y, c, fl = D.verify(*args, want_c_star=True, ld_layout="request")
        torch.cuda.synchronize()
        check_verify(ld, lt, x, Lc, u_acc, u_res, T, host(n), host(y), flags_gpu=host(fl))
        check_labels(ld, lt, T, host(c))


@pytest.mark.parametrize("T", [1.0, 0.0])
def test_tv_labels_request_major(T):
    wl = inputs.SINGLE_USER.with_(name="layout_l", B=6, gamma=4, V=30000, T=T, seed=620)
    ld, lt = inputs.logits(wl)
    c = host(D.tv_labels(dev(ld), dev(lt), T, ld_layout="request"))
    check_labels(ld, lt, T, c)
