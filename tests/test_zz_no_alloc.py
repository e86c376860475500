"""dspark_verify_noalloc: verification for callers that cannot hand the library device scratch
(for example a serving engine that has reserved nearly all HBM for its KV cache and forbids
further allocation while decoding, or plugin code given raw device pointers but no allocator).
It must give the oracle's results and those of dspark_verify with a workspace, call after call,
although every call reuses the same fixed scratch array inside the library, at every size its
documented limits allow.

This file is collected last on purpose: a run that stops at the first failure has then already
run every other test."""

import numpy as np
import pytest
import torch

from speculative_decoding_04_b200 import dspark as D
from speculative_decoding_04_b200 import inputs
from tests.parity import (FLAG_ACCEPT_NEAR_TIE, FLAG_SAMPLE_NEAR_TIE, P_ATOL, P_RTOL, check_labels, check_verify,
                          dev, draw_tokens, host, pm)

pytestmark = pytest.mark.gpu
TIES = FLAG_ACCEPT_NEAR_TIE | FLAG_SAMPLE_NEAR_TIE


def _case(seed, B, G, V, T):
    wl = inputs.SINGLE_USER.with_(name="noalloc", B=B, gamma=G, V=V, T=T, seed=seed)
    ld, lt = inputs.logits(wl)
    u_draft, u_acc, u_res = inputs.uniforms(wl)
    x = draw_tokens(ld, u_draft, T)
    return ld, lt, x, u_acc, u_res


def _both(ld, lt, x, L, u_acc, u_res, T, want_c=True):
    """The workspace call and the no-allocation call on the same device inputs; the outputs of
    the latter are prepared by the caller, so the call itself allocates nothing."""
    B, G = x.shape
    args = (pm(ld), dev(lt), dev(x), None if L is None else dev(L), dev(u_acc), dev(u_res), T)
    n0, y0, c0, f0 = D.verify(*args, want_c_star=want_c)
    n1 = torch.empty(B, dtype=torch.int32, device="cuda")
    y1 = torch.empty((B, G + 1), dtype=torch.int32, device="cuda")
    c1 = torch.empty((B, G), dtype=torch.float32, device="cuda") if want_c else None
    f1 = torch.zeros(B, dtype=torch.int32, device="cuda")
    D.verify_noalloc(*args, n_acc=n1, y_out=y1, c_star=c1, flags=f1)
    torch.cuda.synchronize()
    out0 = (host(n0), host(y0), host(c0) if want_c else None, host(f0))
    out1 = (host(n1), host(y1), host(c1) if want_c else None, host(f1))
    return out0, out1


def _agree(out0, out1):
    """Same n, y and flags except at requests either call flagged as a near-tie; c* within the
    label tolerance."""
    (n0, y0, c0, f0), (n1, y1, c1, f1) = out0, out1
    tie = ((f0 | f1) & TIES) != 0
    assert np.array_equal(n0[~tie], n1[~tie]) and np.array_equal(y0[~tie], y1[~tie])
    assert np.array_equal(f0[~tie], f1[~tie])
    if c0 is not None:
        c0, c1 = c0.astype(np.float64), c1.astype(np.float64)
        assert np.all(np.abs(c1 - c0) <= 2 * (P_RTOL * np.abs(c0) + P_ATOL))


@pytest.mark.parametrize("T", [1.0, 0.0])
def test_noalloc_matches_workspace_verify_twice_in_a_row(T):
    B, G, V = 12, 6, 30000
    L = np.array([6, 0, 3, 5, 1, 6, 2, 4, 6, 6, 0, 1], dtype=np.int32)
    for call, seed in enumerate((21, 22)):   # two calls in a row on the shared scratch
        ld, lt, x, u_acc, u_res = _case(seed, B, G, V, T)
        Lc = L if call else None
        out0, out1 = _both(ld, lt, x, Lc, u_acc, u_res, T)
        _agree(out0, out1)
        n1, y1, c1, f1 = out1
        check_verify(ld, lt, x, Lc, u_acc, u_res, T, n1, y1, flags_gpu=f1)
        check_labels(ld, lt, T, c1)


@pytest.mark.parametrize("T", [0.8, 0.0])
def test_noalloc_headline_size(T):
    # B = 64, gamma = 16, V = 151936: the workspace verify needs about 4 MB of scratch here;
    # the no-allocation call serves it from the fixed array (twice in a row)
    wl = inputs.HIGH_CONCURRENCY.with_(T=T)
    ld, lt = inputs.logits(wl)
    u_draft, u_acc, u_res = inputs.uniforms(wl)
    x = draw_tokens(ld, u_draft, T)
    for _ in range(2):
        out0, out1 = _both(ld, lt, x, None, u_acc, u_res, T)
        _agree(out0, out1)
    n1, y1, c1, f1 = out1
    reqs = range(0, wl.B, 4)   # the oracle on a quarter of the requests (they are independent)
    check_verify(ld, lt, x, None, u_acc, u_res, T, n1, y1, requests=reqs, flags_gpu=f1)
    check_labels(ld, lt, T, c1, requests=reqs)


def test_noalloc_scheduled_step_size():
    # B = 256, gamma = 5, V = 129280 with the scheduler's verify lengths
    wl = inputs.SCHEDULED_STEP
    d = inputs.full_inputs(wl)
    Lg, _, _, _ = D.prefix_schedule(dev(d["c"]), dev(d["sps"]), wl.D_max)
    Lg = host(Lg)
    x = draw_tokens(d["U"], d["u_draft"], wl.T)
    out0, out1 = _both(d["U"], d["lt"], x, Lg, d["u_acc"], d["u_res"], wl.T)
    _agree(out0, out1)
    n1, y1, c1, f1 = out1
    assert np.all(n1 <= Lg)
    reqs = range(0, wl.B, 8)
    check_verify(d["U"], d["lt"], x, Lg, d["u_acc"], d["u_res"], wl.T, n1, y1, requests=reqs, flags_gpu=f1)
    check_labels(d["U"], d["lt"], wl.T, c1, requests=reqs)


def test_noalloc_at_the_documented_edge():
    # B * (gamma + 1) = 16384 rows and B = 4096 requests: the largest sizes the array holds
    B, G, V, T = 4096, 3, 64, 1.0
    ld, lt, x, u_acc, u_res = _case(31, B, G, V, T)
    out0, out1 = _both(ld, lt, x, None, u_acc, u_res, T)
    _agree(out0, out1)
    n1, y1, c1, f1 = out1
    reqs = range(0, B, 64)
    check_verify(ld, lt, x, None, u_acc, u_res, T, n1, y1, requests=reqs, flags_gpu=f1)
    check_labels(ld, lt, T, c1, requests=reqs)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    for B, G in ((4097, 1), (2048, 8)):   # B over 4096; B*(gamma+1) over 16384
        V = 64
        ld = torch.zeros((G, B, V), device="cuda")
        lt = torch.zeros((B, G + 1, V), device="cuda")
        x = torch.zeros((B, G), dtype=torch.int32, device="cuda")
        u = torch.zeros((B, G), device="cuda")
        with pytest.raises(D.DsparkError) as e:
            D.verify_noalloc(ld, lt, x, None, u, u[:, 0].contiguous(), 1.0)
        assert e.value.status == D.EINVAL and "16384" in str(e.value)
