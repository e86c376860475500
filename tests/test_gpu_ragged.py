"""Verification over a flattened target block (Σ(L_b+1) rows plus per-request offsets and token
tags) against the oracle, against the padded call, and with inconsistent offsets."""

import numpy as np
import pytest
import torch

import oracle as O
from speculative_decoding_04_b200 import dspark as D
from speculative_decoding_04_b200 import inputs
from tests.parity import P_ATOL, P_RTOL, check_verify, dev, draw_tokens, host, pm

pytestmark = pytest.mark.gpu
IMPLS = {"stream": 0, "sliced": 1, "rows": 2}


def ragged_case(seed, B, G, V, T, L=None):
    wl = inputs.SINGLE_USER.with_(name="ragged", B=B, gamma=G, V=V, T=T, seed=seed)
    ld, lt = inputs.logits(wl)
    u_draft, u_acc, u_res = inputs.uniforms(wl)
    x = draw_tokens(ld, u_draft, T)
    if L is None:
        L = np.random.default_rng(seed).integers(0, G + 1, B).astype(np.int32)
    return ld, lt, x, np.asarray(L, dtype=np.int32), u_acc, u_res


def check_labels_ragged(ld, lt, L, T, c_gpu, requests=None):
    """c* against the oracle where the block holds the target row (positions k <= L_b); NaN
    elsewhere."""
    G = ld.shape[1]
    for b in (range(ld.shape[0]) if requests is None else requests):
        have = min(int(L[b]) + 1, G)
        assert np.isnan(c_gpu[b, have:]).all(), f"request {b}"
        o = O.tv_labels(ld[b:b + 1, :have], lt[b:b + 1, :have], T)[0]
        g = c_gpu[b, :have].astype(np.float64)
        if T == 0.0:
            assert np.array_equal(g, o)
        else:
            assert np.all(np.abs(g - o) <= P_RTOL * np.abs(o) + P_ATOL), f"request {b}"


@pytest.mark.parametrize("B", [1, 37, 1024, 3000])
def test_layout_offsets_and_tags(B):
    G = 7
    rng = np.random.default_rng(B)
    L = rng.integers(-2, G + 3, B).astype(np.int32)          # out-of-range lengths are clamped
    off, tags = D.ragged_layout(dev(L), G)
    torch.cuda.synchronize()
    assert np.array_equal(host(off), O.ragged_offsets(L, G))
    want = np.full(B * (G + 1), -1, dtype=np.int32)
    t = O.ragged_tags(L, G)
    want[:t.size] = t
    assert np.array_equal(host(tags), want)


@pytest.mark.parametrize("impl", list(IMPLS))
@pytest.mark.parametrize("T", [1.0, 0.7, 0.0])
def test_ragged_matches_oracle_and_padded_call(impl, T):
    B, G, V = 24, 6, 20000
    ld, lt, x, L, u_acc, u_res = ragged_case(40 + int(10 * T), B, G, V, T)
    L[:3] = [0, G, 1]
    packed = O.pack_ragged(lt, L)
    D.set_option("verify_impl", IMPLS[impl])
    off, _ = D.ragged_layout(dev(L), G, want_tags=False)
    n, y, c, fl = D.verify_ragged(pm(ld), dev(packed), off, dev(x), dev(L), dev(u_acc), dev(u_res), T,
                                  want_c_star=True)
    n0, y0, _, fl0 = D.verify(pm(ld), dev(lt), dev(x), dev(L), dev(u_acc), dev(u_res), T)
    torch.cuda.synchronize()
    n, y, c, fl = host(n), host(y), host(c), host(fl)
    assert not np.any(fl & D.FLAG_RAGGED_OFFSETS)
    check_verify(ld, lt, x, L, u_acc, u_res, T, n, y, flags_gpu=fl)
    check_labels_ragged(ld, lt, L, T, c)
    tie = ((fl | host(fl0)) & (D.FLAG_ACCEPT_NEAR_TIE | D.FLAG_SAMPLE_NEAR_TIE)) != 0
    assert np.array_equal(n[~tie], host(n0)[~tie]) and np.array_equal(y[~tie], host(y0)[~tie])


def test_ragged_request_major_ld():
    B, G, V, T = 10, 4, 30000, 0.9
    ld, lt, x, L, u_acc, u_res = ragged_case(77, B, G, V, T)
    off, _ = D.ragged_layout(dev(L), G, want_tags=False)
    n, y, c, fl = D.verify_ragged(dev(ld), dev(O.pack_ragged(lt, L)), off, dev(x), dev(L), dev(u_acc), dev(u_res), T,
                                  want_c_star=True, ld_layout="request")
    torch.cuda.synchronize()
    check_verify(ld, lt, x, L, u_acc, u_res, T, host(n), host(y), flags_gpu=host(fl))
    check_labels_ragged(ld, lt, L, T, host(c))


def test_scheduled_step_size():
    # B = 256, gamma = 5, V = 129280 with the scheduler's lengths: the flattened block holds
    # sum(L_b + 1) rows instead of 6 * 256
    wl = inputs.SCHEDULED_STEP
    d = inputs.full_inputs(wl)
    Lg, _, _, _ = D.prefix_schedule(dev(d["c"]), dev(d["sps"]), wl.D_max)
    L = host(Lg)
    x = draw_tokens(d["U"], d["u_draft"], wl.T)
    packed = O.pack_ragged(d["lt"], L)
    assert packed.shape[0] == int(L.sum()) + wl.B < wl.B * (wl.gamma + 1)
    off, tags = D.ragged_layout(Lg, wl.gamma)
    n, y, c, fl = D.verify_ragged(pm(d["U"]), dev(packed), off, dev(x), Lg, dev(d["u_acc"]), dev(d["u_res"]), wl.T,
                                  want_c_star=True)
    torch.cuda.synchronize()
    n, y, c, fl = host(n), host(y), host(c), host(fl)
    assert np.all(n <= L) and not np.any(fl & D.FLAG_RAGGED_OFFSETS)
    reqs = range(0, wl.B, 8)
    check_verify(d["U"], d["lt"], x, L, d["u_acc"], d["u_res"], wl.T, n, y, requests=reqs, flags_gpu=fl)
    check_labels_ragged(d["U"], d["lt"], L, wl.T, c, requests=reqs)
    t = host(tags)
    assert np.array_equal(t[:packed.shape[0]], O.ragged_tags(L, wl.gamma)) and np.all(t[packed.shape[0]:] == -1)


@pytest.mark.parametrize("impl", ["stream", "rows"])
def test_inconsistent_offsets_are_flagged_and_stay_in_bounds(impl):
    # request 2's segment is one row short (its neighbour's one row long) and the last segment
    # runs past the array; every row index is clamped into the array, the requests are flagged
    B, G, V, T = 6, 3, 8192, 1.0
    ld, lt, x, L, u_acc, u_res = ragged_case(91, B, G, V, T, L=[3, 1, 2, 0, 3, 2])
    packed = O.pack_ragged(lt, L)
    off = O.ragged_offsets(L, G)
    off[3] -= 1          # request 2 gets L_2 rows, request 3 gets L_3 + 2
    off[B] += 4          # the last request's segment ends past the array
    D.set_option("verify_impl", IMPLS[impl])
    n, y, c, fl = D.verify_ragged(pm(ld), dev(packed), dev(off), dev(x), dev(L), dev(u_acc), dev(u_res), T,
                                  want_c_star=True)
    torch.cuda.synchronize()
    fl = host(fl)
    bad = (fl & D.FLAG_RAGGED_OFFSETS) != 0
    assert bad.tolist() == [False, False, True, True, False, True]
    # the others are verified as usual
    ok = [0, 1, 4]
    check_verify(ld, lt, x, L, u_acc, u_res, T, host(n), host(y), requests=ok, flags_gpu=fl)


def test_ragged_rejects_missing_lengths():
    ld = torch.zeros((2, 3, 64), device="cuda")
    lt = torch.zeros((5, 64), device="cuda")
    off = torch.zeros(4, dtype=torch.int64, device="cuda")
    x = torch.zeros((3, 2), dtype=torch.int32, device="cuda")
    u = torch.zeros((3, 2), device="cuda")
    ws = D.workspace(D.WS_VERIFY, 3, 2, 64)
    st = D.lib.dspark_verify_ragged(D._p(ld), D._p(lt), D._p(off), 5, D._p(x), None, D._p(u), D._p(u[:, 0].contiguous()),
                                    3, 2, 64, 1.0, 0, D._p(torch.empty(3, dtype=torch.int32, device="cuda")),
                                    D._p(torch.empty((3, 3), dtype=torch.int32, device="cuda")), None,
                                    D._p(torch.zeros(3, dtype=torch.int32, device="cuda")), D._p(ws), ws.numel(), None)
    assert st == D.EINVAL and "null" in D.last_error()
