"""Near-tie and small-residual flag bits of the CUDA path against the oracle, on inputs built so
that each condition holds (or clearly does not) for chosen requests.

The flags are part of the output contract: tokens and accepted lengths are compared exactly
except at flagged near-ties, so a device that failed to raise a bit where the oracle finds the
condition would hide a disagreement.  Each case checks (a) the requests built to be near a
threshold carry the bit and the others do not, and (b) the two-sided comparison of
tests/parity.py (device bit set <=> oracle distance inside the window, with a 4x margin).
"""

import numpy as np
import pytest
import torch

import oracle as O
from speculative_decoding_04_b200 import dspark as D
from tests.parity import check_draft, check_verify, dev, dev_weights, host, host_rm, pm

pytestmark = pytest.mark.gpu

VERIFY_IMPLS = ["sliced", "stream", "rows", "noalloc"]


def run_verify(impl, ld, lt, x, L, u_acc, u_res, T):
    D.set_option("verify_impl", {"stream": 0, "sliced": 1, "rows": 2, "noalloc": 0}[impl])
    args = (pm(ld), dev(lt), dev(x), None if L is None else dev(L), dev(u_acc), dev(u_res), T)
    if impl == "noalloc":
        n, y, c, fl = D.verify_noalloc(*args, want_c_star=True)
    else:
        n, y, c, fl = D.verify(*args, want_c_star=True)
    torch.cuda.synchronize()
    return host(n), host(y), host(fl)


# --------------------------------------------------------------------------- draft

@pytest.mark.parametrize("path", [1, 2])
def test_draft_near_tie_on_cdf_boundaries(path):
    # uniform logits (U = 0, W2 = 0): F_v = (v+1)/V exactly for V = 4096; even requests draw
    # u on a boundary, odd ones in the middle of an interval
    B, G, V, r = 12, 2, 4096, 64
    rng = np.random.default_rng(1)
    U = np.zeros((B, G, V), dtype=np.float32)
    W1 = rng.normal(0, 0.02, (V, r)).astype(np.float32)
    W2 = np.zeros((r, V), dtype=np.float32)
    x0 = rng.integers(0, V, B).astype(np.int32)
    j = rng.integers(1, V, (B, G))
    u = ((j + np.where(np.arange(B) % 2 == 0, 0.0, 0.5)[:, None]) / V).astype(np.float32)
    D.set_option("draft_path", path)
    Wd1, Wd2 = dev_weights(W1, W2, "bf16")
    x, ld, fl = D.markov_draft(pm(U), Wd1, Wd2, dev(x0), dev(u), 1.0)
    torch.cuda.synchronize()
    x, ld, fl = host(x), host_rm(ld), host(fl)
    tie = (fl & D.FLAG_DRAFT_NEAR_TIE) != 0
    assert tie[0::2].all() and not tie[1::2].any()
    check_draft(U, W1, W2.astype(np.float32), x0, u, 1.0, x, ld, fl)


@pytest.mark.parametrize("path", [1, 2])
def test_draft_greedy_top2_gap(path):
    B, G, V, r = 10, 2, 4096, 64
    rng = np.random.default_rng(2)
    U = rng.normal(0, 1, (B, G, V)).astype(np.float32)
    for b in range(B):
        for k in range(G):
            U[b, k, 100 + b] = 8.0
            U[b, k, 3000 - b] = 8.0 if b % 2 == 0 else 7.99     # exact tie / clear gap
    W1 = rng.normal(0, 0.02, (V, r)).astype(np.float32)
    W2 = np.zeros((r, V), dtype=np.float32)
    x0 = rng.integers(0, V, B).astype(np.int32)
    D.set_option("draft_path", path)
    Wd1, Wd2 = dev_weights(W1, W2, "bf16")
    x, ld, fl = D.markov_draft(pm(U), Wd1, Wd2, dev(x0), None, 0.0)
    torch.cuda.synchronize()
    x, ld, fl = host(x), host_rm(ld), host(fl)
    tie = (fl & D.FLAG_DRAFT_NEAR_TIE) != 0
    assert tie[0::2].all() and not tie[1::2].any()
    assert np.array_equal(x[:, 0], 100 + np.arange(B))          # lowest index wins the tie
    check_draft(U, W1, W2, x0, np.zeros((B, G), np.float32), 0.0, x, ld, fl)


# --------------------------------------------------------------------------- verify

def _rows(B, G, V, sigma, seed):
    rng = np.random.default_rng(seed)
    ld = rng.normal(0, 1.5, (B, G, V)).astype(np.float32)
    lt = np.concatenate([ld + rng.normal(0, sigma, (B, G, V)).astype(np.float32),
                         rng.normal(0, 1.5, (B, 1, V)).astype(np.float32)], axis=1)
    return ld, lt


@pytest.mark.parametrize("impl", VERIFY_IMPLS)
def test_acceptance_near_tie(impl):
    # one verified position: x where p_t < p_d, u = fl32(p_t/p_d) (near) or p_t/p_d - 1e-4 (clear)
    B, G, V = 8, 1, 4096
    ld, lt = _rows(B, G, V, 0.5, 3)
    x = np.zeros((B, G), dtype=np.int32)
    u = np.zeros((B, G), dtype=np.float32)
    for b in range(B):
        pd, pt = O.softmax(ld[b, 0], 1.0), O.softmax(lt[b, 0], 1.0)
        x[b, 0] = int(np.argmax(pd - pt))
        ratio = pt[x[b, 0]] / pd[x[b, 0]]
        u[b, 0] = np.float32(ratio) if b % 2 == 0 else np.float32(ratio - 1e-4)
    u_res = np.full(B, 0.37, dtype=np.float32)
    n, y, fl = run_verify(impl, ld, lt, x, None, u, u_res, 1.0)
    tie = (fl & D.FLAG_ACCEPT_NEAR_TIE) != 0
    assert tie[0::2].all() and not tie[1::2].any()
    assert np.all(n[1::2] == 1)                                  # u clearly below the ratio
    check_verify(ld, lt, x, None, u, u_res, 1.0, n, y, flags_gpu=fl)


@pytest.mark.parametrize("impl", VERIFY_IMPLS)
def test_bonus_sample_near_tie(impl):
    # everything accepted (u = 0), bonus row uniform over V = 4096: u_res on a boundary or not
    B, G, V = 8, 2, 4096
    ld, lt = _rows(B, G, V, 0.3, 4)
    lt[:, G] = 0.0
    x = np.argmax(ld, axis=2).astype(np.int32)
    u = np.zeros((B, G), dtype=np.float32)
    j = np.random.default_rng(5).integers(1, V, B)
    u_res = ((j + np.where(np.arange(B) % 2 == 0, 0.0, 0.5)) / V).astype(np.float32)
    n, y, fl = run_verify(impl, ld, lt, x, None, u, u_res, 1.0)
    assert np.all(n == G)
    tie = (fl & D.FLAG_SAMPLE_NEAR_TIE) != 0
    assert tie[0::2].all() and not tie[1::2].any()
    check_verify(ld, lt, x, None, u, u_res, 1.0, n, y, flags_gpu=fl)


@pytest.mark.parametrize("impl", VERIFY_IMPLS)
def test_residual_sample_near_tie(impl):
    # p_d one-hot on token 0, p_t uniform over tokens 4..V-1 (and 0 at token 0): certain
    # rejection at position 0 and a uniform residual over 4092 tokens
    B, G, V = 6, 1, 4096
    ld = np.full((B, G, V), -1e4, dtype=np.float32)
    ld[:, :, 0] = 0.0
    lt = np.zeros((B, G + 1, V), dtype=np.float32)
    lt[:, 0, :4] = -1e4
    x = np.zeros((B, G), dtype=np.int32)
    u = np.full((B, G), 0.5, dtype=np.float32)
    j = np.random.default_rng(6).integers(1, V - 4, B)
    u_res = ((j + np.where(np.arange(B) % 2 == 0, 0.0, 0.5)) / (V - 4)).astype(np.float32)
    n, y, fl = run_verify(impl, ld, lt, x, None, u, u_res, 1.0)
    assert np.all(n == 0)
    tie = (fl & D.FLAG_SAMPLE_NEAR_TIE) != 0
    assert tie[0::2].all() and not tie[1::2].any()
    assert not np.any(fl & D.FLAG_SMALL_RESIDUAL)
    check_verify(ld, lt, x, None, u, u_res, 1.0, n, y, flags_gpu=fl)


@pytest.mark.parametrize("impl", VERIFY_IMPLS)
def test_small_residual(impl):
    # rejection at position 0 in every request; even requests have a target within 1e-4 of the
    # draft (residual mass far below 1e-3), odd ones a clearly different target
    B, G, V = 8, 1, 4096
    ld, _ = _rows(B, G, V, 0.0, 7)
    rng = np.random.default_rng(8)
    lt = np.empty((B, G + 1, V), dtype=np.float32)
    for b in range(B):
        s = 1e-4 if b % 2 == 0 else 1.0
        lt[b, 0] = ld[b, 0] + rng.normal(0, s, V).astype(np.float32)
        lt[b, 1] = rng.normal(0, 1.5, V).astype(np.float32)
    x = np.zeros((B, G), dtype=np.int32)
    for b in range(B):
        pd, pt = O.softmax(ld[b, 0], 1.0), O.softmax(lt[b, 0], 1.0)
        x[b, 0] = int(np.argmax((pd - pt) / pd))                   # smallest ratio p_t/p_d
    u = np.full((B, G), np.nextafter(np.float32(1), np.float32(0)), dtype=np.float32)
    u_res = np.full(B, 0.41, dtype=np.float32)
    n, y, fl = run_verify(impl, ld, lt, x, None, u, u_res, 1.0)
    assert np.all(n == 0)
    small = (fl & D.FLAG_SMALL_RESIDUAL) != 0
    assert small[0::2].all() and not small[1::2].any()
    check_verify(ld, lt, x, None, u, u_res, 1.0, n, y, requests=range(1, B, 2), flags_gpu=fl)
    # a flagged residual is ill-conditioned in fp32 (q = p_t - p_d cancels to a few digits), so
    # its token is only required to carry positive residual mass in the oracle
    for b in range(0, B, 2):
        q = np.maximum(0.0, O.softmax(lt[b, 0], 1.0) - O.softmax(ld[b, 0], 1.0))
        assert q[int(y[b, 0])] > 0 and q.sum() < 1e-3


@pytest.mark.parametrize("impl", VERIFY_IMPLS)
def test_greedy_target_ties(impl):
    # T = 0: even requests have an exact top-2 tie in the target rows (acceptance and bonus)
    B, G, V = 6, 2, 4096
    ld, lt = _rows(B, G, V, 0.3, 9)
    for b in range(B):
        for k in range(G + 1):
            lt[b, k, 50 + b] = 9.0
            lt[b, k, 2000 + b] = 9.0 if b % 2 == 0 else 8.9
    x = np.tile((50 + np.arange(B))[:, None], (1, G)).astype(np.int32)   # the argmax: all accepted
    u = np.zeros((B, G), dtype=np.float32)
    n, y, fl = run_verify(impl, ld, lt, x, None, u, np.zeros(B, np.float32), 0.0)
    assert np.all(n == G) and np.array_equal(y[:, G], 50 + np.arange(B))
    for bit in (D.FLAG_ACCEPT_NEAR_TIE, D.FLAG_SAMPLE_NEAR_TIE):
        tie = (fl & bit) != 0
        assert tie[0::2].all() and not tie[1::2].any()
    check_verify(ld, lt, x, None, u, np.zeros(B, np.float32), 0.0, n, y, flags_gpu=fl)
