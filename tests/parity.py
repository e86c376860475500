"""Helpers that compare the CUDA path (through the C ABI) with the CPU oracle.

Tolerances (stated once, used by every GPU parity test):
  * draft logits l_d: |gpu - oracle| <= 1e-5 * max(1, |oracle|) (fp32 accumulation of bf16
    products against an fp64 sum, then one fp32 rounding);
  * probabilities and TV labels: relative 1e-5, absolute 1e-9 below 1e-9;
  * tokens, accepted lengths and schedules: exact, except where either side reports a
    near-tie (|u - F| < 1e-6, |u - p_t/p_d| < 1e-6, greedy top-2 gap <= 1e-6*max(1,|z|), or
    scheduler Θ within 1e-12 relative); there the GPU's choice must be one of the outcomes
    the oracle reports as valid, and the oracle then follows that branch.
  * flag bits (near-ties, small residual): the device computes its decisions in its own
    arithmetic, so the comparison has a margin of 4x on each side of the window: where the
    oracle's distance to a decision threshold is below a quarter of the window the bit must be
    set, and a set bit needs an oracle distance below four windows (residual mass: 0.9e-3 and
    1.1e-3 around the 1e-3 threshold).
"""

import numpy as np
import torch

import oracle as O

LD_TOL = 1e-5
P_RTOL = 1e-5
P_ATOL = 1e-9

FLAG_DRAFT_NEAR_TIE = 1 << 0
FLAG_ACCEPT_NEAR_TIE = 1 << 1
FLAG_SAMPLE_NEAR_TIE = 1 << 2
FLAG_SMALL_RESIDUAL = 1 << 3

STRICT = 0.25 * O.NEAR_TIE   # oracle distance below this: the device must flag
LOOSE = 4.0 * O.NEAR_TIE     # a device flag needs an oracle distance below this
SMALL_RES_STRICT, SMALL_RES_LOOSE = 0.9e-3, 1.1e-3


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def pm(a):
    """Host [B, gamma, V] -> device position-major [gamma, B, V] (the layout of U and l_d)."""
    return dev(np.ascontiguousarray(np.asarray(a).transpose(1, 0, 2)))


def host_rm(t):
    """Device position-major [gamma, B, V] -> host [B, gamma, V]."""
    return host(t).transpose(1, 0, 2)


def dev_weights(W1, W2, w_dtype):
    dt = torch.bfloat16 if w_dtype == "bf16" else torch.float32
    return dev(W1, dt), dev(W2, dt)


def host(t):
    return t.detach().cpu().numpy()


def cdf_distance(p, u, x):
    """Distance of u to the two ends of token x's interval of the running sum of p."""
    F = np.cumsum(np.asarray(p, dtype=np.float64))
    hi = F[x]
    lo = hi - p[x]
    return min(abs(float(u) - lo), abs(hi - float(u)))


def greedy_gap(row):
    """Top-2 gap of a logit row relative to max(1, |max|) (the greedy near-tie measure)."""
    z = np.sort(np.asarray(row, dtype=np.float32).astype(np.float64))
    return (z[-1] - z[-2]) / max(1.0, abs(z[-1]))


def _flag_agrees(bit_set, dist, what, b, strict=STRICT, loose=LOOSE):
    if dist < strict:
        assert bit_set, f"request {b}: oracle {what} distance {dist:.3e} but the device did not flag it"
    if bit_set:
        assert dist < loose, f"request {b}: device flagged {what} but the oracle distance is {dist:.3e}"


def check_draft_flags(ld_o, x_o, u_draft, T, flags_gpu, reqs):
    """DRAFT_NEAR_TIE against the oracle's distances at every drafted position."""
    for i, b in enumerate(reqs):
        d = np.inf
        for k in range(x_o.shape[1]):
            if T == 0.0:
                d = min(d, greedy_gap(ld_o[i, k]))
            else:
                d = min(d, cdf_distance(O.softmax(ld_o[i, k], T), u_draft[b, k], int(x_o[i, k])))
        _flag_agrees(bool(int(flags_gpu[b]) & FLAG_DRAFT_NEAR_TIE), d, "draft sample", b)


def check_draft(U, W1, W2, x0, u_draft, T, x_gpu, ld_gpu, flags_gpu=None, requests=None):
    """Run the oracle on the given requests, following the GPU's token wherever the oracle
    reports it as a valid outcome, and check every token and the stored draft logits (and,
    given the device flags, the draft near-tie bit).

    Returns the number of near-tie positions met.
    """
    reqs = list(range(U.shape[0])) if requests is None else list(requests)
    follow = {(i, k): int(x_gpu[b, k]) for i, b in enumerate(reqs) for k in range(U.shape[1])}
    x_o, ld_o, alts = O.markov_draft(U[reqs], W1, W2, x0[reqs], u_draft[reqs], T, follow=follow)
    assert np.array_equal(x_o, x_gpu[reqs])
    ld_g = ld_gpu[reqs].astype(np.float64)
    ref = ld_o.astype(np.float64)
    err = np.abs(ld_g - ref) / np.maximum(1.0, np.abs(ref))
    assert err.max() <= LD_TOL, f"l_d max scaled error {err.max():.3e}"
    if flags_gpu is not None:
        check_draft_flags(ld_o, x_o, u_draft, T, flags_gpu, reqs)
    return len(alts)


def verify_outcome(ld_b, lt_b, x_b, Lb, u_acc_b, u_res_b, T, n_gpu, y_gpu):
    """Oracle outcome for one request that agrees with the GPU wherever a near-tie allows it.

    Raises AssertionError if the GPU's (n, y) is not a valid outcome.
    """
    force = {}
    for _ in range(len(x_b) + 2):
        r = O.verify_request(ld_b, lt_b, x_b, Lb, u_acc_b, u_res_b, T, force_accept=force)
        if r["n"] != n_gpu:
            k = min(r["n"], n_gpu)
            assert k in r["accept_ties"], f"accept decision at position {k} differs and is not a near-tie"
            force[k] = n_gpu > k
            continue
        tok = int(y_gpu[n_gpu])
        if tok != int(r["y"][n_gpu]):
            assert tok in r["sample_alts"], f"token {tok} not among the valid outcomes {r['sample_alts']}"
            r = O.verify_request(ld_b, lt_b, x_b, Lb, u_acc_b, u_res_b, T, force_accept=force, force_token=tok)
        assert np.array_equal(r["y"], y_gpu), f"y differs: oracle {r['y']} gpu {y_gpu}"
        return r
    raise AssertionError("could not align the oracle with the GPU outcome")


def check_verify_flags(ld_b, lt_b, x_b, Lb, u_acc_b, u_res_b, T, r, flags_b, b):
    """ACCEPT_NEAR_TIE, SAMPLE_NEAR_TIE and SMALL_RESIDUAL of one request against the oracle's
    outcome r (already aligned with the device's n and y)."""
    n = r["n"]
    fl = int(flags_b)
    # acceptance decisions taken: positions 0..n (the first rejection included), below L
    d_acc = np.inf
    for k in range(min(n + 1, Lb)):
        if T == 0.0:
            d_acc = min(d_acc, greedy_gap(lt_b[k]))
        elif 0 <= int(x_b[k]) < ld_b.shape[-1]:
            pd = O.softmax(ld_b[k], T)[int(x_b[k])]
            pt = O.softmax(lt_b[k], T)[int(x_b[k])]
            if pd > 0:
                d_acc = min(d_acc, abs(float(u_acc_b[k]) - pt / pd))
    _flag_agrees(bool(fl & FLAG_ACCEPT_NEAR_TIE), d_acc, "acceptance", b)
    # the residual or bonus sample
    tok = int(r["y"][n])
    if T == 0.0:
        d_smp = greedy_gap(lt_b[n])
    else:
        pt = O.softmax(lt_b[n], T)
        p = pt
        if n < Lb:
            q = np.maximum(0.0, pt - O.softmax(ld_b[n], T))
            if q.sum() > 0:
                p = q / q.sum()
        d_smp = cdf_distance(p, u_res_b, tok)
    _flag_agrees(bool(fl & FLAG_SAMPLE_NEAR_TIE), d_smp, "residual/bonus sample", b)
    z = r["residual_mass"] if (T > 0 and n < Lb) else np.inf
    _flag_agrees(bool(fl & FLAG_SMALL_RESIDUAL), z, "residual mass", b, SMALL_RES_STRICT, SMALL_RES_LOOSE)


def check_verify(ld, lt, x, L, u_acc, u_res, T, n_gpu, y_gpu, requests=None, flags_gpu=None):
    """Check n and y of every given request against the oracle (and, given the device flags,
    the verification's flag bits).  Returns the number of requests with a near-tie."""
    reqs = list(range(ld.shape[0])) if requests is None else list(requests)
    G = ld.shape[1]
    ties = 0
    for b in reqs:
        Lb = G if L is None else int(L[b])
        r = verify_outcome(ld[b], lt[b], x[b], Lb, u_acc[b], u_res[b], T, int(n_gpu[b]), y_gpu[b])
        if flags_gpu is not None:
            check_verify_flags(ld[b], lt[b], x[b], Lb, u_acc[b], u_res[b], T, r, flags_gpu[b], b)
        ties += bool(r["accept_ties"]) or len(r["sample_alts"]) > 1
    return ties


def check_labels(ld, lt, T, c_gpu, requests=None):
    reqs = list(range(ld.shape[0])) if requests is None else list(requests)
    G = ld.shape[1]
    c_o = O.tv_labels(ld[reqs], lt[reqs][:, :G], T)
    c_g = c_gpu[reqs].astype(np.float64)
    if T == 0.0:
        assert np.array_equal(c_g, c_o)
        return
    bad = np.abs(c_g - c_o) > P_RTOL * np.abs(c_o) + P_ATOL
    assert not bad.any(), f"c* mismatch at {np.argwhere(bad)[:5]}: gpu {c_g[bad][:5]} oracle {c_o[bad][:5]}"


def draw_tokens(ld, u, T):
    """Draft tokens drawn by the oracle's own sampler from given draft logits (verify inputs)."""
    B, G, V = ld.shape
    x = np.zeros((B, G), dtype=np.int32)
    for b in range(B):
        for k in range(G):
            x[b, k] = O.greedy_choice(ld[b, k])[0] if T == 0.0 else O.inverse_cdf(O.softmax(ld[b, k], T), u[b, k])[0]
    return x
