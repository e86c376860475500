"""Asynchronous (t-2) scheduling on the GPU against the oracle: the ring carries each step's
global-search result two steps forward, and one captured CUDA graph of the whole round (draft,
schedule, verify) replays step after step with no host synchronisation in between."""

import numpy as np
import pytest
import torch

import oracle as O
from speculative_decoding_04_b200 import dspark as D
from speculative_decoding_04_b200 import inputs
from tests.parity import check_draft, check_verify, dev, dev_weights, host, host_rm, pm

pytestmark = pytest.mark.gpu


def run_steps(cs, sps, D_max, mode=O.SCHED_ARGMAX, K_init=-1):
    """One prefix_schedule_t2 call per step on a fresh ring; returns per-step host results."""
    ring = D.schedule_ring()
    sps_d = dev(np.asarray(sps, dtype=np.float64))
    Dm = [D_max] * len(cs) if np.isscalar(D_max) else D_max
    out = []
    for c, dm in zip(cs, Dm):
        L, _, th, K, fl = D.prefix_schedule_t2(dev(c), sps_d, dm, ring, mode, K_init)
        out.append((L, th, K, fl))
    torch.cuda.synchronize()
    res = [dict(L=host(L), theta=float(host(th)[0]), K=int(host(K)[0]), fl=host(fl)) for L, th, K, fl in out]
    return res, D.ring_state(ring)


def check_steps(cs, sps, D_max, mode=O.SCHED_ARGMAX, K_init=-1):
    got, ring = run_steps(cs, sps, D_max, mode, K_init)
    ref = O.prefix_schedule_t2(cs, sps, D_max, mode, None if K_init < 0 else K_init)
    lo = O.prefix_schedule_t2(cs, sps, D_max, mode, None if K_init < 0 else K_init, near=0.25 * O.THETA_NEAR_TIE)
    hi = O.prefix_schedule_t2(cs, sps, D_max, mode, None if K_init < 0 else K_init, near=4 * O.THETA_NEAR_TIE)
    for t, (g, r) in enumerate(zip(got, ref)):
        flagged = bool(g["fl"][0] & D.FLAG_SCHED_NEAR_TIE)
        assert np.all(((g["fl"] & D.FLAG_SCHED_NEAR_TIE) != 0) == flagged)
        if lo[t]["near_tie"]:
            assert flagged, f"step {t}: the decision of step {t - 2} is a near-tie the device did not flag"
        if flagged:
            assert hi[t]["near_tie"]
        if not (flagged or r["near_tie"]):
            assert g["K"] == r["K"], f"step {t}"
            assert np.array_equal(g["L"], r["L"]), f"step {t}"
            assert g["theta"] == pytest.approx(r["theta"], rel=1e-12)
        assert g["L"].sum() == g["K"]
    assert ring["t"] == len(cs)
    # the ring holds the search results (and applied capacities) of the last four steps
    for t in range(max(0, len(cs) - 4), len(cs)):
        if not ref[t]["decision_tie"]:
            assert ring["D"][t % 4] == ref[t]["D"]
        assert ring["K"][t % 4] == got[t]["K"]
    return got, ref


def test_hand_example():
    # the closed-form sequence of the oracle's pin: capacities 12, 12, 5, 3, 6, 0
    ms = [[4, 0, 1], [1, 1, 1], [2, 2, 2], [0, 0, 0], [4, 4, 4], [1, 0, 3]]
    cs = [np.array([[1.0 if j < m else 0.0 for j in range(4)] for m in mb], dtype=np.float32) for mb in ms]
    got, _ = run_steps(cs, np.ones(13), 12, K_init=12)
    assert [g["K"] for g in got] == [12, 12, 5, 3, 6, 0]
    assert [g["L"].tolist() for g in got] == [[4, 4, 4], [4, 4, 4], [2, 2, 1], [3, 0, 0], [4, 2, 0], [0, 0, 0]]
    assert [g["theta"] for g in got] == [8.0, 6.0, 8.0, 3.0, 9.0, 3.0]


@pytest.mark.parametrize("mode", [O.SCHED_ARGMAX, O.SCHED_EARLY_STOP])
@pytest.mark.parametrize("seed", range(4))
def test_random_sequences(mode, seed):
    rng = np.random.default_rng(700 + seed)
    B, G = 48, 6
    sps = 1.0 / (0.004 + 0.00003 * (B + np.arange(B * G + 1)))
    cs = [rng.beta(rng.uniform(2, 8), 2, size=(B, G)).astype(np.float32) for _ in range(7)]
    check_steps(cs, sps, B * G, mode)
    check_steps(cs, sps, B * G // 2, mode, K_init=17)


def test_scheduled_step_size_with_changing_batch():
    # B = 256, gamma = 5 with the affine-latency table; the batch shrinks and grows between
    # steps (continuous batching), so a capacity from a larger step is clamped
    wl = inputs.SCHEDULED_STEP
    sps = inputs.sps_table(wl)
    Bs = [256, 256, 200, 120, 256, 64, 256]
    cs = [inputs.confidences(wl.with_(B=b, seed=800 + i)) for i, b in enumerate(Bs)]
    check_steps(cs, sps, [b * wl.gamma for b in Bs])


def test_ring_rejects_misuse():
    c = torch.zeros((4, 3), device="cuda")
    sps = torch.ones(14, dtype=torch.float64, device="cuda")
    ring = D.schedule_ring()
    with pytest.raises(D.DsparkError) as e:
        D.prefix_schedule_t2(c, sps, 13, ring)                     # D_max above B * gamma
    assert e.value.status == D.EINVAL
    # a ring 4 bytes off an 8-byte boundary is refused before anything is launched
    L = torch.empty(4, dtype=torch.int32, device="cuda")
    th = torch.empty(1, dtype=torch.float64, device="cuda")
    raw = torch.zeros(40, dtype=torch.int32, device="cuda")
    st = D.lib.dspark_prefix_schedule_t2(D._p(c), D._p(sps), 4, 3, 12, 0, -1, raw.data_ptr() + 4, D._p(L), None,
                                         D._p(th), None, None, None)
    assert st == D.EINVAL and "aligned" in D.last_error()
    assert D.ring_state(ring)["t"] == 0


# --------------------------------------------------------------------------- the round in one CUDA graph

def test_graph_replayed_round_uses_t2_schedules():
    B, G, V, r, T, S = 32, 5, 8200, 64, 1.0, 5
    base = inputs.SCHEDULED_STEP.with_(name="t2_graph", B=B, gamma=G, V=V, r=r, T=T)
    sps_h = inputs.sps_table(base)
    d0 = inputs.full_inputs(base.with_(seed=900))
    W1, W2 = dev_weights(d0["W1"], d0["W2"], "bf16")
    steps_h = [inputs.full_inputs(base.with_(seed=901 + t)) for t in range(S)]
    keys = ("U", "lt", "x0", "u_draft", "u_acc", "u_res", "c")
    steps_d = [{k: (pm(h[k]) if k == "U" else dev(h[k])) for k in keys} for h in steps_h]
    st = {k: torch.empty_like(v) for k, v in steps_d[0].items()}         # the graph's input buffers
    sps = dev(sps_h)
    x = torch.empty((B, G), dtype=torch.int32, device="cuda")
    ld = torch.empty((G, B, V), dtype=torch.float32, device="cuda")
    L = torch.empty(B, dtype=torch.int32, device="cuda")
    th = torch.empty(1, dtype=torch.float64, device="cuda")
    K = torch.empty(1, dtype=torch.int32, device="cuda")
    n = torch.empty(B, dtype=torch.int32, device="cuda")
    y = torch.empty((B, G + 1), dtype=torch.int32, device="cuda")
    fl = torch.zeros(B, dtype=torch.int32, device="cuda")
    ws_d = D.workspace(D.WS_DRAFT, B, G, V, r)
    ws_v = D.workspace(D.WS_VERIFY, B, G, V)
    ring = D.schedule_ring()

    def round_():
        fl.zero_()
        D.markov_draft(st["U"], W1, W2, st["x0"], st["u_draft"], T, x_out=x, ld_out=ld, flags=fl, ws=ws_d)
        D.prefix_schedule_t2(st["c"], sps, B * G, ring, L_out=L, theta_out=th, K_out=K, flags=fl)
        D.verify(ld, st["lt"], x, L, st["u_acc"], st["u_res"], T, n_acc=n, y_out=y, flags=fl, ws=ws_v)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for k in st:
            st[k].copy_(steps_d[0][k])
        round_()                    # eager warm-up (function attributes, tensor maps) on the ring
        ring.zero_()                # then a new sequence of steps starts
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        round_()
    hist = {k: [] for k in ("x", "ld", "L", "K", "n", "y", "fl")}
    with torch.cuda.stream(s):
        for t in range(S):          # no host synchronisation between steps
            for k in st:
                st[k].copy_(steps_d[t][k], non_blocking=True)
            g.replay()
            for k, v in (("x", x), ("ld", ld), ("L", L), ("K", K), ("n", n), ("y", y), ("fl", fl)):
                hist[k].append(v.clone())
    s.synchronize()
    assert D.ring_state(ring)["t"] == S

    ref = O.prefix_schedule_t2([h["c"] for h in steps_h], sps_h, B * G)
    assert ref[2]["K"] != ref[3]["K"] or ref[3]["K"] != ref[4]["K"], "inputs should move the capacity"
    for t, h in enumerate(steps_h):
        fl_t = host(hist["fl"][t])
        x_t, ld_t, L_t = host(hist["x"][t]), host_rm(hist["ld"][t]), host(hist["L"][t])
        check_draft(h["U"], d0["W1"], d0["W2"], h["x0"], h["u_draft"], T, x_t, ld_t, fl_t)
        if not (fl_t[0] & D.FLAG_SCHED_NEAR_TIE or ref[t]["near_tie"]):
            assert int(host(hist["K"][t])[0]) == ref[t]["K"], f"step {t}"
            assert np.array_equal(L_t, ref[t]["L"]), f"step {t}"
        check_verify(ld_t, h["lt"], x_t, L_t, h["u_acc"], h["u_res"], T, host(hist["n"][t]), host(hist["y"][t]),
                     flags_gpu=fl_t)
