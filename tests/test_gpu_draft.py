"""Markov-head draft on the GPU (both main-pass kernels) against the oracle."""

import numpy as np
import pytest
import torch

from speculative_decoding_04_b200 import dspark as D
from speculative_decoding_04_b200 import inputs
from tests.parity import check_draft, dev, dev_weights, host, host_rm, pm

pytestmark = pytest.mark.gpu


def run_draft(d, wl, path=0):
    D.set_option("draft_path", path)
    W1, W2 = dev_weights(d["W1"], d["W2"], wl.w_dtype)
    x, ld, fl = D.markov_draft(pm(d["U"]), W1, W2, dev(d["x0"]), dev(d["u_draft"]), wl.T)
    torch.cuda.synchronize()
    return host(x), host_rm(ld), host(fl)


def small(B, gamma, V, r, T, w_dtype="bf16", seed=77, logits="logzipf"):
    wl = inputs.SINGLE_USER.with_(name="small", B=B, gamma=gamma, V=V, r=r, T=T, w_dtype=w_dtype, seed=seed,
                                  logits=logits, w_sigma=0.05)
    return wl, inputs.full_inputs(wl)


@pytest.mark.parametrize("T", [1.0, 0.0])
def test_tiny_fp32_weights(T):
    wl = inputs.TINY.with_(T=T)
    d = inputs.full_inputs(wl)
    x, ld, fl = run_draft(d, wl)
    check_draft(d["U"], d["W1"], d["W2"], d["x0"], d["u_draft"], wl.T, x, ld, fl)
    assert (fl & ~D.FLAG_DRAFT_NEAR_TIE == 0).all()


@pytest.mark.parametrize("path", [1, 2])
@pytest.mark.parametrize("B", [1, 3, 16, 130])
@pytest.mark.parametrize("T", [1.0, 0.7, 0.0])
@pytest.mark.parametrize("r", [64, 256])
def test_bf16_paths_ragged_tail(path, B, T, r):
    # V = 4104: the last 64-column tile holds 8 columns, the last 32-column chunk 8
    wl, d = small(B, 5, 4104, r, T, seed=1000 + B + r)
    x, ld, fl = run_draft(d, wl, path)
    check_draft(d["U"], d["W1"], d["W2"], d["x0"], d["u_draft"], wl.T, x, ld, fl)
    assert x.min() >= 0 and x.max() < wl.V


@pytest.mark.parametrize("fused", [1, 0])
@pytest.mark.parametrize("B", [16, 64, 100])
@pytest.mark.parametrize("T", [1.0, 0.0])
def test_tensor_core_steps_fused_and_per_step(fused, B, T):
    # fused: all positions in one cooperative launch with grid barriers; else one launch pair
    # (main pass + combine) per position.  V = 30000: partitions of about 200 columns, a ragged
    # last tile; B = 100 takes two request groups.
    D.set_option("draft_fused", fused)
    wl, d = small(B, 6, 30000, 256, T, seed=2000 + B + fused)
    x, ld, fl = run_draft(d, wl, 2)
    check_draft(d["U"], d["W1"], d["W2"], d["x0"], d["u_draft"], wl.T, x, ld, fl)


@pytest.mark.parametrize("T", [1.0, 0.0])
def test_tensor_core_and_gemv_passes_both_match_the_oracle(T):
    # the same 24 requests through both main passes, each checked against the oracle
    wl, d = small(24, 6, 8192, 256, T, seed=5)
    for path in (1, 2):
        x, ld, fl = run_draft(d, wl, path)
        check_draft(d["U"], d["W1"], d["W2"], d["x0"], d["u_draft"], wl.T, x, ld, fl)


@pytest.mark.parametrize("w_dtype", ["f32", "bf16"])
def test_gemv_odd_vocabulary(w_dtype):
    # V odd: scalar (unvectorised) loads everywhere
    wl, d = small(3, 4, 1001, 16, 1.0, w_dtype=w_dtype, seed=9, logits="gaussian")
    x, ld, fl = run_draft(d, wl)
    check_draft(d["U"], d["W1"], d["W2"], d["x0"], d["u_draft"], wl.T, x, ld, fl)


def test_forced_markov_chain():
    # W1 = one-hot rows, W2 pushes token (i+1) mod V: the chain is x0+1, x0+2, ...
    V, r, B, G = 1024, 64, 16, 8
    W1 = np.zeros((V, r), dtype=np.float32)
    W1[np.arange(V), np.arange(V) % r] = 1.0
    W2 = np.zeros((r, V), dtype=np.float32)
    x0 = (np.arange(B) * 37 % r).astype(np.int32)          # x0 < r, so W1 row selects W2 row x0
    for i in range(r):
        W2[i, (i + 1) % r] = 64.0
    U = np.zeros((B, G, V), dtype=np.float32)
    u = np.full((B, G), 0.5, dtype=np.float32)
    for path in (1, 2):
        D.set_option("draft_path", path)
        Wd1, Wd2 = dev_weights(W1, W2, "bf16")
        x, ld, fl = D.markov_draft(pm(U), Wd1, Wd2, dev(x0), dev(u), 1.0)
        x = host(x)
        want = (x0[:, None] + 1 + np.arange(G)[None, :]) % r
        assert np.array_equal(x, want), path


def test_out_of_range_start_token_is_flagged():
    wl, d = small(2, 3, 2048, 64, 1.0, seed=3)
    d["x0"][1] = wl.V + 5
    x, ld, fl = run_draft(d, wl, 1)
    assert fl[1] & D.FLAG_TOKEN_RANGE and not fl[0] & D.FLAG_TOKEN_RANGE
    assert x.min() >= 0 and x.max() < wl.V


def test_nonfinite_logits_are_flagged():
    wl, d = small(2, 3, 2048, 64, 1.0, seed=4)
    d["U"][0, 1, 17] = np.nan
    x, ld, fl = run_draft(d, wl, 1)
    assert fl[0] & D.FLAG_NONFINITE and not fl[1] & D.FLAG_NONFINITE
    assert x.min() >= 0 and x.max() < wl.V


def test_graph_capture_replays_the_same_draft():
    wl, d = small(16, 4, 4104, 256, 1.0, seed=6)
    W1, W2 = dev_weights(d["W1"], d["W2"], "bf16")
    U, x0, u = pm(d["U"]), dev(d["x0"]), dev(d["u_draft"])
    x = torch.empty((16, 4), dtype=torch.int32, device="cuda")
    ld = torch.empty((4, 16, wl.V), dtype=torch.float32, device="cuda")
    fl = torch.zeros(16, dtype=torch.int32, device="cuda")
    ws = D.workspace(D.WS_DRAFT, 16, 4, wl.V, 256)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        D.markov_draft(U, W1, W2, x0, u, wl.T, x_out=x, ld_out=ld, flags=fl, ws=ws)
    torch.cuda.synchronize()
    ref = host(x).copy()
    x.fill_(-1)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        D.markov_draft(U, W1, W2, x0, u, wl.T, x_out=x, ld_out=ld, flags=fl, ws=ws)
    g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(host(x), ref)
