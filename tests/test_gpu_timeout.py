"""Bounded device waits.  A wait that cannot be satisfied must make the kernel return with a
timeout status -- DSPARK_ETIMEOUT in the workspace status word and DEVICE_TIMEOUT in the flags of
the requests -- and leave the CUDA context usable.  The unsatisfiable wait comes from a test-only
option (a barrier that expects one arrival more than the grid or the cluster provides) with a
short wait limit; nothing faults, traps or hangs."""

import numpy as np
import pytest
import torch

from speculative_decoding_04_b200 import dspark as D
from speculative_decoding_04_b200 import inputs
from tests.parity import check_draft, check_labels, check_verify, dev, dev_weights, draw_tokens, host, host_rm, pm

pytestmark = pytest.mark.gpu


def timed_out(fl):
    """DEVICE_TIMEOUT (bit 31) of each flags word (the words come back as int32)."""
    return (np.asarray(fl).view(np.uint32) & np.uint32(D.FLAG_DEVICE_TIMEOUT)) != 0


def _draft_inputs():
    wl = inputs.SINGLE_USER.with_(name="timeout", B=16, gamma=3, V=4096, r=64, T=1.0, seed=71, w_sigma=0.05)
    return wl, inputs.full_inputs(wl)


def test_fused_draft_grid_barrier_times_out_and_returns():
    wl, d = _draft_inputs()
    W1, W2 = dev_weights(d["W1"], d["W2"], "bf16")
    args = (pm(d["U"]), W1, W2, dev(d["x0"]), dev(d["u_draft"]), wl.T)
    ws = D.workspace(D.WS_DRAFT, wl.B, wl.gamma, wl.V, wl.r)
    D.set_option("draft_path", 2)
    D.set_option("draft_fused", 1)
    D.set_option("debug_wait_limit", 1 << 14)         # polls per wait
    D.set_option("debug_unreachable_barrier", 1)      # the first grid barrier expects one CTA more
    x, ld, fl = D.markov_draft(*args, ws=ws)
    torch.cuda.synchronize()                          # the kernel returned
    assert D.workspace_status(ws) == D.ETIMEOUT
    assert np.all(timed_out(host(fl)))
    # the context is still usable: the same call without the option completes and matches the oracle
    D.set_option("debug_unreachable_barrier", 0)
    D.set_option("debug_wait_limit", 0)
    x, ld, fl = D.markov_draft(*args, ws=ws)
    torch.cuda.synchronize()
    assert D.workspace_status(ws) == D.OK
    assert not np.any(timed_out(host(fl)))
    check_draft(d["U"], d["W1"], d["W2"], d["x0"], d["u_draft"], wl.T, host(x), host_rm(ld), host(fl))


@pytest.mark.parametrize("T", [1.0, 0.0])
def test_stream_verify_exchange_times_out_and_returns(T):
    wl = inputs.SINGLE_USER.with_(name="timeout_v", B=10, gamma=4, V=20000, T=T, seed=72)
    ld, lt = inputs.logits(wl)
    u_draft, u_acc, u_res = inputs.uniforms(wl)
    x = draw_tokens(ld, u_draft, T)
    ws = D.workspace(D.WS_VERIFY, wl.B, wl.gamma, wl.V)
    args = (pm(ld), dev(lt), dev(x), None, dev(u_acc), dev(u_res), T)
    D.set_option("verify_impl", 0)                    # the streaming kernels
    D.set_option("debug_wait_limit", 20_000_000)      # nanoseconds per wait
    D.set_option("debug_unreachable_barrier", 2)      # the cluster exchange expects one CTA more
    n, y, c, fl = D.verify(*args, want_c_star=True, ws=ws)
    torch.cuda.synchronize()
    assert D.workspace_status(ws) == D.ETIMEOUT
    assert np.all(timed_out(host(fl)))
    D.set_option("debug_unreachable_barrier", 0)
    D.set_option("debug_wait_limit", 0)
    n, y, c, fl = D.verify(*args, want_c_star=True, ws=ws)
    torch.cuda.synchronize()
    assert D.workspace_status(ws) == D.OK
    check_verify(ld, lt, x, None, u_acc, u_res, T, host(n), host(y), flags_gpu=host(fl))
    check_labels(ld, lt, T, host(c))
