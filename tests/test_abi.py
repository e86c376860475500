"""The C-ABI library loads, exports every symbol include/dspark.h declares, and rejects bad
arguments on the host before anything is launched (no GPU needed)."""

import ctypes

import pytest
import torch

from speculative_decoding_04_b200 import build

build.build()
from speculative_decoding_04_b200 import dspark as D  # noqa: E402

# fake device addresses: only ever reach argument checks that fail before any launch
FAKE = ctypes.c_void_p(4096)
no_gpu = pytest.mark.skipif(torch.cuda.is_available(), reason="fake pointers are only passed where no GPU exists")


def test_every_declared_symbol_is_exported():
    names = D.declared_functions()
    assert {"dspark_markov_draft", "dspark_verify", "dspark_tv_labels", "dspark_prefix_schedule",
            "dspark_workspace_size", "dspark_status_string"} <= set(names)
    for n in names:
        assert hasattr(D.lib, n), n


def test_status_strings_and_options():
    assert D.status_string(D.OK) == "DSPARK_OK"
    assert D.status_string(D.EINVAL) == "DSPARK_EINVAL"
    assert D.status_string(D.ETIMEOUT) == "DSPARK_ETIMEOUT"
    assert D.status_string(99) == "DSPARK_UNKNOWN"
    with pytest.raises(D.DsparkError):
        D.set_option("no_such_option", 1)
    D.set_option("draft_pdl", 1)


def test_workspace_sizes():
    w1 = D.workspace_size(D.WS_DRAFT, 64, 16, 151936, 256)
    w2 = D.workspace_size(D.WS_DRAFT, 128, 16, 151936, 256)
    assert 256 < w1 < w2
    assert w1 >= 256 + 64 * 148 * 16            # one 16-byte record per (partition, request)
    v = D.workspace_size(D.WS_VERIFY, 64, 16, 151936, 0)
    assert v >= 256 + 64 * 17 * 32 + 64 * 17 * 149 * 12   # row records + per-1024-column tile records
    assert D.workspace_size(D.WS_SCHEDULE, 64, 16, 151936, 0) == 0
    assert D.workspace_size(7, 64, 16, 151936, 0) == 0
    assert D.workspace_size(D.WS_DRAFT, 0, 16, 151936, 256) == 0


def _draft(**kw):
    a = dict(U=FAKE, W1=FAKE, W2=FAKE, w=D.BF16, x0=FAKE, u=FAKE, B=4, G=4, V=1024, r=16, T=1.0,
             layout=D.POSITION_MAJOR, x=FAKE, ld=FAKE, flags=FAKE, ws=ctypes.c_void_p(4096 * 256), wsb=1 << 30,
             stream=None)
    a.update(kw)
    return D.lib.dspark_markov_draft(a["U"], a["W1"], a["W2"], a["w"], a["x0"], a["u"], a["B"], a["G"], a["V"],
                                     a["r"], a["T"], a["layout"], a["x"], a["ld"], a["flags"], a["ws"], a["wsb"],
                                     a["stream"])


@no_gpu
def test_draft_argument_checks():
    assert _draft(U=None) == D.EINVAL
    assert _draft(G=0) == D.EINVAL
    assert _draft(G=65) == D.EINVAL
    assert _draft(B=0) == D.EINVAL
    assert _draft(V=1) == D.EINVAL
    assert _draft(T=-1.0) == D.EINVAL
    assert _draft(T=float("inf")) == D.EINVAL
    assert _draft(T=float("nan")) == D.EINVAL
    assert _draft(w=7) == D.EINVAL
    assert _draft(wsb=100) == D.EINVAL
    assert _draft(ws=ctypes.c_void_p(4096 * 256 + 16)) == D.EINVAL
    assert _draft(layout=2) == D.EINVAL
    assert "layout" in D.last_error()
    assert _draft(u=None) == D.EINVAL           # sampling needs uniforms
    assert "gamma" in D.last_error() or "u_draft" in D.last_error()


def _verify(**kw):
    a = dict(ld=FAKE, lt=FAKE, x=FAKE, L=None, ua=FAKE, ur=FAKE, B=4, G=4, V=1024, T=1.0, layout=D.REQUEST_MAJOR,
             n=FAKE, y=FAKE, c=None, flags=FAKE, ws=ctypes.c_void_p(4096 * 256), wsb=1 << 30, stream=None)
    a.update(kw)
    return D.lib.dspark_verify(a["ld"], a["lt"], a["x"], a["L"], a["ua"], a["ur"], a["B"], a["G"], a["V"], a["T"],
                               a["layout"], a["n"], a["y"], a["c"], a["flags"], a["ws"], a["wsb"], a["stream"])


@no_gpu
def test_verify_and_labels_argument_checks():
    assert _verify(ld=None) == D.EINVAL
    assert _verify(G=65) == D.EINVAL
    assert _verify(T=-0.5) == D.EINVAL
    assert _verify(ua=None) == D.EINVAL
    assert _verify(wsb=8) == D.EINVAL
    assert _verify(layout=-1) == D.EINVAL
    assert D.lib.dspark_tv_labels(FAKE, FAKE, 2, 4, 1024, 3, 1.0, 0, FAKE, None) == D.EINVAL   # lt_rows
    assert D.lib.dspark_tv_labels(None, FAKE, 2, 4, 1024, 4, 1.0, 0, FAKE, None) == D.EINVAL
    assert D.lib.dspark_tv_labels(FAKE, FAKE, 2, 4, 1, 4, 1.0, 0, FAKE, None) == D.EINVAL
    assert D.lib.dspark_tv_labels(FAKE, FAKE, 2, 4, 1024, 4, 1.0, 3, FAKE, None) == D.EINVAL   # layout


@no_gpu
def test_schedule_argument_checks():
    s = D.lib.dspark_prefix_schedule
    assert s(FAKE, FAKE, 2, 4, 9, 0, FAKE, None, FAKE, None, None, 0, None) == D.EINVAL      # D_max > B*gamma
    assert s(FAKE, FAKE, 2, 4, -1, 0, FAKE, None, FAKE, None, None, 0, None) == D.EINVAL
    assert s(FAKE, FAKE, 2, 4, 8, 5, FAKE, None, FAKE, None, None, 0, None) == D.EINVAL      # mode
    assert s(FAKE, FAKE, 4096, 8, 8, 0, FAKE, None, FAKE, None, None, 0, None) == D.EINVAL   # > 16384 items
    assert s(None, FAKE, 2, 4, 8, 0, FAKE, None, FAKE, None, None, 0, None) == D.EINVAL


def test_binding_refuses_cpu_tensors():
    U = torch.zeros(1, 2, 8)
    W = torch.zeros(8, 2)
    with pytest.raises(ValueError):
        D.markov_draft(U, W, W.t().contiguous(), torch.zeros(1, dtype=torch.int32), None, 0.0)


@no_gpu
def test_new_entry_points_argument_checks():
    # asynchronous (t-2) scheduler: ring required and 8-byte aligned; the same limits as the
    # synchronous scheduler
    t2 = D.lib.dspark_prefix_schedule_t2
    assert t2(FAKE, FAKE, 2, 4, 8, 0, -1, None, FAKE, None, FAKE, None, None, None) == D.EINVAL
    assert t2(FAKE, FAKE, 2, 4, 8, 0, -1, ctypes.c_void_p(4100), FAKE, None, FAKE, None, None, None) == D.EINVAL
    assert "aligned" in D.last_error()
    assert t2(FAKE, FAKE, 2, 4, 9, 0, -1, FAKE, FAKE, None, FAKE, None, None, None) == D.EINVAL
    assert t2(FAKE, FAKE, 2, 4, 8, 3, -1, FAKE, FAKE, None, FAKE, None, None, None) == D.EINVAL
    # flattened verify: lengths and offsets required, at least one row
    vr = D.lib.dspark_verify_ragged
    ws = ctypes.c_void_p(4096 * 256)
    args = [FAKE, FAKE, FAKE, 10, FAKE, FAKE, FAKE, FAKE, 4, 4, 1024, 1.0, 0, FAKE, FAKE, None, FAKE, ws, 1 << 30, None]
    for i, bad in ((5, None), (2, None), (3, 0), (12, 2), (11, -1.0)):
        a = list(args)
        a[i] = bad
        assert vr(*a) == D.EINVAL, i
    assert D.lib.dspark_ragged_layout(None, 4, 4, FAKE, None, None) == D.EINVAL
    assert D.lib.dspark_ragged_layout(FAKE, 4, 65, FAKE, None, None) == D.EINVAL
    # calibration
    assert D.lib.dspark_sts_workspace_size(0, 4, 8, 15) == 0
    assert D.lib.dspark_sts_workspace_size(100, 4, 8, 15) >= 2 * 100 * 8 + 4 * 9 * 15 * 8
    fit = D.lib.dspark_sts_fit
    big = ctypes.c_void_p(4096 * 256)
    assert fit(FAKE, FAKE, 100, 4, FAKE, 8, 15, None, None, None, None, None, big, 1 << 30, None) == D.EINVAL
    assert fit(FAKE, FAKE, 100, 4, FAKE, 2000, 15, FAKE, None, None, None, None, big, 1 << 30, None) == D.EINVAL
    assert "25600" in D.last_error()
    assert fit(FAKE, FAKE, 100, 4, FAKE, 8, 15, FAKE, None, None, None, None, big, 16, None) == D.EINVAL
    assert D.lib.dspark_sts_apply(FAKE, None, 4, 4, FAKE, None) == D.EINVAL
    assert D.lib.dspark_sts_apply(FAKE, FAKE, 4, 65, FAKE, None) == D.EINVAL
    # recurrent draft head: state matrix required, rank <= 1024
    rd = D.lib.dspark_rnn_draft
    a = [FAKE, FAKE, FAKE, FAKE, D.BF16, FAKE, FAKE, 4, 4, 1024, 16, 1.0, 0, FAKE, FAKE, None, FAKE,
         ctypes.c_void_p(4096 * 256), 1 << 30, None]
    for i, bad in ((3, None), (10, 1025), (4, 7), (12, 5), (18, 64)):
        b = list(a)
        b[i] = bad
        assert rd(*b) == D.EINVAL, i
    assert D.workspace_size(D.WS_RNN_DRAFT, 4, 4, 1024, 16) == D.workspace_size(D.WS_DRAFT, 4, 4, 1024, 16) + 256
