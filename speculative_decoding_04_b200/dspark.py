"""Thin ctypes binding of libdspark.so (argument marshalling only).

Every function takes CUDA torch tensors, checks dtype / shape / contiguity,
passes raw device pointers and the current CUDA stream to the C ABI declared
in include/dspark.h, and raises DsparkError on a non-zero status.  All
arithmetic runs in the library's CUDA kernels; there is no CPU fallback:
importing this module raises if the library has not been built.
"""

from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Tuple

import numpy as np
import torch

from .build import LIB_PATH, ROOT

OK, EINVAL, ECUDA, ENOTIMPL, ETIMEOUT = 0, 1, 2, 3, 4
F32, BF16 = 0, 1
POSITION_MAJOR, REQUEST_MAJOR = 0, 1
_LAYOUTS = {"position": POSITION_MAJOR, "request": REQUEST_MAJOR}
SCHED_ARGMAX, SCHED_EARLY_STOP = 0, 1
WS_DRAFT, WS_VERIFY, WS_SCHEDULE, WS_RNN_DRAFT = 0, 1, 2, 3
T2_RING_BYTES = 128

FLAG_DRAFT_NEAR_TIE = 1 << 0
FLAG_ACCEPT_NEAR_TIE = 1 << 1
FLAG_SAMPLE_NEAR_TIE = 1 << 2
FLAG_SMALL_RESIDUAL = 1 << 3
FLAG_NONFINITE = 1 << 4
FLAG_TOKEN_RANGE = 1 << 5
FLAG_CONF_RANGE = 1 << 6
FLAG_SCHED_NEAR_TIE = 1 << 7
FLAG_RAGGED_OFFSETS = 1 << 8
FLAG_DEVICE_TIMEOUT = 1 << 31

HEADER = os.path.join(ROOT, "include", "dspark.h")


class DsparkError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {status_string(status)}: {msg}")
        self.status = status


_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m speculative_decoding_04_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    lib.dspark_status_string.restype = ctypes.c_char_p
    lib.dspark_status_string.argtypes = [_i]
    lib.dspark_last_error.restype = ctypes.c_char_p
    lib.dspark_last_error.argtypes = []
    lib.dspark_set_option.restype = _i
    lib.dspark_set_option.argtypes = [ctypes.c_char_p, ctypes.c_long]
    lib.dspark_workspace_size.restype = _sz
    lib.dspark_workspace_size.argtypes = [_i, _i, _i, _i, _i]
    lib.dspark_workspace_status.restype = _i
    lib.dspark_workspace_status.argtypes = [_vp, _vp]
    lib.dspark_markov_draft.restype = _i
    lib.dspark_markov_draft.argtypes = [_vp, _vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _vp, _vp, _vp, _sz,
                                        _vp]
    lib.dspark_verify.restype = _i
    lib.dspark_verify.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _f, _i, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    lib.dspark_verify_noalloc.restype = _i
    lib.dspark_verify_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _f, _i, _vp, _vp, _vp, _vp, _vp]
    lib.dspark_tv_labels.restype = _i
    lib.dspark_tv_labels.argtypes = [_vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _vp]
    lib.dspark_prefix_schedule.restype = _i
    lib.dspark_prefix_schedule.argtypes = [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    lib.dspark_rnn_draft.restype = _i
    lib.dspark_rnn_draft.argtypes = [_vp, _vp, _vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _vp, _vp, _vp, _vp,
                                     _sz, _vp]
    lib.dspark_sts_workspace_size.restype = _sz
    lib.dspark_sts_workspace_size.argtypes = [ctypes.c_int64, _i, _i, _i]
    lib.dspark_sts_fit.restype = _i
    lib.dspark_sts_fit.argtypes = [_vp, _vp, ctypes.c_int64, _i, _vp, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    lib.dspark_sts_apply.restype = _i
    lib.dspark_sts_apply.argtypes = [_vp, _vp, _i, _i, _vp, _vp]
    lib.dspark_ragged_layout.restype = _i
    lib.dspark_ragged_layout.argtypes = [_vp, _i, _i, _vp, _vp, _vp]
    lib.dspark_verify_ragged.restype = _i
    lib.dspark_verify_ragged.argtypes = [_vp, _vp, _vp, ctypes.c_int64, _vp, _vp, _vp, _vp, _i, _i, _i, _f, _i, _vp,
                                         _vp, _vp, _vp, _vp, _sz, _vp]
    lib.dspark_prefix_schedule_t2.restype = _i
    lib.dspark_prefix_schedule_t2.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
    return lib


lib = _load()


def declared_functions() -> list:
    """Names of the functions include/dspark.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dspark_\w+)\s*\(", text)))


def status_string(status: int) -> str:
    return lib.dspark_status_string(status).decode()


def last_error() -> str:
    return lib.dspark_last_error().decode()


def _check(fn: str, status: int):
    if status != OK:
        raise DsparkError(fn, status, last_error())


def set_option(key: str, value: int):
    _check("dspark_set_option", lib.dspark_set_option(key.encode(), int(value)))


def workspace_size(which: int, B: int, gamma: int, V: int, r: int = 0) -> int:
    return int(lib.dspark_workspace_size(which, B, gamma, V, r))


def workspace(which: int, B: int, gamma: int, V: int, r: int = 0, device=None) -> torch.Tensor:
    n = max(256, workspace_size(which, B, gamma, V, r))
    return torch.empty(n, dtype=torch.uint8, device=device or torch.device("cuda"))


def workspace_status(ws: torch.Tensor, stream=None) -> int:
    return int(lib.dspark_workspace_status(_p(ws), _s(stream)))


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _bgv(t: torch.Tensor, layout: str):
    """(B, gamma, V) of a logit tensor in the given layout ("position": [gamma, B, V],
    "request": [B, gamma, V])."""
    if layout not in _LAYOUTS:
        raise ValueError(f"layout must be one of {sorted(_LAYOUTS)}")
    if t.dim() != 3:
        raise ValueError("logits must be 3-D")
    a, b, V = t.shape
    return (b, a, V) if layout == "position" else (a, b, V)


def markov_draft(U: torch.Tensor, W1: torch.Tensor, W2: torch.Tensor, x0: torch.Tensor,
                 u_draft: Optional[torch.Tensor], T: float, *, layout: str = "position", x_out=None, ld_out=None,
                 flags=None, ws=None, stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Markov-head draft of gamma tokens per request.

    U is [gamma, B, V] (layout "position", the fast one) or [B, gamma, V] ("request"); returns
    (x [B, gamma], l_d in the layout of U, flags [B])."""
    B, G, V = _bgv(U, layout)
    r = W1.shape[1]
    _need(U, "U", torch.float32)
    if W1.dtype not in (torch.bfloat16, torch.float32) or W2.dtype != W1.dtype:
        raise ValueError("W1 and W2 must both be bf16 or both fp32")
    _need(W1, "W1", W1.dtype, (V, r))
    _need(W2, "W2", W1.dtype, (r, V))
    _need(x0, "x0", torch.int32, (B,))
    if u_draft is not None:
        _need(u_draft, "u_draft", torch.float32, (B, G))
    dev = U.device
    x_out = torch.empty((B, G), dtype=torch.int32, device=dev) if x_out is None else x_out
    ld_out = torch.empty(U.shape, dtype=torch.float32, device=dev) if ld_out is None else ld_out
    flags = torch.zeros(B, dtype=torch.int32, device=dev) if flags is None else flags
    ws = workspace(WS_DRAFT, B, G, V, r, dev) if ws is None else ws
    _need(x_out, "x_out", torch.int32, (B, G))
    _need(ld_out, "ld_out", torch.float32, tuple(U.shape))
    _need(flags, "flags", torch.int32, (B,))
    st = lib.dspark_markov_draft(_p(U), _p(W1), _p(W2), BF16 if W1.dtype == torch.bfloat16 else F32, _p(x0),
                                 _p(u_draft), B, G, V, r, float(T), _LAYOUTS[layout], _p(x_out), _p(ld_out),
                                 _p(flags), _p(ws),
                                 ws.numel(), _s(stream))
    _check("dspark_markov_draft", st)
    return x_out, ld_out, flags


def rnn_draft(U: torch.Tensor, W1: torch.Tensor, W2: torch.Tensor, Wh: torch.Tensor, x0: torch.Tensor,
              u_draft: Optional[torch.Tensor], T: float, *, layout: str = "position", want_h: bool = False,
              x_out=None, ld_out=None, h_out=None, flags=None, ws=None, stream=None):
    """Draft with the recurrent head; returns (x [B, gamma], l_d in the layout of U, h [B, gamma, r]
    or None, flags [B])."""
    B, G, V = _bgv(U, layout)
    r = W1.shape[1]
    _need(U, "U", torch.float32)
    if W1.dtype not in (torch.bfloat16, torch.float32) or W2.dtype != W1.dtype or Wh.dtype != W1.dtype:
        raise ValueError("W1, W2 and Wh must all be bf16 or all fp32")
    _need(W1, "W1", W1.dtype, (V, r))
    _need(W2, "W2", W1.dtype, (r, V))
    _need(Wh, "Wh", W1.dtype, (r, r))
    _need(x0, "x0", torch.int32, (B,))
    if u_draft is not None:
        _need(u_draft, "u_draft", torch.float32, (B, G))
    dev = U.device
    x_out = torch.empty((B, G), dtype=torch.int32, device=dev) if x_out is None else x_out
    ld_out = torch.empty(U.shape, dtype=torch.float32, device=dev) if ld_out is None else ld_out
    if h_out is None and want_h:
        h_out = torch.empty((B, G, r), dtype=torch.float32, device=dev)
    flags = torch.zeros(B, dtype=torch.int32, device=dev) if flags is None else flags
    ws = workspace(WS_RNN_DRAFT, B, G, V, r, dev) if ws is None else ws
    _need(x_out, "x_out", torch.int32, (B, G))
    _need(ld_out, "ld_out", torch.float32, tuple(U.shape))
    _need(flags, "flags", torch.int32, (B,))
    if h_out is not None:
        _need(h_out, "h_out", torch.float32, (B, G, r))
    wdt = BF16 if W1.dtype == torch.bfloat16 else F32
    st = lib.dspark_rnn_draft(_p(U), _p(W1), _p(W2), _p(Wh), wdt, _p(x0), _p(u_draft), B, G, V, r, float(T),
                              _LAYOUTS[layout], _p(x_out), _p(ld_out), _p(h_out), _p(flags), _p(ws), ws.numel(),
                              _s(stream))
    _check("dspark_rnn_draft", st)
    return x_out, ld_out, h_out, flags


def verify(ld: torch.Tensor, lt: torch.Tensor, x: torch.Tensor, L: Optional[torch.Tensor],
           u_acc: Optional[torch.Tensor], u_res: Optional[torch.Tensor], T: float, *, want_c_star: bool = False,
           ld_layout: str = "position", n_acc=None, y_out=None, c_star=None, flags=None, ws=None, stream=None):
    """Rejection-sampling verification of l_d ([gamma, B, V], or [B, gamma, V] with ld_layout
    "request") against l_t [B, gamma+1, V]; returns (n_acc [B], y [B, gamma+1], c_star [B, gamma]
    or None, flags [B])."""
    B, G, V = _bgv(ld, ld_layout)
    _need(ld, "ld", torch.float32)
    _need(lt, "lt", torch.float32, (B, G + 1, V))
    _need(x, "x", torch.int32, (B, G))
    if L is not None:
        _need(L, "L", torch.int32, (B,))
    if u_acc is not None:
        _need(u_acc, "u_acc", torch.float32, (B, G))
    if u_res is not None:
        _need(u_res, "u_res", torch.float32, (B,))
    dev = ld.device
    n_acc = torch.empty(B, dtype=torch.int32, device=dev) if n_acc is None else n_acc
    y_out = torch.empty((B, G + 1), dtype=torch.int32, device=dev) if y_out is None else y_out
    if c_star is None and want_c_star:
        c_star = torch.empty((B, G), dtype=torch.float32, device=dev)
    flags = torch.zeros(B, dtype=torch.int32, device=dev) if flags is None else flags
    ws = workspace(WS_VERIFY, B, G, V, 0, dev) if ws is None else ws
    _need(n_acc, "n_acc", torch.int32, (B,))
    _need(y_out, "y_out", torch.int32, (B, G + 1))
    _need(flags, "flags", torch.int32, (B,))
    if c_star is not None:
        _need(c_star, "c_star", torch.float32, (B, G))
    st = lib.dspark_verify(_p(ld), _p(lt), _p(x), _p(L), _p(u_acc), _p(u_res), B, G, V, float(T),
                           _LAYOUTS[ld_layout], _p(n_acc),
                           _p(y_out), _p(c_star), _p(flags), _p(ws), ws.numel(), _s(stream))
    _check("dspark_verify", st)
    return n_acc, y_out, c_star, flags


def sts_fit(c: torch.Tensor, n_acc: torch.Tensor, grid: torch.Tensor, n_bins: int = 15, *, want_curve: bool = False,
            ws=None, stream=None):
    """Sequential temperature scaling on a validation set (c [N, gamma] fp32, n_acc [N] int32,
    grid [J] fp64); returns dict(tau, index, ece_raw, ece_cal, curve or None) of device tensors."""
    N, G = c.shape
    _need(c, "c", torch.float32)
    _need(n_acc, "n_acc", torch.int32, (N,))
    _need(grid, "grid", torch.float64)
    J = grid.numel()
    dev = c.device
    out = {"tau": torch.empty(G, dtype=torch.float64, device=dev),
           "index": torch.empty(G, dtype=torch.int32, device=dev),
           "ece_raw": torch.empty(G, dtype=torch.float64, device=dev),
           "ece_cal": torch.empty(G, dtype=torch.float64, device=dev),
           "curve": torch.empty((G, J), dtype=torch.float64, device=dev) if want_curve else None}
    if ws is None:
        ws = torch.empty(max(1, lib.dspark_sts_workspace_size(N, G, J, n_bins)), dtype=torch.uint8, device=dev)
    st = lib.dspark_sts_fit(_p(c), _p(n_acc), N, G, _p(grid), J, int(n_bins), _p(out["tau"]), _p(out["index"]),
                            _p(out["ece_raw"]), _p(out["ece_cal"]), _p(out["curve"]), _p(ws), ws.numel(), _s(stream))
    _check("dspark_sts_fit", st)
    return out


def sts_apply(c: torch.Tensor, tau: torch.Tensor, *, c_out=None, stream=None) -> torch.Tensor:
    """Calibrated confidences fp32(sigma(logit(c) / tau[k])) of a [B, gamma] round."""
    B, G = c.shape
    _need(c, "c", torch.float32)
    _need(tau, "tau", torch.float64, (G,))
    c_out = torch.empty_like(c) if c_out is None else c_out
    _need(c_out, "c_out", torch.float32, (B, G))
    _check("dspark_sts_apply", lib.dspark_sts_apply(_p(c), _p(tau), B, G, _p(c_out), _s(stream)))
    return c_out


def ragged_layout(L: torch.Tensor, gamma: int, *, lt_off=None, tags=None, want_tags: bool = True, stream=None):
    """Row offsets [B+1] int64 (and tags [B*(gamma+1)] int32) of the flattened verify block for the
    verify lengths L [B]."""
    _need(L, "L", torch.int32)
    B = L.shape[0]
    lt_off = torch.empty(B + 1, dtype=torch.int64, device=L.device) if lt_off is None else lt_off
    if tags is None and want_tags:
        tags = torch.empty(B * (gamma + 1), dtype=torch.int32, device=L.device)
    _need(lt_off, "lt_off", torch.int64, (B + 1,))
    if tags is not None:
        _need(tags, "tags", torch.int32, (B * (gamma + 1),))
    _check("dspark_ragged_layout", lib.dspark_ragged_layout(_p(L), B, int(gamma), _p(lt_off), _p(tags), _s(stream)))
    return lt_off, tags


def verify_ragged(ld: torch.Tensor, lt: torch.Tensor, lt_off: torch.Tensor, x: torch.Tensor, L: torch.Tensor,
                  u_acc: Optional[torch.Tensor], u_res: Optional[torch.Tensor], T: float, *, want_c_star: bool = False,
                  ld_layout: str = "position", n_acc=None, y_out=None, c_star=None, flags=None, ws=None, stream=None):
    """verify() with the target logits flattened: lt [rows, V], request b's rows from lt_off[b]."""
    B, G, V = _bgv(ld, ld_layout)
    _need(ld, "ld", torch.float32)
    _need(lt, "lt", torch.float32)
    if lt.dim() != 2 or lt.shape[1] != V:
        raise ValueError("lt must be [rows, V]")
    _need(lt_off, "lt_off", torch.int64, (B + 1,))
    _need(x, "x", torch.int32, (B, G))
    _need(L, "L", torch.int32, (B,))
    if u_acc is not None:
        _need(u_acc, "u_acc", torch.float32, (B, G))
    if u_res is not None:
        _need(u_res, "u_res", torch.float32, (B,))
    dev = ld.device
    n_acc = torch.empty(B, dtype=torch.int32, device=dev) if n_acc is None else n_acc
    y_out = torch.empty((B, G + 1), dtype=torch.int32, device=dev) if y_out is None else y_out
    if c_star is None and want_c_star:
        c_star = torch.empty((B, G), dtype=torch.float32, device=dev)
    flags = torch.zeros(B, dtype=torch.int32, device=dev) if flags is None else flags
    ws = workspace(WS_VERIFY, B, G, V, 0, dev) if ws is None else ws
    _need(n_acc, "n_acc", torch.int32, (B,))
    _need(y_out, "y_out", torch.int32, (B, G + 1))
    _need(flags, "flags", torch.int32, (B,))
    if c_star is not None:
        _need(c_star, "c_star", torch.float32, (B, G))
    st = lib.dspark_verify_ragged(_p(ld), _p(lt), _p(lt_off), lt.shape[0], _p(x), _p(L), _p(u_acc), _p(u_res), B, G,
                                  V, float(T), _LAYOUTS[ld_layout], _p(n_acc), _p(y_out), _p(c_star), _p(flags),
                                  _p(ws), ws.numel(), _s(stream))
    _check("dspark_verify_ragged", st)
    return n_acc, y_out, c_star, flags


def verify_noalloc(ld: torch.Tensor, lt: torch.Tensor, x: torch.Tensor, L: Optional[torch.Tensor],
                   u_acc: Optional[torch.Tensor], u_res: Optional[torch.Tensor], T: float, *,
                   want_c_star: bool = False, ld_layout: str = "position", n_acc=None, y_out=None, c_star=None,
                   flags=None, stream=None):
    """verify() for callers that cannot provide device scratch: the library uses a fixed array of
    its own (B <= 4096, B*(gamma+1) <= 16384).  Outputs are allocated here only when not passed."""
    B, G, V = _bgv(ld, ld_layout)
    _need(ld, "ld", torch.float32)
    _need(lt, "lt", torch.float32, (B, G + 1, V))
    _need(x, "x", torch.int32, (B, G))
    if L is not None:
        _need(L, "L", torch.int32, (B,))
    dev = ld.device
    n_acc = torch.empty(B, dtype=torch.int32, device=dev) if n_acc is None else n_acc
    y_out = torch.empty((B, G + 1), dtype=torch.int32, device=dev) if y_out is None else y_out
    if c_star is None and want_c_star:
        c_star = torch.empty((B, G), dtype=torch.float32, device=dev)
    flags = torch.zeros(B, dtype=torch.int32, device=dev) if flags is None else flags
    st = lib.dspark_verify_noalloc(_p(ld), _p(lt), _p(x), _p(L), _p(u_acc), _p(u_res), B, G, V, float(T),
                                   _LAYOUTS[ld_layout], _p(n_acc),
                                   _p(y_out), _p(c_star), _p(flags), _s(stream))
    _check("dspark_verify_noalloc", st)
    return n_acc, y_out, c_star, flags


def tv_labels(ld: torch.Tensor, lt: torch.Tensor, T: float, *, ld_layout: str = "position", c_star=None,
              stream=None) -> torch.Tensor:
    """c*_k = 1 - ½‖p_d,k - p_t,k‖₁ for every drafted position; l_d is [gamma, B, V] (or
    [B, gamma, V] with ld_layout "request") and l_t [B, gamma or gamma+1, V]."""
    B, G, V = _bgv(ld, ld_layout)
    _need(ld, "ld", torch.float32)
    _need(lt, "lt", torch.float32)
    if lt.dim() != 3 or lt.shape[0] != B or lt.shape[2] != V or lt.shape[1] not in (G, G + 1):
        raise ValueError("lt must be [B, gamma or gamma+1, V]")
    c_star = torch.empty((B, G), dtype=torch.float32, device=ld.device) if c_star is None else c_star
    _need(c_star, "c_star", torch.float32, (B, G))
    _check("dspark_tv_labels", lib.dspark_tv_labels(_p(ld), _p(lt), B, G, V, lt.shape[1], float(T),
                                                    _LAYOUTS[ld_layout], _p(c_star), _s(stream)))
    return c_star


def prefix_schedule(c: torch.Tensor, sps: torch.Tensor, D_max: int, mode: int = SCHED_ARGMAX, *, L_out=None,
                    a_out=None, theta_out=None, flags=None, want_a: bool = True, stream=None):
    """Prefix survival + greedy scheduler; returns (L [B], a [B, gamma] or None, theta [1] fp64, flags [B])."""
    B, G = c.shape
    _need(c, "c", torch.float32)
    _need(sps, "sps", torch.float64)
    if sps.numel() < D_max + 1:
        raise ValueError("sps must hold D_max + 1 entries")
    dev = c.device
    L_out = torch.empty(B, dtype=torch.int32, device=dev) if L_out is None else L_out
    if a_out is None and want_a:
        a_out = torch.empty((B, G), dtype=torch.float32, device=dev)
    theta_out = torch.empty(1, dtype=torch.float64, device=dev) if theta_out is None else theta_out
    flags = torch.zeros(B, dtype=torch.int32, device=dev) if flags is None else flags
    st = lib.dspark_prefix_schedule(_p(c), _p(sps), B, G, int(D_max), int(mode), _p(L_out), _p(a_out),
                                    _p(theta_out), _p(flags), None, 0, _s(stream))
    _check("dspark_prefix_schedule", st)
    return L_out, a_out, theta_out, flags


def schedule_ring(device=None) -> torch.Tensor:
    """A zeroed ring for prefix_schedule_t2 (the start of a new sequence of steps)."""
    return torch.zeros(T2_RING_BYTES // 8, dtype=torch.int64, device=device or "cuda")


def ring_state(ring: torch.Tensor) -> dict:
    """The ring's fields, read back to the host (synchronises)."""
    raw = ring.cpu().numpy().view(np.uint8)
    return {"t": int(raw[0:8].view(np.int64)[0]), "D": raw[8:24].view(np.int32).tolist(),
            "tie": raw[24:40].view(np.uint32).tolist(), "theta": raw[40:72].view(np.float64).tolist(),
            "K": raw[72:88].view(np.int32).tolist()}


def prefix_schedule_t2(c: torch.Tensor, sps: torch.Tensor, D_max: int, ring: torch.Tensor,
                       mode: int = SCHED_ARGMAX, K_init: int = -1, *, L_out=None, a_out=None, theta_out=None,
                       K_out=None, flags=None, want_a: bool = False, stream=None):
    """Asynchronous (t-2) scheduler step on `ring`; returns (L [B], a or None, theta [1] fp64,
    K [1] int32, flags [B])."""
    B, G = c.shape
    _need(c, "c", torch.float32)
    _need(sps, "sps", torch.float64)
    if sps.numel() < D_max + 1:
        raise ValueError("sps must hold D_max + 1 entries")
    if ring.device != c.device or ring.numel() * ring.element_size() < T2_RING_BYTES or not ring.is_contiguous():
        raise ValueError("ring must be a contiguous device tensor of T2_RING_BYTES bytes")
    dev = c.device
    L_out = torch.empty(B, dtype=torch.int32, device=dev) if L_out is None else L_out
    if a_out is None and want_a:
        a_out = torch.empty((B, G), dtype=torch.float32, device=dev)
    theta_out = torch.empty(1, dtype=torch.float64, device=dev) if theta_out is None else theta_out
    K_out = torch.empty(1, dtype=torch.int32, device=dev) if K_out is None else K_out
    flags = torch.zeros(B, dtype=torch.int32, device=dev) if flags is None else flags
    st = lib.dspark_prefix_schedule_t2(_p(c), _p(sps), B, G, int(D_max), int(mode), int(K_init), _p(ring),
                                       _p(L_out), _p(a_out), _p(theta_out), _p(K_out), _p(flags), _s(stream))
    _check("dspark_prefix_schedule_t2", st)
    return L_out, a_out, theta_out, K_out, flags
