"""Seeded synthetic workloads for the draft/verify round.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no softmax, no bias contraction, no sampling, no
scheduling).  It is the one module that both the CUDA path's callers (tests,
bench) and the oracle's callers use, so that both sides see identical inputs.

The workloads follow the five cases the round is specified on (tiny, single
user, high concurrency, scheduled serving step, vocabulary sweep).  The pages
measure on model-generated logits over public math/code/chat suites; those
models and suites are not available, so logits are synthesised with the
shapes and value structure stated below:

* Gaussian logits (tiny case): U_ext ~ N(0, 2) of shape [B, gamma+1, V],
  target = U_ext + N(0, 0.5).
* log-Zipf logits (all other cases): a seeded permutation pi of the
  vocabulary gives each token a rank in 1..V shared by every row, the prior is
  -s*ln(rank) with s = 1.1, U_ext = prior + N(0, 1.5) and the target rows are
  U_ext + N(0, sigma_k).  sigma_k is constant or grows linearly with the block
  position (suffix decay), with its own value for the bonus row.
* U = U_ext[:, :gamma] are the draft base logits; the target has gamma+1 rows
  (one per drafted position plus the bonus position).
* W1 [V, r] and W2 [r, V] ~ N(0, sigma_w), stored as fp32 or rounded to bf16
  (round to nearest even).
* x0 ~ U{0..V-1}; every uniform (draft, acceptance, residual) ~ U[0, 1) fp32.
* confidences c ~ Beta(a, b) per (request, position), optionally decayed by
  a geometric factor per position.
* steps/s tables indexed by D, the number of scheduled draft tokens.
* calibration sets: true pass probabilities q ~ Beta(a, b), accepted counts drawn from them,
  and over-confident raw confidences c = 1 - (1 - q)^s (s between 1.1 and 1.3 along the block).

Every tensor is drawn from its own Philox stream keyed by
(workload seed, tensor id[, request]); logits are keyed per request so that a
single request can be regenerated on its own.
"""

from __future__ import annotations

import dataclasses
from typing import Optional, Tuple

import numpy as np

# tensor ids for the Philox key
_T_UEXT, _T_TNOISE, _T_W1, _T_W2, _T_X0, _T_UDRAFT, _T_UACC, _T_URES, _T_CONF, _T_PERM, _T_CALIB = range(1, 12)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    gamma: int
    V: int
    r: int
    T: float
    w_dtype: str            # "bf16" or "f32"
    w_sigma: float
    logits: str             # "gaussian" or "logzipf"
    u_sigma: float          # noise of the draft base logits
    t_sigma_first: float    # target noise at block position 1
    t_sigma_last: float     # target noise at block position gamma (linear in between)
    t_sigma_bonus: float    # target noise of the bonus row
    conf_a: float
    conf_b: float
    conf_decay: float       # c_{b,k} *= conf_decay**(k-1)
    sps: str                # "linear" or "affine_latency"
    seed: int
    zipf_s: float = 1.1

    @property
    def D_max(self) -> int:
        return self.B * self.gamma

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _lz(name, B, gamma, V, T, seed, t_first=0.7, t_last=0.7, t_bonus=0.7,
        conf=(6.0, 2.0), decay=1.0, sps="affine_latency"):
    return Workload(name=name, B=B, gamma=gamma, V=V, r=256, T=T, w_dtype="bf16", w_sigma=0.02,
                    logits="logzipf", u_sigma=1.5, t_sigma_first=t_first, t_sigma_last=t_last,
                    t_sigma_bonus=t_bonus, conf_a=conf[0], conf_b=conf[1], conf_decay=decay,
                    sps=sps, seed=seed)


TINY = Workload(name="tiny", B=2, gamma=4, V=1024, r=16, T=1.0, w_dtype="f32", w_sigma=0.1,
                logits="gaussian", u_sigma=2.0, t_sigma_first=0.5, t_sigma_last=0.5,
                t_sigma_bonus=0.5, conf_a=8.0, conf_b=2.0, conf_decay=1.0, sps="linear", seed=0)
SINGLE_USER = _lz("single_user", B=1, gamma=7, V=151936, T=1.0, seed=2)
SINGLE_USER_GREEDY = SINGLE_USER.with_(name="single_user_greedy", T=0.0)
HIGH_CONCURRENCY = _lz("high_concurrency", B=64, gamma=16, V=151936, T=0.8, seed=3,
                       t_first=0.3, t_last=1.2, t_bonus=1.2)
SCHEDULED_STEP = _lz("scheduled_step", B=256, gamma=5, V=129280, T=1.0, seed=4,
                     conf=(6.0, 2.0), decay=0.9)
SWEEP_B = (1, 8, 32, 128, 512)
SWEEP_GAMMA = (4, 8, 16)


def sweep_point(B: int, gamma: int) -> Workload:
    return _lz(f"sweep_B{B}_g{gamma}", B=B, gamma=gamma, V=262144, T=1.0, seed=5000 + 100 * B + gamma)


WORKLOADS = {w.name: w for w in (TINY, SINGLE_USER, SINGLE_USER_GREEDY, HIGH_CONCURRENCY, SCHEDULED_STEP)}


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, *key])))


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """fp32 -> nearest-even bf16 value, returned as fp32 (exactly representable)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) & 0xFFFF0000
    return bits.astype(np.uint32).view(np.float32)


def weights(wl: Workload) -> Tuple[np.ndarray, np.ndarray]:
    """W1 [V, r], W2 [r, V] as fp32 arrays (bf16-exact values when w_dtype == 'bf16')."""
    W1 = _rng(wl.seed, _T_W1).standard_normal((wl.V, wl.r), dtype=np.float32) * np.float32(wl.w_sigma)
    W2 = _rng(wl.seed, _T_W2).standard_normal((wl.r, wl.V), dtype=np.float32) * np.float32(wl.w_sigma)
    if wl.w_dtype == "bf16":
        W1, W2 = round_to_bf16(W1), round_to_bf16(W2)
    return W1, W2


def logzipf_prior(wl: Workload) -> np.ndarray:
    """-s*ln(rank) over a seeded permutation of the vocabulary, fp32 [V]."""
    perm = _rng(wl.seed, _T_PERM).permutation(wl.V)
    rank = np.empty(wl.V, dtype=np.float64)
    rank[perm] = np.arange(1, wl.V + 1, dtype=np.float64)
    return (-wl.zipf_s * np.log(rank)).astype(np.float32)


def target_sigmas(wl: Workload) -> np.ndarray:
    """Noise std of the gamma+1 target rows (positions 1..gamma, then the bonus row)."""
    g = wl.gamma
    if g > 1:
        s = wl.t_sigma_first + (wl.t_sigma_last - wl.t_sigma_first) * np.arange(g) / (g - 1)
    else:
        s = np.array([wl.t_sigma_first])
    return np.concatenate([s, [wl.t_sigma_bonus]]).astype(np.float32)


def request_logits(wl: Workload, b: int, prior: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """(U_b [gamma, V], lt_b [gamma+1, V]) fp32 for request b alone."""
    G, V = wl.gamma, wl.V
    u_ext = _rng(wl.seed, _T_UEXT, b).standard_normal((G + 1, V), dtype=np.float32)
    u_ext *= np.float32(wl.u_sigma)
    if wl.logits == "logzipf":
        u_ext += prior if prior is not None else logzipf_prior(wl)
    noise = _rng(wl.seed, _T_TNOISE, b).standard_normal((G + 1, V), dtype=np.float32)
    noise *= target_sigmas(wl)[:, None]
    lt = u_ext + noise
    return np.ascontiguousarray(u_ext[:G]), lt


def logits(wl: Workload, requests=None) -> Tuple[np.ndarray, np.ndarray]:
    """(U [n, gamma, V], lt [n, gamma+1, V]) fp32 for the given requests (default all)."""
    reqs = list(range(wl.B)) if requests is None else list(requests)
    prior = logzipf_prior(wl) if wl.logits == "logzipf" else None
    U = np.empty((len(reqs), wl.gamma, wl.V), dtype=np.float32)
    lt = np.empty((len(reqs), wl.gamma + 1, wl.V), dtype=np.float32)
    for i, b in enumerate(reqs):
        U[i], lt[i] = request_logits(wl, b, prior)
    return U, lt


def tokens(wl: Workload) -> np.ndarray:
    return _rng(wl.seed, _T_X0).integers(0, wl.V, size=wl.B, dtype=np.int64).astype(np.int32)


def uniforms(wl: Workload) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(u_draft [B, gamma], u_acc [B, gamma], u_res [B]) fp32 in [0, 1)."""
    B, G = wl.B, wl.gamma
    u_draft = _rng(wl.seed, _T_UDRAFT).random((B, G), dtype=np.float32)
    u_acc = _rng(wl.seed, _T_UACC).random((B, G), dtype=np.float32)
    u_res = _rng(wl.seed, _T_URES).random(B, dtype=np.float32)
    return u_draft, u_acc, u_res


def confidences(wl: Workload) -> np.ndarray:
    """c [B, gamma] fp32: Beta(a, b) draws, decayed geometrically along the block."""
    c = _rng(wl.seed, _T_CONF).beta(wl.conf_a, wl.conf_b, size=(wl.B, wl.gamma))
    c = c * wl.conf_decay ** np.arange(wl.gamma)[None, :]
    return c.astype(np.float32)


def calibration_set(N: int, gamma: int, seed: int, a: float = 5.0, b: float = 2.0,
                    over: Tuple[float, float] = (1.1, 1.3)) -> Tuple[np.ndarray, np.ndarray]:
    """A validation set for confidence calibration: (c [N, gamma] fp32 raw confidences,
    n [N] int32 accepted counts).

    q ~ Beta(a, b) is the true probability that position k of sample i passes given that the
    positions before it passed; the sample's count n is its number of leading passes
    (position k passes when a U[0, 1) draw is below q).  The raw confidence overstates q as an
    over-confident head would: c = 1 - (1 - q)^s_k, with s_k rising linearly along the block
    from over[0] to over[1].
    """
    rng = _rng(seed, _T_CALIB)
    q = rng.beta(a, b, size=(N, gamma))
    u = rng.random((N, gamma))
    passed = np.cumprod(u < q, axis=1)
    n = passed.sum(axis=1).astype(np.int32)
    s = np.linspace(over[0], over[1], gamma)[None, :]
    c = 1.0 - (1.0 - q) ** s
    return c.astype(np.float32), n


def sps_table(wl: Workload, D_max: Optional[int] = None) -> np.ndarray:
    """steps/s of the verify forward as a function of D, the scheduled draft tokens, fp64 [D_max+1].

    The verify forward processes one committed token plus L_b draft tokens per
    request, so the batch it sees is B + D tokens.
    * "affine_latency": SPS(n) = 1 / (a + b*n), a = 5 ms, b = 0.04 ms per token.
    * "linear": SPS(n) = 100 * (1 - n / (2*B*(gamma+1))), a plain decreasing line.
    """
    D_max = wl.D_max if D_max is None else D_max
    n = wl.B + np.arange(D_max + 1, dtype=np.float64)
    if wl.sps == "affine_latency":
        return 1.0 / (0.005 + 0.00004 * n)
    if wl.sps == "linear":
        return 100.0 * (1.0 - n / (2.0 * wl.B * (wl.gamma + 1)))
    raise ValueError(wl.sps)


def full_inputs(wl: Workload) -> dict:
    """All host inputs of one round as numpy arrays."""
    U, lt = logits(wl)
    W1, W2 = weights(wl)
    u_draft, u_acc, u_res = uniforms(wl)
    return dict(U=U, lt=lt, W1=W1, W2=W2, x0=tokens(wl), u_draft=u_draft, u_acc=u_acc,
                u_res=u_res, c=confidences(wl), sps=sps_table(wl))


def device_logits(wl: Workload, device, requests=None):
    """(U [gamma, n, V] position-major, lt [n, gamma+1, V]) fp32 drawn on `device` with a seeded
    torch generator.

    Same shapes and value recipe as `logits`, for workloads too large to draw on
    the host (the vocabulary sweep); the values differ from `logits` but are
    reproducible for a given workload.  Rows of a request are a function of
    (seed, request) only, so any subset can be regenerated.
    """
    import torch

    reqs = list(range(wl.B)) if requests is None else list(requests)
    G, V = wl.gamma, wl.V
    prior = torch.from_numpy(logzipf_prior(wl)).to(device) if wl.logits == "logzipf" else None
    sig = torch.from_numpy(target_sigmas(wl)).to(device)[:, None]
    U = torch.empty((G, len(reqs), V), dtype=torch.float32, device=device)
    lt = torch.empty((len(reqs), G + 1, V), dtype=torch.float32, device=device)
    g = torch.Generator(device=device)
    for i, b in enumerate(reqs):
        g.manual_seed(wl.seed * 1_000_003 + b)
        u_ext = torch.randn((G + 1, V), generator=g, device=device) * wl.u_sigma
        if prior is not None:
            u_ext += prior
        U[:, i] = u_ext[:G]
        lt[i] = u_ext + torch.randn((G + 1, V), generator=g, device=device) * sig
    return U, lt
