"""CPU oracle of the DSpark draft/verify round (test infrastructure).

This is a plain, slow, float64 NumPy restatement of what the round computes.
It is test infrastructure: only the tests, the package smoke check and the
benchmark's CPU-baseline leg may import it.  It shares no code with the CUDA
path and never takes an input or an expected value from it.

Sources (three public web pages on DSpark):
  [P1] "大模型推理加速的系统级工程：DeepSeek V4-Pro DSpark 推测解码方案深度解析与开源工具链 DeepSpec"
       (austery.github.io write-up of a Best Partners TV video)
  [P2] "DeepSeek 开源 DSpark，一个可将大语言模型推理速度提升高达 85% 的新框架"
       (Chinese translation of a VentureBeat article)
  [P3] "DSpark Speculative Decoding" (lukebest.github.io concept note)

What each function follows:
  * draft      -- P3 §Semi-Autoregressive Generation: p_k(v) ∝ exp(U_k(v) + B_k(v)),
                  Markov head B(x_{k-1}, ·) = W1[x_{k-1}] W2 of low rank r;
                  P1 §"DSpark 架构设计：半自回归生成与马尔可夫修正" (one previous
                  token only, positions filled left to right).
  * rnn_draft  -- P1 §"DSpark 架构设计：半自回归生成与马尔可夫修正" (the optional RNN head: a
                  hidden state updated over the drafted prefix); P3 §Semi-Autoregressive
                  Generation (B_k(x_<k, v); RNN head with a recurrent state in the block).
  * verify     -- P1 §"大模型推理的显存瓶颈与推测解码的演进逻辑" (rejection
                  sampling: accept the longest prefix, resample at the first
                  rejection, drop the rest) and P3 opening paragraph (longest
                  consistent prefix plus a bonus token).
  * tv_labels  -- P3 §Confidence-Scheduled Verification: c*_k = 1 - ½‖p_d - p_t‖₁;
                  P1 §"硬件感知与置信度自适应调度机制" (label = analytic acceptance rate).
  * ragged_offsets, ragged_tags, pack_ragged, verify_ragged, tv_labels_ragged --
                  P1 §极致的工程实现与内核优化 (inference: all tokens to verify flattened into one
                  1-D array with a light token-tag tensor, no padding) and P3 production notes
                  (variable-length verify over flattened tokens with a marker tensor).
  * ece, sts_scale, sts_fit -- P1 §"硬件感知与置信度自适应调度机制" (sequential temperature
                  scaling: per-position 1-D grid search on a validation set, order-preserving,
                  ECE from 3-8 % to about 1 %); P3 §Confidence-Scheduled Verification (STS
                  calibrates the cumulative product position by position).
  * prefix_survival -- P3 §Confidence-Scheduled Verification: a_{r,j} = ∏_{i≤j} c_{r,i}.
  * prefix_schedule -- P3 §Confidence-Scheduled Verification (Algorithm 1,
                  Θ = τ·SPS(B)); P1 §"硬件感知与置信度自适应调度机制" (sort all
                  candidate tokens by survival, add them one at a time, evaluate
                  expected throughput, stop when it falls; global search on the GPU).
  * prefix_schedule_t2 -- P1 §"硬件感知与置信度自适应调度机制", last paragraph (the
                  truncation of step t decided from step t-2's confidence history);
                  P3 §Confidence-Scheduled Verification, production notes ("asynchronous":
                  confidences two steps back predict the batch capacity K).

Readings where the pages leave a step open:
  * temperature: p ∝ exp(ℓ/T) on both draft and target; the scaling is an fp32
    multiply of the fp32 logits by fl32(1/T), so that both sides take every
    sampling and acceptance decision from the same fp32 scaled logits; all
    later arithmetic is fp64.  T = 0 means greedy (argmax, lowest index).
  * the draft logits ℓ_d = U + bias are stored as fp32; sampling uses the
    stored values.
  * acceptance is strict: accept iff u·p_d(x) < p_t(x) (u in [0, 1)).
  * inverse CDF in vocabulary order: the first v with F_v > u; if rounding
    leaves u ≥ F_{V-1}, the last v with positive mass.
  * a zero residual after a rejection (only possible through rounding) falls
    back to sampling the target row.
  * one uniform u_res per request serves whichever of residual or bonus
    sample happens; the bonus uses target row L+1 (1-based).
  * Θ(D) = (B + S(D))·sps[D]: τ counts the always-emitted residual/bonus
    token of every request plus the expected accepted drafts S(D), the sum
    of the D largest survivals; sps is indexed by D.
  * ties in the survival sort: survival descending, then request, then position.
  * ARGMAX mode takes the smallest D attaining max Θ (global search);
    EARLY_STOP takes the first D with Θ(D+1) ≤ Θ(D).
  * RNN head: the pages give no form; here h_k = tanh(W1[x_{k-1}] + h_{k-1} W_h) (rank r,
    h_{-1} = 0) and the bias is h_k W2, so that W_h = 0 is the Markov head on tanh(W1).
  * flattened verification: request b owns target rows off[b] .. off[b] + L_b of one
    packed [Σ(L_b+1), V] array (off = exclusive prefix sum of L_b + 1); its tag is
    b·(γ+1) + k; it is verified exactly as the padded block; TV labels exist for the
    positions k <= min(L_b, γ-1) whose target row is present.
  * sequential temperature scaling: a confidence is scaled as σ(logit(c)/τ); positions are
    fitted in order, τ_k minimising (first grid value on ties) the ECE of the calibrated
    cumulative product against "positions 1..k accepted"; ECE uses 15 equal-width bins.
  * asynchronous (t-2) scheduling: only the capacity K_t (how many drafts step t
    verifies) comes from step t-2, as the search result D*_{t-2}; which drafts fill it is
    the first K_t items of step t's own survival order; steps 0 and 1 use a given
    initial capacity (default D_max).
  * near-ties: a decision closer than 1e-6 (|u - F|, |u - p_t/p_d|, a greedy
    top-2 gap of 1e-6·max(1,|z|)) or than 1e-12 relative (scheduler Θ) is
    reported together with every outcome that is valid within that window.
"""

from __future__ import annotations

import itertools
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

NEAR_TIE = 1e-6
THETA_NEAR_TIE = 1e-12

SCHED_ARGMAX = 0
SCHED_EARLY_STOP = 1


# --------------------------------------------------------------------------- shared definitions

def scaled_logits(logits, T: float) -> np.ndarray:
    """z = ℓ / T as the fp32 product ℓ · fl32(1/T) (reading of the temperature)."""
    l32 = np.asarray(logits, dtype=np.float32)
    inv_t = np.float32(1.0) / np.float32(T)
    return (l32 * inv_t).astype(np.float32)


def softmax(logits, T: float) -> np.ndarray:
    """p ∝ exp(ℓ/T) over the last axis, fp64 (P3 §Semi-Autoregressive Generation)."""
    z = scaled_logits(logits, T).astype(np.float64)
    m = np.max(z, axis=-1, keepdims=True)
    e = np.exp(z - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def greedy_choice(logits, near: float = NEAR_TIE) -> Tuple[int, List[int]]:
    """argmax with the lowest index on ties, plus every index within the near-tie gap
    near·max(1, |max|) of the maximum."""
    z = np.asarray(logits, dtype=np.float32).astype(np.float64)
    x = int(np.argmax(z))
    gap = near * max(1.0, abs(z[x]))
    alts = [int(v) for v in np.nonzero(z >= z[x] - gap)[0]]
    return x, alts


def inverse_cdf(p: np.ndarray, u: float, near: float = NEAR_TIE) -> Tuple[int, List[int]]:
    """Sample index v = min{v : F_v > u}, F the running sum of p in vocabulary order.

    Returns the index and every index whose CDF interval lies within `near` of u.
    """
    p = np.asarray(p, dtype=np.float64)
    F = np.cumsum(p)
    u = float(u)
    v = int(np.searchsorted(F, u, side="right"))
    if v >= p.shape[0]:
        v = int(np.nonzero(p > 0)[0][-1])
    lo = np.concatenate([[0.0], F[:-1]])
    close = (p > 0) & (lo - near <= u) & (u < F + near)
    alts = sorted(set(int(i) for i in np.nonzero(close)[0]) | {v})
    return v, alts


# --------------------------------------------------------------------------- draft (Markov head)

def markov_bias(W1, W2, prev) -> np.ndarray:
    """B(x_{k-1}, ·) = W1[x_{k-1}] · W2 in fp64 from the stored weights (P3 §Semi-Autoregressive Generation)."""
    W1 = np.asarray(W1)
    W2 = np.asarray(W2)
    g = W1[np.asarray(prev)].astype(np.float64)
    return g @ W2.astype(np.float64)


def draft_step(U_k, W1, W2, prev, u, T: float, W2_64: Optional[np.ndarray] = None):
    """One sequential step for one request: ℓ_d = U_k + W1[prev]·W2, then x ~ softmax(ℓ_d/T).

    Returns (x, ld32 [V], alternatives).  ld32 is ℓ_d rounded to fp32 (its stored type).
    """
    g = np.asarray(W1)[int(prev)].astype(np.float64)
    bias = g @ (W2_64 if W2_64 is not None else np.asarray(W2).astype(np.float64))
    ld32 = (np.asarray(U_k, dtype=np.float32).astype(np.float64) + bias).astype(np.float32)
    if T == 0.0:
        x, alts = greedy_choice(ld32)
    else:
        x, alts = inverse_cdf(softmax(ld32, T), u)
    return x, ld32, alts


def _sequential_draft(U, bias_of, x0, u_draft, T: float, follow: Optional[Dict], near: float):
    """The γ left-to-right sampling steps shared by both heads: step k stores
    ℓ_d = fl32(U_k + bias_of(k, previous tokens)) and samples x_k from it."""
    U = np.asarray(U, dtype=np.float32)
    B, G, V = U.shape
    x = np.zeros((B, G), dtype=np.int32)
    ld = np.zeros((B, G, V), dtype=np.float32)
    alts = {}
    prev = np.asarray(x0, dtype=np.int64).copy()
    for k in range(G):
        bias = bias_of(k, prev)                                   # [B, V] fp64
        ld[:, k] = (U[:, k].astype(np.float64) + bias).astype(np.float32)
        for b in range(B):
            if T == 0.0:
                xk, a = greedy_choice(ld[b, k], near)
            else:
                xk, a = inverse_cdf(softmax(ld[b, k], T), u_draft[b, k], near)
            if len(a) > 1:
                alts[(b, k)] = a
            if follow is not None and (b, k) in follow:
                f = int(follow[(b, k)])
                if f not in a:
                    raise ValueError(f"token {f} is not a valid outcome at {(b, k)}: {a}")
                xk = f
            x[b, k] = xk
        prev = x[:, k].astype(np.int64)
    return x, ld, alts


def markov_draft(U, W1, W2, x0, u_draft, T: float, follow: Optional[Dict] = None, near: float = NEAR_TIE):
    """The γ sequential Markov-head steps for every request.

    U [B, γ, V] fp32, x0 [B], u_draft [B, γ].  Step k uses the token chosen at
    step k-1 (x0 for the first step).  Returns (x [B, γ] int32,
    ld [B, γ, V] fp32, alts) where alts[(b, k)] lists the valid tokens at a
    near-tie.  `follow` maps (b, k) to a token that must be one of the valid
    alternatives at that step; the chain then continues from it (used to
    follow one branch of a near-tie).  `near` is the near-tie window.
    """
    W1 = np.asarray(W1)
    W2_64 = np.asarray(W2).astype(np.float64)
    return _sequential_draft(U, lambda k, prev: markov_bias(W1, W2_64, prev), x0, u_draft, T, follow, near)


def rnn_state(W1, Wh, prev, h_prev) -> np.ndarray:
    """h_k = tanh(W1[x_{k-1}] + h_{k-1} · W_h) in fp64 (row vectors; h before the block is 0)."""
    return np.tanh(np.asarray(W1)[np.asarray(prev)].astype(np.float64) + h_prev @ np.asarray(Wh).astype(np.float64))


def rnn_draft(U, W1, W2, Wh, x0, u_draft, T: float, follow: Optional[Dict] = None, near: float = NEAR_TIE):
    """The γ sequential steps with the recurrent head instead of the Markov head.

    P1 §DSpark 架构设计：半自回归生成与马尔可夫修正 (the optional RNN head keeps and updates a
    hidden state over the whole drafted prefix); P3 §Semi-Autoregressive Generation
    (p_k(v) ∝ exp(U_k(v) + B_k(x_<k, v)), RNN head: a recurrent state inside the block).
    Reading: a state h_k of the Markov head's rank r, h_k = tanh(W1[x_{k-1}] + h_{k-1} W_h)
    with h_{-1} = 0 and x_{-1} = x0, and B_k = h_k W2 (the Markov head's projections; W_h = 0
    gives the Markov head on tanh(W1)).  Returns (x, ld, alts, h [B, γ, r] fp64).
    """
    W1 = np.asarray(W1)
    Wh = np.asarray(Wh)
    W2_64 = np.asarray(W2).astype(np.float64)
    B = np.asarray(U).shape[0]
    hs = []
    state = {"h": np.zeros((B, W1.shape[1]))}

    def bias_of(k, prev):
        state["h"] = rnn_state(W1, Wh, prev, state["h"])
        hs.append(state["h"])
        return state["h"] @ W2_64

    x, ld, alts = _sequential_draft(U, bias_of, x0, u_draft, T, follow, near)
    return x, ld, alts, np.stack(hs, axis=1)


# --------------------------------------------------------------------------- verification

def verify_request(ld_b, lt_b, x_b, L: int, u_acc_b, u_res: float, T: float,
                   force_accept: Optional[Dict[int, bool]] = None, force_token: Optional[int] = None,
                   near: float = NEAR_TIE):
    """Rejection-sampling verification of one request's block.

    ld_b [γ, V] draft logits, lt_b [≥L+1, V] target logits, x_b [γ] drafted
    tokens, L the number of positions to verify.  Positions k = 0..L-1 are
    accepted while u·p_d(x_k) < p_t(x_k); at the first rejection one token is
    drawn from norm(max(0, p_t - p_d)); if all L survive, a bonus token is
    drawn from the target row L.

    Returns a dict with n (accepted count), y [γ+1] (x_0..x_{n-1}, the
    resampled/bonus token, then -1), accept_ties (positions whose decision is
    a near-tie), sample_alts (valid tokens for the last emitted one),
    residual_mass (Z when a residual was drawn) and kind ('residual'/'bonus').
    `force_accept`/`force_token` pin a near-tie outcome to one of its valid values
    (an outcome outside the near-tie window raises ValueError); `near` is the window.
    """
    G = len(x_b)
    V = np.asarray(lt_b).shape[-1]
    y = np.full(G + 1, -1, dtype=np.int32)
    accept_ties = []
    n = 0
    for k in range(L):
        xk = int(x_b[k])
        if T == 0.0:
            tk, talts = greedy_choice(lt_b[k], near)
            acc = (0 <= xk < V) and xk == tk
            if len(talts) > 1 and (xk in talts):
                accept_ties.append(k)
        else:
            if not (0 <= xk < V):
                acc = False
            else:
                pd = softmax(ld_b[k], T)[xk]
                pt = softmax(lt_b[k], T)[xk]
                u = float(u_acc_b[k])
                acc = u * pd < pt
                if pd > 0 and abs(u - pt / pd) < near:
                    accept_ties.append(k)
        if force_accept is not None and k in force_accept:
            if k not in accept_ties and force_accept[k] != acc:
                raise ValueError(f"position {k} is not a near-tie")
            acc = force_accept[k]
        if not acc:
            break
        y[k] = xk
        n += 1
    residual_mass = None
    if T == 0.0:
        tok, alts = greedy_choice(lt_b[n], near)
        kind = "residual" if n < L else "bonus"
    elif n < L:
        q = np.maximum(0.0, softmax(lt_b[n], T) - softmax(ld_b[n], T))
        Z = float(np.sum(q))
        residual_mass = Z
        kind = "residual"
        if Z > 0.0:
            tok, alts = inverse_cdf(q / Z, u_res, near)
        else:
            tok, alts = inverse_cdf(softmax(lt_b[n], T), u_res, near)
    else:
        kind = "bonus"
        tok, alts = inverse_cdf(softmax(lt_b[L], T), u_res, near)
    if force_token is not None:
        if force_token not in alts:
            raise ValueError(f"token {force_token} is not a valid outcome: {alts}")
        tok = force_token
    y[n] = tok
    return dict(n=n, y=y, accept_ties=accept_ties, sample_alts=alts, residual_mass=residual_mass, kind=kind)


def verify(ld, lt, x, L, u_acc, u_res, T: float):
    """Verify every request; returns (n_acc [B], y [B, γ+1], per-request detail dicts)."""
    ld = np.asarray(ld, dtype=np.float32)
    lt = np.asarray(lt, dtype=np.float32)
    B, G = np.asarray(x).shape
    n_acc = np.zeros(B, dtype=np.int32)
    y = np.full((B, G + 1), -1, dtype=np.int32)
    detail = []
    for b in range(B):
        Lb = G if L is None else int(L[b])
        r = verify_request(ld[b], lt[b], x[b], Lb, u_acc[b], u_res[b], T)
        n_acc[b], y[b] = r["n"], r["y"]
        detail.append(r)
    return n_acc, y, detail


# --------------------------------------------------------------------------- TV confidence labels

def tv_labels(ld, lt, T: float) -> np.ndarray:
    """c*_k = 1 - ½ Σ_v |p_d,k(v) - p_t,k(v)| for every drafted position (fp64 [B, γ]).

    Greedy (T = 0): the distributions are one-hot at the argmax, so c* is 1 when
    the argmaxes agree and 0 otherwise.
    """
    ld = np.asarray(ld, dtype=np.float32)
    lt = np.asarray(lt, dtype=np.float32)
    B, G, V = ld.shape
    out = np.zeros((B, G), dtype=np.float64)
    for b in range(B):
        for k in range(G):
            if T == 0.0:
                out[b, k] = 1.0 if int(np.argmax(ld[b, k])) == int(np.argmax(lt[b, k])) else 0.0
            else:
                out[b, k] = 1.0 - 0.5 * float(np.sum(np.abs(softmax(ld[b, k], T) - softmax(lt[b, k], T))))
    return out


# --------------------------------------------------------------------------- flattened (ragged) verification

def ragged_offsets(L, gamma: int):
    """Row offsets of the flattened target block: request b owns rows off[b] .. off[b] + L_b
    (its L_b verified positions and the bonus/resample position), so off[0] = 0 and
    off[b+1] = off[b] + L_b + 1; off[B] is the number of rows.  P1 §极致的工程实现与内核优化
    (inference): every token to verify goes into one contiguous 1-D array, no padding.
    L_b is clamped to [0, gamma] first.  Returns int64 [B+1]."""
    Lc = np.clip(np.asarray(L, dtype=np.int64), 0, gamma)
    off = np.zeros(Lc.size + 1, dtype=np.int64)
    for b in range(Lc.size):
        off[b + 1] = off[b] + Lc[b] + 1
    return off


def ragged_tags(L, gamma: int):
    """Token tags of the flattened rows: row off[b] + k carries b*(gamma+1) + k, which names
    its request and its position (P1 §极致的工程实现与内核优化: a light tag tensor marks
    which sequence, and where in it, each flattened token belongs).  int32 [off[B]]."""
    off = ragged_offsets(L, gamma)
    tags = np.empty(int(off[-1]), dtype=np.int32)
    for b in range(off.size - 1):
        for k in range(int(off[b + 1] - off[b])):
            tags[off[b] + k] = b * (gamma + 1) + k
    return tags


def pack_ragged(lt, L):
    """Padded target logits [B, γ+1, V] -> the flattened rows [off[B], V] (rows 0..L_b of b)."""
    lt = np.asarray(lt)
    B, G1, V = lt.shape
    off = ragged_offsets(L, G1 - 1)
    out = np.empty((int(off[-1]), V), dtype=lt.dtype)
    for b in range(B):
        n = int(off[b + 1] - off[b])
        out[off[b]:off[b] + n] = lt[b, :n]
    return out


def verify_ragged(ld, lt_packed, off, x, L, u_acc, u_res, T: float):
    """Verification over flattened target rows: request b's target row k is lt_packed[off[b] + k]
    for k = 0..L_b; otherwise exactly `verify` (rows past L_b are never read there either).
    Returns (n_acc, y, detail) like `verify`."""
    ld = np.asarray(ld, dtype=np.float32)
    lt_packed = np.asarray(lt_packed, dtype=np.float32)
    B, G = np.asarray(x).shape
    V = lt_packed.shape[1]
    n_acc = np.zeros(B, dtype=np.int32)
    y = np.full((B, G + 1), -1, dtype=np.int32)
    detail = []
    for b in range(B):
        Lb = int(L[b])
        assert int(off[b + 1]) - int(off[b]) == Lb + 1, "offsets must hold L_b + 1 rows per request"
        rows = np.full((G + 1, V), np.nan, dtype=np.float32)     # rows past L_b do not exist
        rows[:Lb + 1] = lt_packed[int(off[b]):int(off[b]) + Lb + 1]
        r = verify_request(ld[b], rows, x[b], Lb, u_acc[b], u_res[b], T)
        n_acc[b], y[b] = r["n"], r["y"]
        detail.append(r)
    return n_acc, y, detail


def tv_labels_ragged(ld, lt_packed, off, L, T: float):
    """TV labels of the positions whose target row exists in the flattened block
    (k <= min(L_b, γ-1)); NaN at the others."""
    ld = np.asarray(ld, dtype=np.float32)
    B, G, V = ld.shape
    out = np.full((B, G), np.nan, dtype=np.float64)
    for b in range(B):
        for k in range(min(int(L[b]) + 1, G)):
            out[b, k] = tv_labels(ld[b:b + 1, k:k + 1], np.asarray(lt_packed)[None, int(off[b]) + k:int(off[b]) + k + 1],
                                  T)[0, 0]
    return out


# --------------------------------------------------------------------------- confidence calibration

ECE_BINS = 15


def ece(p, s, n_bins: int = ECE_BINS) -> float:
    """Expected calibration error of predicted probabilities p against 0/1 outcomes s.

    Equal-width bins on [0, 1] (bin m holds p in [m/M, (m+1)/M), p = 1 in the last);
    ECE = Σ_m (|bin m| / N) · |mean outcome − mean prediction| = Σ_m |Σ_{i∈m} (s_i − p_i)| / N.
    P1 §硬件感知与置信度自适应调度机制 reports it before and after calibration."""
    p = np.asarray(p, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    m = np.minimum(np.floor(p * n_bins).astype(np.int64), n_bins - 1)
    total = 0.0
    for j in range(n_bins):
        sel = m == j
        total += abs(float(np.sum(s[sel])) - float(np.sum(p[sel])))
    return total / p.size


def sts_scale(c, tau):
    """Temperature scaling of a probability: σ(logit(c) / τ) in fp64, c clamped to [0, 1]
    (NaN counts as 0); 0 and 1 are fixed points.  Increasing in c for every τ > 0, so the order
    of the confidences is kept (P1 §硬件感知与置信度自适应调度机制)."""
    c = np.clip(np.nan_to_num(np.asarray(c, dtype=np.float64), nan=0.0), 0.0, 1.0)
    with np.errstate(divide="ignore"):
        z = np.log(c) - np.log1p(-c)
        return 1.0 / (1.0 + np.exp(-z / tau))


def sts_fit(c, n_acc, grid, n_bins: int = ECE_BINS, near: float = 1e-12, follow=None):
    """Sequential temperature scaling.

    P1 §硬件感知与置信度自适应调度机制: on a validation set, an independent 1-D grid search per
    candidate position finds the temperature that best calibrates the confidences (ECE from
    3-8 % to about 1 %), order-preserving; P3 §Confidence-Scheduled Verification: STS
    calibrates the cumulative product position by position.

    Reading: for k = 1..γ in order, with τ_1..τ_{k-1} already fixed, τ_k is the grid value
    (the first, on ties) minimising the ECE of the calibrated survival
    a'_k = ∏_{i≤k} σ(logit(c_i)/τ_i) against the outcome "positions 1..k all accepted"
    (n_acc ≥ k).  Products and ECE are fp64.

    c [N, γ], n_acc [N], grid [J] temperatures > 0.  `follow` (indices into the grid, one per
    position) takes those choices instead, each required to be within `near` of the minimum.
    Returns dict(tau [γ], index [γ], ece_raw [γ] (raw products ∏ c_i), ece_cal [γ],
    curves [γ, J], near_tie [γ])."""
    c = np.clip(np.nan_to_num(np.asarray(c, dtype=np.float64), nan=0.0), 0.0, 1.0)
    n_acc = np.asarray(n_acc)
    grid = np.asarray(grid, dtype=np.float64)
    N, G = c.shape
    a_raw = np.ones(N)
    a_cal = np.ones(N)
    out = dict(tau=np.zeros(G), index=np.zeros(G, dtype=np.int32), ece_raw=np.zeros(G), ece_cal=np.zeros(G),
               curves=np.zeros((G, grid.size)), near_tie=np.zeros(G, dtype=bool))
    for k in range(G):
        s = (n_acc >= k + 1).astype(np.float64)
        a_raw = a_raw * c[:, k]
        out["ece_raw"][k] = ece(a_raw, s, n_bins)
        curve = np.array([ece(a_cal * sts_scale(c[:, k], t), s, n_bins) for t in grid])
        j = int(np.argmin(curve))
        valid = np.flatnonzero(curve <= curve[j] + near)
        if follow is not None:
            if int(follow[k]) not in valid:
                raise ValueError(f"position {k}: grid index {follow[k]} is not within {near} of the minimum")
            j = int(follow[k])
        out["curves"][k] = curve
        out["index"][k] = j
        out["tau"][k] = grid[j]
        out["ece_cal"][k] = curve[j]
        out["near_tie"][k] = valid.size > 1
        a_cal = a_cal * sts_scale(c[:, k], grid[j])
    return out


# --------------------------------------------------------------------------- prefix survival + scheduler

def prefix_survival(c) -> np.ndarray:
    """a_{b,j} = ∏_{i≤j} c_{b,i}, multiplied left to right in fp32."""
    c = np.asarray(c, dtype=np.float32)
    return np.cumprod(c, axis=1, dtype=np.float32)


def schedule_order(a) -> np.ndarray:
    """Item order (flat index b*γ + j): survival descending, then request, then position."""
    a = np.asarray(a, dtype=np.float32)
    key = -a.reshape(-1).astype(np.float64)
    key[np.isnan(key)] = np.inf
    return np.argsort(key, kind="stable")


def prefix_schedule(c, sps, D_max: int, mode: int = SCHED_ARGMAX, near: float = THETA_NEAR_TIE):
    """Greedy hardware-aware prefix scheduler.

    All B·γ candidate tokens are ranked by prefix survival; adding them one at a
    time, the expected throughput after D additions is
    Θ(D) = (B + S(D)) · sps[D], with S(D) the sum of the D best survivals.
    ARGMAX keeps the best D over 0..D_max; EARLY_STOP keeps the first D after
    which Θ no longer rises.  L_b is the number of request b's tokens kept.

    Returns dict(L [B] int32, a [B, γ] fp32, theta (Θ at D*), D, thetas, near_tie); near_tie
    says whether another D is within `near` (relative) of the decision.
    """
    a = prefix_survival(c)
    B, G = a.shape
    D_max = int(min(D_max, B * G))
    sps = np.asarray(sps, dtype=np.float64)
    order = schedule_order(a)
    a_sorted = a.reshape(-1)[order].astype(np.float64)
    S = np.concatenate([[0.0], np.cumsum(a_sorted[:D_max])])
    theta = (B + S) * sps[: D_max + 1]
    if mode == SCHED_ARGMAX:
        D = int(np.argmax(theta))
        others = np.delete(theta, D)
        tie = bool(others.size and np.any(np.abs(others - theta[D]) <= near * abs(theta[D])))
    elif mode == SCHED_EARLY_STOP:
        D = D_max
        tie = False
        for d in range(D_max):
            if abs(theta[d + 1] - theta[d]) <= near * abs(theta[d]):
                tie = True
            if theta[d + 1] <= theta[d]:
                D = d
                break
    else:
        raise ValueError(mode)
    L = np.bincount(order[:D] // G, minlength=B).astype(np.int32)
    return dict(L=L, a=a, theta=float(theta[D]), D=D, thetas=theta, near_tie=tie)


def schedule_at_capacity(c, sps, K: int):
    """Algorithm 1 with the number of verified drafts fixed at K instead of searched.

    The first K items of the survival order are kept (K clamped to [0, B·γ]); returns
    (L [B] int32, Θ(K) = (B + S(K))·sps[K])."""
    a = prefix_survival(c)
    B, G = a.shape
    K = int(max(0, min(K, B * G)))
    order = schedule_order(a)
    S = float(np.sum(a.reshape(-1)[order[:K]].astype(np.float64)))
    return np.bincount(order[:K] // G, minlength=B).astype(np.int32), (B + S) * float(np.asarray(sps)[K])


def prefix_schedule_t2(c_steps: Sequence, sps, D_max, mode: int = SCHED_ARGMAX, K_init=None,
                       near: float = THETA_NEAR_TIE):
    """Asynchronous scheduling: the capacity of step t comes from step t-2's confidences.

    P1 §"硬件感知与置信度自适应调度机制", last paragraph: the truncation decision of step t
    rests on the confidence history of step t-2, so the global search can run inside the GPU
    pipeline without a host handshake; P3 §Confidence-Scheduled Verification (production
    notes, "asynchronous"): confidences from two steps earlier predict the batch capacity K.

    Reading: for each step t, D*_t is the global search of `prefix_schedule` on step t's
    confidences; the capacity of step t is K_t = D*_{t-2} (K_init for t < 2, default D_max),
    clamped to [0, min(D_max_t, B_t·γ)]; step t verifies the first K_t items of its own
    survival order (`schedule_at_capacity`).  c_steps is a sequence of [B_t, γ] arrays (B may
    change between steps); D_max is an int or one per step.

    Returns one dict per step: L, K (capacity applied), theta (Θ_t(K_t)), D (D*_t, the
    capacity that step t+2 will apply) and near_tie (whether the decision that gave K_t,
    made at step t-2, was a near-tie; False for t < 2).
    """
    steps = []
    n = len(c_steps)
    Dm = [int(D_max)] * n if np.isscalar(D_max) else [int(d) for d in D_max]
    for t, c in enumerate(c_steps):
        c = np.asarray(c, dtype=np.float32)
        B, G = c.shape
        cap = min(Dm[t], B * G)
        if t >= 2:
            K, tie = steps[t - 2]["D"], steps[t - 2]["decision_tie"]
        else:
            K, tie = (cap if K_init is None else int(K_init)), False
        K = int(max(0, min(K, cap)))
        L, theta = schedule_at_capacity(c, sps, K)
        d = prefix_schedule(c, sps, cap, mode, near)
        steps.append(dict(L=L, K=K, theta=theta, D=d["D"], near_tie=tie, decision_tie=d["near_tie"]))
    return steps


def exhaustive_schedule(c, sps, D_max: int):
    """Brute force over every length vector L ∈ {0..γ}^B with Σ L ≤ D_max.

    Θ(L) = (B + Σ_b Σ_{j<L_b} a_{b,j}) · sps[Σ L].  Returns (best Θ, list of the
    L attaining it within 1e-12 relative).  Only for tiny B and γ.
    """
    a = prefix_survival(c).astype(np.float64)
    B, G = a.shape
    cands = []
    for Ls in itertools.product(range(G + 1), repeat=B):
        D = sum(Ls)
        if D > D_max:
            continue
        tau = B + sum(float(np.sum(a[b, :Ls[b]])) for b in range(B))
        cands.append((tau * float(sps[D]), tuple(Ls)))
    best = max(t for t, _ in cands)
    return best, [Ls for t, Ls in cands if abs(t - best) <= THETA_NEAR_TIE * abs(best)]
