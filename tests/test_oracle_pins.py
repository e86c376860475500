"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these compares the oracle with itself: each check is a closed form,
an invariant, a special case with a known answer, or an exact (bisection)
measurement of the oracle's own u-driven decisions compared with the
distribution the pages say the round must reproduce.
"""

import itertools
import math

import numpy as np
import pytest
from scipy.special import expit, softmax as scipy_softmax

import oracle as O


# --------------------------------------------------------------------------- exact measurement helper

def measure(f, lo=0.0, hi=1.0, tol=1e-12):
    """Measure of {u in [lo, hi): f(u) = o} for each outcome o of a monotone step function f.

    f must be constant on every sub-interval whose two ends give the same
    outcome (true for an inverse CDF and for a threshold test).  Error is at
    most `tol` per breakpoint.
    """
    out = {}
    top = np.nextafter(hi, lo)
    stack = [(lo, top, f(lo), f(top))]
    while stack:
        a, b, fa, fb = stack.pop()
        if fa == fb:
            out[fa] = out.get(fa, 0.0) + (b - a)
            continue
        if b - a < tol:
            out[fa] = out.get(fa, 0.0) + (b - a) / 2
            out[fb] = out.get(fb, 0.0) + (b - a) / 2
            continue
        m = 0.5 * (a + b)
        fm = f(m)
        stack.append((a, m, fa, fm))
        stack.append((m, b, fm, fb))
    # the closed interval endpoints were counted as [lo, top]; top is one ulp below hi
    tot = sum(out.values())
    return {k: v * (hi - lo) / tot for k, v in out.items()}


# --------------------------------------------------------------------------- inverse CDF and softmax

def test_inverse_cdf_strict_threshold():
    p = np.full(4, 0.25)
    # F = [.25, .5, .75, 1]: first v with F_v > u
    assert O.inverse_cdf(p, 0.0)[0] == 0
    assert O.inverse_cdf(p, 0.25)[0] == 1
    assert O.inverse_cdf(p, 0.5)[0] == 2
    assert O.inverse_cdf(p, 0.74)[0] == 2
    assert O.inverse_cdf(p, 0.75)[0] == 3
    assert O.inverse_cdf(p, 0.9999)[0] == 3


def test_inverse_cdf_skips_zero_mass_and_falls_back():
    p = np.array([0.5, 0.0, 0.5])
    assert O.inverse_cdf(p, 0.5)[0] == 2          # never the zero-mass token
    p = np.array([0.25, 0.75, 0.0])
    assert O.inverse_cdf(p, 1.0)[0] == 1          # u beyond F_{V-1}: last positive-mass token


def test_inverse_cdf_uniform_closed_form():
    rng = np.random.default_rng(7)
    V = 1000
    p = np.full(V, 1.0 / V)
    for u in rng.random(200):
        frac = u * V - math.floor(u * V)
        if 1e-6 * V < frac < 1 - 1e-6 * V:
            assert O.inverse_cdf(p, u)[0] == math.floor(u * V)


def test_inverse_cdf_near_tie_alternatives():
    p = np.full(4, 0.25)
    v, alts = O.inverse_cdf(p, 0.5 + 1e-7)
    assert v == 2 and alts == [1, 2]
    v, alts = O.inverse_cdf(p, 0.5 - 1e-7)
    assert v == 1 and alts == [1, 2]
    v, alts = O.inverse_cdf(p, 0.6)
    assert alts == [2]


@pytest.mark.parametrize("T", [1.0, 0.5, 2.0, 0.8])
def test_two_point_softmax_is_logistic(T):
    # p(1) = 1 / (1 + exp(-(l1 - l0)/T)) for a two-token vocabulary
    for d in [-3.0, -0.5, 0.0, 0.25, 4.0]:
        logits = np.array([0.0, d], dtype=np.float32)
        z = O.scaled_logits(logits, T).astype(np.float64)
        p = O.softmax(logits, T)
        assert p[1] == pytest.approx(expit(z[1] - z[0]), rel=1e-14, abs=1e-300)
        # and the scaling itself is within one fp32 rounding of l/T
        assert z[1] == pytest.approx(d / T, rel=2 ** -23)


def test_temperature_sampling_breakpoint():
    # with a two-token vocabulary, x = 1 exactly for u >= p(0)
    T = 0.5
    d = 1.25
    U = np.array([[0.0, d]], dtype=np.float32)
    W1 = np.zeros((2, 1), dtype=np.float32)
    W2 = np.zeros((1, 2), dtype=np.float32)
    m = measure(lambda u: O.draft_step(U[0], W1, W2, 0, u, T)[0])
    assert m[1] == pytest.approx(expit(d / T), abs=1e-11)


@pytest.mark.parametrize("T", [1.0, 0.7])
def test_draft_sampler_distribution_is_the_softmax(T):
    # the draft token, as a function of its uniform, takes each v on a set of measure p_d(v):
    # p_d = softmax((U + W1[prev] W2) / T), here recomputed independently in fp64
    rng = np.random.default_rng(21)
    V, r = 8, 3
    U = rng.normal(scale=1.5, size=V).astype(np.float32)
    W1 = rng.normal(scale=0.7, size=(V, r)).astype(np.float32)
    W2 = rng.normal(scale=0.7, size=(r, V)).astype(np.float32)
    prev = 5
    m = measure(lambda u: O.draft_step(U, W1, W2, prev, u, T)[0])
    ld = U.astype(np.float64) + W1[prev].astype(np.float64) @ W2.astype(np.float64)
    want = scipy_softmax(ld / T)
    got = np.array([m.get(v, 0.0) for v in range(V)])
    np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-9)


def test_greedy_lowest_index_on_ties():
    x, alts = O.greedy_choice(np.array([1.0, 3.0, 3.0, -1.0], dtype=np.float32))
    assert x == 1 and alts == [1, 2]
    x, alts = O.greedy_choice(np.array([1.0, 3.0, 2.9, -1.0], dtype=np.float32))
    assert x == 1 and alts == [1]


# --------------------------------------------------------------------------- Markov-head draft

def test_markov_chain_uses_previous_token():
    # W1 = identity, W2[i, (i+1) % V] = 60: the bias forces x_k = x_{k-1} + 1 (mod V)
    V, G = 6, 5
    W1 = np.eye(V, dtype=np.float32)
    W2 = np.zeros((V, V), dtype=np.float32)
    for i in range(V):
        W2[i, (i + 1) % V] = 60.0
    U = np.zeros((2, G, V), dtype=np.float32)
    x0 = np.array([0, 4], dtype=np.int32)
    u = np.full((2, G), 0.5, dtype=np.float32)
    for T in (1.0, 0.0):
        x, ld, _ = O.markov_draft(U, W1, W2, x0, u, T)
        assert x.tolist() == [[1, 2, 3, 4, 5], [5, 0, 1, 2, 3]]
        # the stored draft logits are U + bias: 60 at the forced token, 0 elsewhere
        assert ld[0, 2, 3] == 60.0 and np.count_nonzero(ld[0, 2]) == 1


def test_markov_bias_rank_one_closed_form():
    # W1[v] = alpha_v e_0, W2[0] = beta: bias(prev) = alpha_prev * beta exactly
    V, r = 7, 3
    alpha = np.arange(1, V + 1, dtype=np.float32) * 0.5
    beta = np.linspace(-2, 2, V).astype(np.float32)
    W1 = np.zeros((V, r), dtype=np.float32)
    W1[:, 0] = alpha
    W2 = np.zeros((r, V), dtype=np.float32)
    W2[0] = beta
    for prev in range(V):
        assert np.array_equal(O.markov_bias(W1, W2, prev), alpha[prev].astype(np.float64) * beta.astype(np.float64))


def test_zero_bias_draft_is_independent_sampling():
    # W2 = 0: every position samples softmax(U_k / T) regardless of the previous token
    rng = np.random.default_rng(3)
    V, G, T = 5, 3, 1.0
    U = rng.normal(size=(1, G, V)).astype(np.float32)
    W1 = rng.normal(size=(V, 2)).astype(np.float32)
    W2 = np.zeros((2, V), dtype=np.float32)
    for k in range(G):
        for prev in range(V):
            m = measure(lambda u: O.draft_step(U[0, k], W1, W2, prev, u, T)[0])
            want = scipy_softmax(U[0, k].astype(np.float64))
            got = np.array([m.get(v, 0.0) for v in range(V)])
            np.testing.assert_allclose(got, want, atol=1e-10)


# --------------------------------------------------------------------------- lossless verification (brute force)

def _lossless_case(V, G, T, seed):
    rng = np.random.default_rng(seed)
    U = rng.normal(size=(G, V)).astype(np.float32)
    W1 = rng.normal(size=(V, 2)).astype(np.float32)
    W2 = rng.normal(size=(2, V)).astype(np.float32)
    x0 = 0
    tables = {}

    def target(prefix):
        # a prefix-dependent target model: fixed random logits per prefix (values on a 1/8 grid,
        # so that the fp32 scaling by 1/T is exact for T = 1 and T = 0.5)
        if prefix not in tables:
            r = np.random.default_rng([seed, len(prefix), *prefix])
            tables[prefix] = (np.round(r.normal(size=V) * 1.5 * 8) / 8).astype(np.float32)
        return tables[prefix]

    def draft_dist(k, prev):
        m = measure(lambda u: O.draft_step(U[k], W1, W2, prev, u, T)[0])
        ld = O.draft_step(U[k], W1, W2, prev, 0.5, T)[1]
        return m, ld

    emitted = {}      # tuple of emitted tokens -> probability
    first_accept = 0.0
    dcache = {}
    for x in np.ndindex(*(V,) * G):
        # draft probability of the sequence and its stored logits
        P = 1.0
        ld = np.zeros((G, V), dtype=np.float32)
        prev = x0
        for k in range(G):
            key = (k, prev)
            if key not in dcache:
                dcache[key] = draft_dist(k, prev)
            m, ld[k] = dcache[key]
            P *= m.get(x[k], 0.0)
            prev = x[k]
        if P == 0.0:
            continue
        lt = np.stack([target(tuple(x[:k])) for k in range(G + 1)])
        xs = np.array(x, dtype=np.int32)

        def run(u_acc, u_res):
            return O.verify_request(ld, lt, xs, G, u_acc, u_res, T)

        # acceptance probability at each position, reaching it with u = 0 before
        r = []
        for k in range(G):
            def acc_k(u, k=k):
                ua = np.zeros(G)
                ua[k] = u
                return run(ua, 0.5)["n"] > k
            mk = measure(acc_k)
            r.append(mk.get(True, 0.0))
        first_accept += P * r[0]
        reach = 1.0
        for m_ in range(G + 1):
            if m_ < G:
                p_stop = reach * (1.0 - r[m_])
            else:
                p_stop = reach
            if p_stop > 0:
                def tok(u, m_=m_):
                    ua = np.zeros(G)
                    if m_ < G:
                        ua[m_] = np.nextafter(1.0, 0.0)
                    out = run(ua, u)
                    assert out["n"] == m_
                    return int(out["y"][m_])
                dist = measure(tok)
                for v, pv in dist.items():
                    seq = tuple(int(t) for t in xs[:m_]) + (v,)
                    emitted[seq] = emitted.get(seq, 0.0) + P * p_stop * pv
            if m_ < G:
                reach *= r[m_]
    return emitted, target, first_accept, U, W1, W2, x0


@pytest.mark.parametrize("V,G,T,seed", [(5, 3, 1.0, 11), (4, 3, 0.5, 12), (8, 2, 1.0, 13)])
def test_verification_is_lossless(V, G, T, seed):
    """Every emitted token is distributed as the target given the emitted prefix."""
    emitted, target, _, *_ = _lossless_case(V, G, T, seed)
    assert sum(emitted.values()) == pytest.approx(1.0, abs=1e-9)
    for m in range(1, G + 2):
        prefixes = {}
        for seq, p in emitted.items():
            if len(seq) >= m:
                prefixes.setdefault(seq[: m - 1], {}).setdefault(seq[m - 1], 0.0)
                prefixes[seq[: m - 1]][seq[m - 1]] += p
        for s, dist in prefixes.items():
            tot = sum(dist.values())
            if tot < 1e-9:
                continue
            got = np.array([dist.get(v, 0.0) / tot for v in range(V)])
            want = scipy_softmax(target(s).astype(np.float64) / T)
            np.testing.assert_allclose(got, want, atol=2e-9 / tot + 1e-10)


def test_first_position_acceptance_rate_is_the_tv_label():
    # P(accept position 1) = sum_x p_d(x) min(1, p_t(x)/p_d(x)) = c*_1
    V, G, T, seed = 5, 3, 1.0, 11
    _, target, first_accept, U, W1, W2, x0 = _lossless_case(V, G, T, seed)
    ld0 = O.draft_step(U[0], W1, W2, x0, 0.5, T)[1]
    c = O.tv_labels(ld0[None, None], target(())[None, None], T)[0, 0]
    assert first_accept == pytest.approx(c, abs=1e-9)


def test_greedy_verification_emits_target_argmax_chain():
    rng = np.random.default_rng(5)
    V, G = 6, 4
    for trial in range(20):
        ld = rng.normal(size=(G, V)).astype(np.float32)
        x = rng.integers(0, V, size=G).astype(np.int32)
        lt = rng.normal(size=(G + 1, V)).astype(np.float32)
        # make some drafted tokens agree with the target argmax
        for k in range(G):
            if rng.random() < 0.6:
                lt[k, x[k]] = 10.0
        r = O.verify_request(ld, lt, x, G, np.full(G, 0.3), 0.7, 0.0)
        n = r["n"]
        expect_n = 0
        while expect_n < G and int(np.argmax(lt[expect_n])) == x[expect_n]:
            expect_n += 1
        assert n == expect_n
        assert r["y"][:n].tolist() == x[:n].tolist()
        assert r["y"][n] == int(np.argmax(lt[n]))
        assert (r["y"][n + 1:] == -1).all()


def test_identical_logits_accept_everything_and_bonus():
    rng = np.random.default_rng(9)
    V, G = 50, 5
    ld = rng.normal(size=(G, V)).astype(np.float32) * 3
    lt = np.concatenate([ld, rng.normal(size=(1, V)).astype(np.float32)])
    x = rng.integers(0, V, size=G).astype(np.int32)
    for T in (1.0, 0.7):
        u = np.nextafter(np.float32(1.0), np.float32(0.0)) * np.ones(G)
        r = O.verify_request(ld, lt, x, G, u, 0.3, T)
        assert r["n"] == G and r["kind"] == "bonus"
        assert r["y"][G] == O.inverse_cdf(O.softmax(lt[G], T), 0.3)[0]
        # scheduled L < gamma: bonus from row L
        r = O.verify_request(ld, lt, x, 2, u, 0.3, T)
        assert r["n"] == 2 and r["y"][2] == O.inverse_cdf(O.softmax(lt[2], T), 0.3)[0]
        assert (r["y"][3:] == -1).all()


def test_disjoint_support_rejects_and_resamples_target():
    V = 6
    ld = np.full((1, V), -1e4, dtype=np.float32)
    ld[0, 2] = 0.0                                   # draft is one-hot at token 2
    lt = np.zeros((2, V), dtype=np.float32)
    lt[0, 2] = -1e4                                  # target puts no mass on token 2
    x = np.array([2], dtype=np.int32)
    for u in (0.0, 0.5):
        r = O.verify_request(ld, lt, x, 1, np.array([u]), 0.45, 1.0)
        assert r["n"] == 0 and r["kind"] == "residual"
        assert r["residual_mass"] == pytest.approx(1.0, abs=1e-15)
        # residual = p_t: uniform over the 5 tokens != 2, u = 0.45 -> third of them
        assert r["y"][0] == [0, 1, 3, 4, 5][2]
    assert O.tv_labels(ld[None], lt[None, :1], 1.0)[0, 0] == pytest.approx(0.0, abs=1e-15)


# --------------------------------------------------------------------------- TV labels

def test_tv_two_point_closed_form_and_symmetry():
    for a, b in [(0.2, 0.7), (0.5, 0.5), (0.9, 0.1), (0.01, 0.99)]:
        ld = np.log(np.array([[[a, 1 - a]]])).astype(np.float32)
        lt = np.log(np.array([[[b, 1 - b]]])).astype(np.float32)
        pa = O.softmax(ld[0, 0], 1.0)[0]
        pb = O.softmax(lt[0, 0], 1.0)[0]
        c = O.tv_labels(ld, lt, 1.0)[0, 0]
        assert c == pytest.approx(1 - abs(pa - pb), abs=1e-15)
        assert c == pytest.approx(1 - abs(a - b), abs=1e-7)
        assert O.tv_labels(lt, ld, 1.0)[0, 0] == pytest.approx(c, abs=1e-16)


def test_tv_identity_and_range_and_min_identity():
    rng = np.random.default_rng(21)
    B, G, V = 3, 4, 200
    ld = (rng.normal(size=(B, G, V)) * 2).astype(np.float32)
    lt = (ld + rng.normal(size=(B, G, V)) * 0.8).astype(np.float32)
    for T in (1.0, 0.8):
        assert np.all(O.tv_labels(ld, ld, T) == 1.0)
        c = O.tv_labels(ld, lt, T)
        assert np.all((c >= 0) & (c <= 1))
        np.testing.assert_allclose(c, O.tv_labels(lt, ld, T), rtol=0, atol=1e-15)
        for b in range(B):
            for k in range(G):
                pd, pt = O.softmax(ld[b, k], T), O.softmax(lt[b, k], T)
                # 1 - TV = sum of the pointwise minimum = 1 - residual mass
                assert c[b, k] == pytest.approx(np.minimum(pd, pt).sum(), abs=1e-14)
                assert c[b, k] == pytest.approx(1 - np.maximum(0, pt - pd).sum(), abs=1e-14)


def test_tv_greedy_is_argmax_agreement():
    ld = np.array([[[0.0, 2.0, 1.0], [3.0, 0.0, 0.0]]], dtype=np.float32)
    lt = np.array([[[0.0, 5.0, 1.0], [0.0, 3.0, 0.0]]], dtype=np.float32)
    assert O.tv_labels(ld, lt, 0.0).tolist() == [[1.0, 0.0]]


# --------------------------------------------------------------------------- prefix survival

def test_prefix_survival_constant_and_monotone():
    for c0 in (0.9, 0.5, 0.123):
        c = np.full((2, 10), c0, dtype=np.float32)
        a = O.prefix_survival(c)
        want = np.float64(np.float32(c0)) ** np.arange(1, 11)
        np.testing.assert_allclose(a[0], want, rtol=1e-6)
    rng = np.random.default_rng(1)
    c = rng.random((5, 16)).astype(np.float32)
    a = O.prefix_survival(c)
    assert np.all(np.diff(a, axis=1) <= 0)
    assert np.array_equal(a[:, 0], c[:, 0])
    # one zero kills the rest of the block
    c[0, 3] = 0.0
    assert np.all(O.prefix_survival(c)[0, 3:] == 0)


# --------------------------------------------------------------------------- scheduler

def test_scheduler_hand_example():
    # B = 1, gamma = 2, c = (0.5, 0.5): a = (0.5, 0.25)
    # Θ(0) = 1*1 = 1, Θ(1) = 1.5*1 = 1.5, Θ(2) = 1.75*0.1 = 0.175  ->  D* = 1, L = (1)
    c = np.array([[0.5, 0.5]], dtype=np.float32)
    sps = np.array([1.0, 1.0, 0.1])
    r = O.prefix_schedule(c, sps, 2)
    assert r["D"] == 1 and r["L"].tolist() == [1] and r["theta"] == 1.5
    # two requests: a = (0.9, 0.45) and (0.6, 0.06); sps flat -> everything is worth adding
    c = np.array([[0.9, 0.5], [0.6, 0.1]], dtype=np.float32)
    r = O.prefix_schedule(c, np.ones(5), 4)
    assert r["D"] == 4 and r["L"].tolist() == [2, 2]
    # budget of 2: the two best survivals are 0.9 (request 0) and 0.6 (request 1)
    r = O.prefix_schedule(c, np.ones(5), 2)
    assert r["L"].tolist() == [1, 1]
    assert r["theta"] == pytest.approx(2 + np.float32(0.9) + np.float32(0.6), rel=1e-15)


def _staircase(n_max, B):
    # tensor-core-like staircase: flat within blocks of 8 tokens, dropping at each block edge
    n = B + np.arange(n_max + 1)
    return 1000.0 / (1.0 + np.ceil(n / 8.0))


@pytest.mark.parametrize("seed", range(12))
def test_scheduler_matches_exhaustive_search(seed):
    rng = np.random.default_rng(100 + seed)
    B = int(rng.integers(1, 4))
    G = int(rng.integers(1, 5))
    c = rng.beta(4, 2, size=(B, G)).astype(np.float32)
    D_max = int(rng.integers(0, B * G + 1))
    tables = [
        1.0 / (0.005 + 0.0004 * (B + np.arange(B * G + 1))),
        100.0 * (1.0 - (B + np.arange(B * G + 1)) / (2.0 * B * (G + 1))),
        _staircase(B * G, B),
        np.ones(B * G + 1),
    ]
    for sps in tables:
        r = O.prefix_schedule(c, sps, D_max)
        best, arg = O.exhaustive_schedule(c, sps, D_max)
        assert r["theta"] == pytest.approx(best, rel=1e-12)
        assert tuple(r["L"].tolist()) in arg or r["near_tie"]
        assert r["L"].sum() == r["D"] <= D_max
        assert np.all(r["L"] <= G)


def test_scheduler_constant_sps_takes_every_positive_item():
    rng = np.random.default_rng(8)
    c = rng.uniform(0.05, 1.0, size=(3, 4)).astype(np.float32)
    r = O.prefix_schedule(c, np.full(13, 7.0), 12)
    assert r["D"] == 12 and r["L"].tolist() == [4, 4, 4]
    c[1, 2] = 0.0        # a zero survival adds nothing, so ARGMAX keeps the smaller D
    r = O.prefix_schedule(c, np.full(13, 7.0), 12)
    assert r["L"].tolist() == [4, 2, 4]


def test_staircase_early_stop_falls_short_of_global_search():
    # Θ dips at the first stair and then recovers: early stopping is trapped in the
    # local optimum; the global search is not
    c = np.full((4, 4), 0.97, dtype=np.float32)
    sps = np.array([10.0, 6.0] + [5.9] * 15)
    e = O.prefix_schedule(c, sps, 16, O.SCHED_EARLY_STOP)
    g = O.prefix_schedule(c, sps, 16, O.SCHED_ARGMAX)
    assert e["D"] == 0 and g["D"] == 16 and e["theta"] < g["theta"]
    # concave Θ: the two modes agree
    sps2 = 1.0 / (0.005 + 0.00004 * (4 + np.arange(17)))
    e = O.prefix_schedule(c, sps2, 16, O.SCHED_EARLY_STOP)
    g = O.prefix_schedule(c, sps2, 16, O.SCHED_ARGMAX)
    assert e["D"] == g["D"]


def test_scheduler_ties_by_request_then_position():
    c = np.array([[0.5, 1.0], [0.5, 1.0]], dtype=np.float32)   # a = (0.5, 0.5) for both
    order = O.schedule_order(O.prefix_survival(c))
    assert order.tolist() == [0, 1, 2, 3]
    r = O.prefix_schedule(c, np.ones(5), 3)
    assert r["L"].tolist() == [2, 1]


# --------------------------------------------------------------------------- asynchronous (t-2) scheduling

def _ones_then_zeros(m, G):
    # request b passes its first m[b] positions for sure and fails the rest: a = 1 ... 1 0 ... 0
    return np.array([[1.0 if j < mb else 0.0 for j in range(G)] for mb in m], dtype=np.float32)


def test_t2_schedule_hand_example():
    # B = 3, gamma = 4, flat sps: Θ(D) = B + S(D) stops rising after the last positive survival,
    # so D*_t = sum(m_t).  Capacities: K_0 = K_1 = K_init = 12, then K_t = D*_{t-2}.
    # The survival order puts the ones first by (request, position), then the zeros likewise.
    #   t=2: m=[2,2,2], K=D*_0=5: ones (0,0)(0,1)(1,0)(1,1)(2,0)      -> L = [2,2,1]
    #   t=3: m=[0,0,0], K=D*_1=3: zeros (0,0)(0,1)(0,2)               -> L = [3,0,0]
    #   t=4: m=[4,4,4], K=D*_2=6: ones (0,0..3)(1,0)(1,1)             -> L = [4,2,0]
    #   t=5: m=[1,0,3], K=D*_3=0                                      -> L = [0,0,0]
    # A one-step lag would give K_2 = 3 and L_2 = [2,1,0].
    ms = [[4, 0, 1], [1, 1, 1], [2, 2, 2], [0, 0, 0], [4, 4, 4], [1, 0, 3]]
    c = [_ones_then_zeros(m, 4) for m in ms]
    r = O.prefix_schedule_t2(c, np.ones(13), 12, K_init=12)
    assert [s["D"] for s in r] == [5, 3, 6, 0, 12, 4]
    assert [s["K"] for s in r] == [12, 12, 5, 3, 6, 0]
    assert [s["L"].tolist() for s in r] == [[4, 4, 4], [4, 4, 4], [2, 2, 1], [3, 0, 0], [4, 2, 0], [0, 0, 0]]
    # Θ_t(K_t) = B + (number of ones among the first K_t items)
    assert [s["theta"] for s in r] == [8.0, 6.0, 8.0, 3.0, 9.0, 3.0]


def _exhaustive_at_capacity(a, K):
    """Largest Σ_b Σ_{j<L_b} a_{b,j} over prefix lengths with Σ L = K, by brute force."""
    B, G = a.shape
    best = -1.0
    for Ls in itertools.product(range(G + 1), repeat=B):
        if sum(Ls) == K:
            best = max(best, sum(float(np.sum(a[b, :Ls[b]], dtype=np.float64)) for b in range(B)))
    return best


@pytest.mark.parametrize("seed", range(8))
def test_capacity_schedule_maximises_expected_accepts(seed):
    # for a fixed number K of verified drafts, the first K items of the survival order carry
    # the largest expected number of accepted drafts among all prefix-closed choices
    rng = np.random.default_rng(300 + seed)
    B, G = int(rng.integers(1, 4)), int(rng.integers(1, 5))
    c = rng.beta(3, 2, size=(B, G)).astype(np.float32)
    a = O.prefix_survival(c).astype(np.float64)
    for K in range(B * G + 1):
        L, theta = O.schedule_at_capacity(c, np.ones(B * G + 1), K)
        assert L.sum() == K and np.all(L <= G)
        assert theta - B == pytest.approx(_exhaustive_at_capacity(a, K), rel=1e-12)


def test_t2_schedule_lag_and_clamp():
    rng = np.random.default_rng(41)
    sps = 1.0 / (0.005 + 0.0004 * (6 + np.arange(6 * 5 + 1)))
    c = [rng.beta(4, 2, size=(6, 5)).astype(np.float32) for _ in range(6)]
    r = O.prefix_schedule_t2(c, sps, 30)
    sync = [O.prefix_schedule(ct, sps, 30) for ct in c]
    assert r[0]["K"] == r[1]["K"] == 30                       # default initial capacity: D_max
    for t in range(6):
        assert r[t]["D"] == sync[t]["D"]
        if t >= 2:
            assert r[t]["K"] == sync[t - 2]["D"]
            assert r[t]["near_tie"] == sync[t - 2]["near_tie"]
    # stationary confidences: from step 2 on, the asynchronous schedule is the synchronous one
    r = O.prefix_schedule_t2([c[0]] * 4, sps, 30)
    for t in (2, 3):
        assert np.array_equal(r[t]["L"], sync[0]["L"]) and r[t]["theta"] == pytest.approx(sync[0]["theta"], rel=1e-15)
    # the batch shrinks: a capacity from a larger step is clamped to the new B * gamma and D_max
    c2 = [c[0], c[1], c[2][:2], c[3][:1]]
    r = O.prefix_schedule_t2(c2, sps, [30, 30, 7, 30])
    assert r[2]["K"] == min(sync[0]["D"], 7) and r[3]["K"] == min(sync[1]["D"], 5)
    assert r[3]["L"].sum() == r[3]["K"]


# --------------------------------------------------------------------------- flattened (ragged) verification

def test_ragged_offsets_and_tags_hand_example():
    # request b owns L_b + 1 rows: lengths 3, 1, 6, 2 -> offsets 0, 3, 4, 10, 12
    assert O.ragged_offsets([2, 0, 5, 1], 5).tolist() == [0, 3, 4, 10, 12]
    # tags b*(gamma+1) + k with gamma = 3: request 0 rows k=0..2, request 1 k=0, request 2 k=0..1
    assert O.ragged_tags([2, 0, 1], 3).tolist() == [0, 1, 2, 4, 8, 9]
    # lengths outside [0, gamma] are clamped first
    assert O.ragged_offsets([7, -1], 5).tolist() == [0, 6, 7]
    assert O.ragged_offsets([], 4).tolist() == [0]


@pytest.mark.parametrize("T", [1.0, 0.7, 0.0])
def test_ragged_verify_is_the_padded_verify(T):
    rng = np.random.default_rng(51)
    B, G, V = 7, 4, 300
    ld = rng.normal(0, 1.5, (B, G, V)).astype(np.float32)
    lt = (ld[:, [0, 1, 2, 3, 3]] + rng.normal(0, 0.7, (B, G + 1, V))).astype(np.float32)
    L = np.array([0, 4, 2, 1, 3, 4, 0], dtype=np.int32)
    x = np.argmax(ld + rng.gumbel(size=ld.shape).astype(np.float32), axis=2).astype(np.int32)
    u_acc = rng.random((B, G)).astype(np.float32)
    u_res = rng.random(B).astype(np.float32)
    # rows past L_b are NaN in the padded block: neither form may read them
    lt_pad = lt.copy()
    for b in range(B):
        lt_pad[b, L[b] + 1:] = np.nan
    packed = O.pack_ragged(lt_pad, L)
    off = O.ragged_offsets(L, G)
    assert packed.shape == (int(L.sum()) + B, V) and not np.isnan(packed).any()
    n0, y0, _ = O.verify(ld, lt_pad, x, L, u_acc, u_res, T)
    n1, y1, _ = O.verify_ragged(ld, packed, off, x, L, u_acc, u_res, T)
    assert np.array_equal(n0, n1) and np.array_equal(y0, y1)
    assert np.all(n1 <= L) and np.all(y1[np.arange(B), n1] >= 0)
    # TV labels where the target row exists, NaN elsewhere
    c = O.tv_labels_ragged(ld, packed, off, L, T)
    full = O.tv_labels(ld, lt, T)
    for b in range(B):
        k_have = min(int(L[b]) + 1, G)
        assert np.array_equal(c[b, :k_have], full[b, :k_have]) and np.isnan(c[b, k_have:]).all()


# --------------------------------------------------------------------------- calibration (STS, ECE)

def test_ece_closed_forms():
    # one bin, predictions equal to the bin's frequency: 0
    assert O.ece([0.75] * 4, [1, 1, 1, 0]) == 0.0
    # bins 1 and 13 (15 bins): (|1 - 0.1| + |0 - 0.9|) / 2
    assert O.ece([0.1, 0.9], [1, 0]) == pytest.approx(0.9, rel=1e-15)
    # p = 1 falls in the last bin together with 0.95: |2 - 1.95| / 2
    assert O.ece([1.0, 0.95], [1, 1]) == pytest.approx(0.025, rel=1e-12)
    # two bins of 10 bins: (|3 - 4*0.25| + |1 - 2*0.85|) / 6
    assert O.ece([0.25] * 4 + [0.85] * 2, [1, 1, 1, 0, 1, 0], n_bins=10) == pytest.approx((2.0 + 0.7) / 6, rel=1e-12)


def test_ece_matches_the_library_reliability_curve():
    from sklearn.calibration import calibration_curve
    rng = np.random.default_rng(61)
    p = rng.beta(3, 2, 5000)
    s = (rng.random(5000) < p ** 1.3).astype(np.int64)
    frac_pos, mean_pred = calibration_curve(s, p, n_bins=15, strategy="uniform")
    counts = np.bincount(np.minimum((p * 15).astype(int), 14), minlength=15)
    w = counts[counts > 0] / p.size
    assert O.ece(p, s) == pytest.approx(float(np.sum(w * np.abs(frac_pos - mean_pred))), rel=1e-12)


def test_temperature_scaling_closed_forms_and_order():
    # logit(0.8) = ln 4; halved: ln 2 -> 2/3
    assert float(O.sts_scale(0.8, 2.0)) == pytest.approx(2.0 / 3.0, rel=1e-15)
    assert float(O.sts_scale(0.2, 0.5)) == pytest.approx(1.0 / 17.0, rel=1e-14)   # logit -ln 4 doubled
    c = np.array([0.0, 1e-6, 0.3, 0.5, 0.9, 1.0, np.nan, 1.5, -0.2])
    for tau in (0.3, 1.0, 2.7):
        out = O.sts_scale(c, tau)
        assert out[0] == 0.0 and out[5] == 1.0 and out[3] == 0.5 and out[6] == 0.0
        assert out[7] == 1.0 and out[8] == 0.0                          # clamped into [0, 1]
        assert np.all(np.diff(out[:6]) > 0)                             # order kept
    assert np.allclose(O.sts_scale(c[:6], 1.0), c[:6], rtol=1e-15, atol=0)


def _logit_overconfident(N, scales, seed):
    from scipy.special import expit, logit
    rng = np.random.default_rng(seed)
    G = len(scales)
    q = rng.beta(4, 2, size=(N, G))
    n = np.cumprod(rng.random((N, G)) < q, axis=1).sum(axis=1)
    c = expit(logit(q) * np.asarray(scales)[None, :])
    return c, n


def test_sts_recovers_known_temperatures_position_by_position():
    # confidences miscalibrated by a known temperature per position (over-, under-, over-
    # confident): the fit recovers each one, which it can only do if position k is fitted on
    # top of the calibrated positions before it
    scales = [2.0, 0.5, 1.5]
    c, n = _logit_overconfident(200_000, scales, 62)
    grid = np.exp(np.linspace(np.log(0.25), np.log(4.0), 81))
    r = O.sts_fit(c, n, grid)
    assert np.all(np.abs(np.log(r["tau"]) - np.log(scales)) < 0.08), r["tau"]
    assert np.all(r["ece_cal"] < 0.01) and np.all(r["ece_cal"] < r["ece_raw"])
    assert np.all(r["curves"][np.arange(3), r["index"]] == r["ece_cal"])
    # following a grid value that is not the minimum is refused
    with pytest.raises(ValueError):
        O.sts_fit(c, n, grid, follow=[0, 0, 0])


def test_sts_on_the_synthetic_validation_set():
    # the pages: ECE of 3-8 % before calibration, about 1 % after
    from speculative_decoding_04_b200 import inputs
    c, n = inputs.calibration_set(40_000, 8, 5)
    grid = np.exp(np.linspace(np.log(0.25), np.log(4.0), 81))
    r = O.sts_fit(c, n, grid)
    assert np.all((r["ece_raw"] > 0.02) & (r["ece_raw"] < 0.08))
    assert np.all(r["ece_cal"] < 0.02) and np.mean(r["ece_cal"]) < 0.013
    assert np.all(r["tau"] > 1.0)                                       # over-confident: flattened


# --------------------------------------------------------------------------- RNN head

def test_rnn_head_hand_example():
    # V = 2, r = 2, greedy with token 0 far ahead everywhere, so x_k = 0 throughout:
    #   h_0 = tanh(W1[0]),  h_k = tanh(W1[0] + h_{k-1} Wh)  (row vector times Wh, Wh not symmetric)
    #   l_d[k] = U[k] + h_k W2
    W1 = np.array([[0.5, -0.25], [0.1, 0.3]])
    Wh = np.array([[0.8, -0.4], [0.3, 0.6]])
    W2 = np.array([[1.0, -1.0], [0.5, 2.0]])
    U = np.zeros((1, 3, 2), dtype=np.float32)
    U[0, :, 0] = 10.0
    x, ld, _, h = O.rnn_draft(U, W1, W2, Wh, np.array([0]), np.zeros((1, 3)), 0.0)
    assert x.tolist() == [[0, 0, 0]]
    hk = [math.tanh(0.5), math.tanh(-0.25)]
    for k in range(3):
        if k:
            hk = [math.tanh(0.5 + hk[0] * 0.8 + hk[1] * 0.3), math.tanh(-0.25 + hk[0] * -0.4 + hk[1] * 0.6)]
        assert h[0, k].tolist() == pytest.approx(hk, rel=1e-15)
        want = [10.0 + hk[0] * 1.0 + hk[1] * 0.5, hk[0] * -1.0 + hk[1] * 2.0]
        assert ld[0, k].tolist() == pytest.approx(np.float32(want).tolist(), rel=0, abs=0)


def test_rnn_head_without_recurrence_is_the_markov_head_on_tanh_embeddings():
    rng = np.random.default_rng(71)
    B, G, V, r = 5, 4, 300, 8
    U = rng.normal(0, 1.0, (B, G, V)).astype(np.float32)
    W1 = rng.normal(0, 0.8, (V, r))
    W2 = rng.normal(0, 0.5, (r, V))
    x0 = rng.integers(0, V, B)
    u = rng.random((B, G)).astype(np.float32)
    for T in (1.0, 0.0):
        x, ld, _, _ = O.rnn_draft(U, W1, W2, np.zeros((r, r)), x0, u, T)
        xm, ldm, _ = O.markov_draft(U, np.tanh(W1), W2, x0, u, T)
        assert np.array_equal(x, xm) and np.array_equal(ld, ldm)


def test_rnn_head_sees_the_whole_prefix():
    # the same token at position 0 after different starting tokens: the Markov head's logits at
    # position 1 agree, the recurrent head's do not (its state still carries x0)
    rng = np.random.default_rng(72)
    V, r = 50, 6
    W1 = rng.normal(0, 0.8, (V, r))
    W2 = rng.normal(0, 0.5, (r, V))
    Wh = rng.normal(0, 0.5, (r, r))
    U = np.zeros((2, 2, V), dtype=np.float32)
    U[:, 0, 7] = 50.0                                              # position 0 drafts token 7 in both
    x0 = np.array([3, 11])
    u = np.full((2, 2), 0.5, dtype=np.float32)
    x, ld, _, _ = O.rnn_draft(U, W1, W2, Wh, x0, u, 1.0)
    assert x[0, 0] == x[1, 0] == 7
    assert not np.allclose(ld[0, 1], ld[1, 1])
    xm, ldm, _ = O.markov_draft(U, W1, W2, x0, u, 1.0)
    assert np.array_equal(ldm[0, 1], ldm[1, 1])
