"""Rejection-sampling verification and TV labels on the GPU against the oracle."""

import numpy as np
import pytest
import torch

import oracle as O
from speculative_decoding_04_b200 import dspark as D
from speculative_decoding_04_b200 import inputs
from tests.parity import check_labels, check_verify, dev, draw_tokens, host, pm

pytestmark = pytest.mark.gpu


def case(B, G, V, T, seed, sigma_t=0.7, logits="logzipf"):
    wl = inputs.SINGLE_USER.with_(name="vcase", B=B, gamma=G, V=V, T=T, seed=seed, logits=logits,
                                  t_sigma_first=sigma_t, t_sigma_last=sigma_t, t_sigma_bonus=sigma_t)
    U, lt = inputs.logits(wl)
    ld = U  # draft logits of the case (any fp32 logits serve)
    u_draft, u_acc, u_res = inputs.uniforms(wl)
    x = draw_tokens(ld, u_draft, T)
    return ld, lt, x, u_acc, u_res


def run_verify(ld, lt, x, L, u_acc, u_res, T, want_c=True):
    n, y, c, fl = D.verify(pm(ld), dev(lt), dev(x), None if L is None else dev(L), dev(u_acc), dev(u_res), T,
                           want_c_star=want_c)
    torch.cuda.synchronize()
    return host(n), host(y), (host(c) if c is not None else None), host(fl)


# kernels: "stream-C" = streaming kernels with clusters of C CTAs (the default with a workspace;
# C = 0: automatic, C > 8: non-portable cluster sizes); "sliced-G" = column-sliced kernels with G groups of CTAs (0: slices of about 16 KB);
# "rows-C" = one cluster of C CTAs per row (0: chosen from V), which serves calls without a
# workspace, V not a multiple of 4 and the labels entry point.
IMPLS = ["sliced-0", "sliced-1", "sliced-3", "sliced-16", "stream-0", "stream-16", "stream-8", "stream-3", "stream-1",
         "rows-0", "rows-1", "rows-4", "rows-16"]


def use_impl(impl):
    kind, c = impl.split("-")
    D.set_option("verify_impl", {"stream": 0, "sliced": 1, "rows": 2}[kind])
    if kind == "sliced":
        D.set_option("verify_groups", int(c))
    elif kind == "stream":
        D.set_option("verify_stream_cluster", int(c))
    else:
        D.set_option("verify_cluster", int(c))
    return kind, int(c)


@pytest.mark.parametrize("V", [1003, 4096, 30000])
@pytest.mark.parametrize("T", [1.0, 0.7, 0.0])
@pytest.mark.parametrize("scheduled", [False, True])
@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("labels", [True, False])
def test_verify_matches_oracle(V, T, scheduled, impl, labels):
    kind, cluster = use_impl(impl)
    if kind == "rows" and cluster and V < 4096 and cluster > 4:
        pytest.skip("slice smaller than the block")
    if kind in ("stream", "sliced") and V % 4:
        pytest.skip("the sliced and streaming kernels need V % 4 == 0 (other V take the per-row kernels)")
    B, G = 6, 4
    ld, lt, x, u_acc, u_res = case(B, G, V, T, seed=V + int(T * 10) + cluster)
    # without labels, rows past L_b + 1 are skipped by the kernels
    L = np.array([0, 1, 2, 3, 4, 2], dtype=np.int32) if scheduled else None
    n, y, c, fl = run_verify(ld, lt, x, L, u_acc, u_res, T, want_c=labels)
    check_verify(ld, lt, x, L, u_acc, u_res, T, n, y, flags_gpu=fl)
    if labels:
        check_labels(ld, lt, T, c)
    G_ = G if L is None else L
    assert np.all(n <= G_)


@pytest.mark.parametrize("T", [1.0, 0.8])
def test_identical_logits_accept_all_and_label_one(T):
    ld, lt, x, u_acc, u_res = case(5, 6, 20000, T, seed=3)
    lt[:, :6] = ld
    u_acc[:] = np.nextafter(np.float32(1), np.float32(0))
    for L in (None, np.array([6, 0, 3, 5, 1], dtype=np.int32)):
        n, y, c, fl = run_verify(ld, lt, x, L, u_acc, u_res, T)
        want_n = np.full(5, 6) if L is None else L
        assert np.array_equal(n, want_n)
        assert np.all(c == 1.0)
        check_verify(ld, lt, x, L, u_acc, u_res, T, n, y, flags_gpu=fl)


def test_disjoint_support_is_certain_rejection():
    B, G, V = 2, 2, 4096
    ld = np.full((B, G, V), -1e4, dtype=np.float32)
    ld[:, :, 7] = 0.0
    lt = np.zeros((B, G + 1, V), dtype=np.float32)
    lt[:, :, 7] = -1e4
    x = np.full((B, G), 7, dtype=np.int32)
    u_acc = np.zeros((B, G), dtype=np.float32)
    u_res = np.array([0.5 / (V - 1), 1 - 0.5 / (V - 1)], dtype=np.float32)   # middle of the first / last interval
    n, y, c, fl = run_verify(ld, lt, x, None, u_acc, u_res, 1.0)
    assert np.all(n == 0) and np.all(c == 0.0)
    assert y[0, 0] == 0 and y[1, 0] == V - 1
    check_verify(ld, lt, x, None, u_acc, u_res, 1.0, n, y, flags_gpu=fl)


@pytest.mark.parametrize("lt_rows", ["gamma", "gamma+1"])
@pytest.mark.parametrize("T", [1.0, 0.5, 0.0])
def test_tv_labels_entry_point(lt_rows, T):
    ld, lt, x, u_acc, u_res = case(4, 5, 50000, T, seed=11, sigma_t=1.5)
    if lt_rows == "gamma":
        lt = np.ascontiguousarray(lt[:, :5])
    c = host(D.tv_labels(pm(ld), dev(lt), T))
    check_labels(ld, lt, T, c)
    assert np.all((c >= 0) & (c <= 1))


def test_bad_token_and_nonfinite_are_flagged():
    ld, lt, x, u_acc, u_res = case(3, 3, 4096, 1.0, seed=12)
    x[0, 0] = -3
    lt[2, 1, 100] = np.inf
    n, y, c, fl = run_verify(ld, lt, x, None, u_acc, u_res, 1.0)
    assert fl[0] & D.FLAG_TOKEN_RANGE and n[0] == 0
    assert fl[2] & D.FLAG_NONFINITE
    assert np.all((y[:, 0] >= 0) & (y[:, 0] < 4096))
    check_verify(ld, lt, x, None, u_acc, u_res, 1.0, n, y, requests=[1])


@pytest.mark.parametrize("cluster", [0, 16])
def test_acceptance_rate_matches_label_statistically(cluster):
    # P(accept position 1) = c*_1 = sum min(p_d, p_t): many requests sharing the same rows, so that
    # hundreds of rows per cluster pass through the exchange slots (clusters of 16: CTAs without tiles)
    D.set_option("verify_stream_cluster", cluster)
    B, G, V = 4000, 1, 512
    rng = np.random.default_rng(0)
    ld1 = (rng.normal(size=V) * 2).astype(np.float32)
    lt1 = (ld1 + rng.normal(size=V)).astype(np.float32)
    ld = np.broadcast_to(ld1, (B, G, V)).copy()
    lt = np.broadcast_to(np.stack([lt1, lt1]), (B, G + 1, V)).copy()
    u = rng.random((B, G), dtype=np.float32)
    x = draw_tokens(ld, rng.random((B, G), dtype=np.float32), 1.0)
    n, y, c, fl = run_verify(ld, lt, x, None, u, rng.random(B, dtype=np.float32), 1.0)
    c1 = O.tv_labels(ld[:1], lt[:1, :1], 1.0)[0, 0]
    rate = n.mean()
    assert abs(rate - c1) < 4 * np.sqrt(c1 * (1 - c1) / B)


@pytest.mark.parametrize("impl", ["sliced-0", "sliced-7", "stream-8", "stream-2", "persistent-1", "persistent-0"])
def test_scheduled_rows_skipped_many_requests(impl):
    kind, v = impl.split("-")
    D.set_option("verify_impl", {"stream": 0, "sliced": 1, "persistent": 2}[kind])
    if kind == "sliced":
        D.set_option("verify_groups", int(v))
    elif kind == "stream":
        D.set_option("verify_stream_cluster", int(v))
    else:
        D.set_option("verify_persistent", int(v))
    B, G, V = 40, 6, 20000
    ld, lt, x, u_acc, u_res = case(B, G, V, 1.0, seed=77)
    L = (np.arange(B) * 7 % (G + 1)).astype(np.int32)
    n, y, c, fl = run_verify(ld, lt, x, L, u_acc, u_res, 1.0, want_c=False)
    check_verify(ld, lt, x, L, u_acc, u_res, 1.0, n, y, flags_gpu=fl)
    assert np.all(n <= L)


@pytest.mark.parametrize("T", [1.0, 0.0])
def test_stream_vocabulary_beyond_per_row_kernels(T):
    # V = 500,000: more than one 16-CTA cluster can hold per row; the streaming kernels take it
    # (rows of 489 tiles, the last one 288 columns wide), the per-row kernels refuse it
    B, G, V = 3, 3, 500_000
    ld, lt, x, u_acc, u_res = case(B, G, V, T, seed=91)
    n, y, c, fl = run_verify(ld, lt, x, None, u_acc, u_res, T)
    check_verify(ld, lt, x, None, u_acc, u_res, T, n, y, flags_gpu=fl)
    check_labels(ld, lt, T, c)
    D.set_option("verify_impl", 2)
    with pytest.raises(D.DsparkError) as e:
        run_verify(ld, lt, x, None, u_acc, u_res, T)
    assert e.value.status == D.ENOTIMPL


@pytest.mark.parametrize("cluster", [2, 8, 12])
@pytest.mark.parametrize("T", [1.0, 0.0])
def test_stream_scheduled_rows_with_and_without_labels(cluster, T):
    # rows past L_b + 1 skipped when no labels are asked for; all rows read with labels
    D.set_option("verify_impl", 0)
    D.set_option("verify_stream_cluster", cluster)
    B, G, V = 24, 5, 20000
    ld, lt, x, u_acc, u_res = case(B, G, V, T, seed=300 + cluster)
    L = (np.arange(B) * 5 % (G + 1)).astype(np.int32)
    for want_c in (True, False):
        n, y, c, fl = run_verify(ld, lt, x, L, u_acc, u_res, T, want_c=want_c)
        check_verify(ld, lt, x, L, u_acc, u_res, T, n, y, flags_gpu=fl)
        if want_c:
            check_labels(ld, lt, T, c)


@pytest.mark.parametrize("groups", [1, 5, 30])
@pytest.mark.parametrize("T", [0.9, 0.0])
def test_sliced_many_jobs_per_group(groups, T):
    D.set_option("verify_impl", 1)
    # more jobs per group than slots of the partial and decision rings (16) and stages of the
    # copy ring; scheduled rows skipped; labels on and off
    D.set_option("verify_groups", groups)
    B, G, V = 40, 5, 12000
    ld, lt, x, u_acc, u_res = case(B, G, V, T, seed=400 + groups)
    L = (np.arange(B) * 5 % (G + 1)).astype(np.int32)
    for want_c in (True, False):
        for Lc in (L, None):
            n, y, c, fl = run_verify(ld, lt, x, Lc, u_acc, u_res, T, want_c=want_c)
            check_verify(ld, lt, x, Lc, u_acc, u_res, T, n, y, flags_gpu=fl)
            if want_c:
                check_labels(ld, lt, T, c)


@pytest.mark.parametrize("V", [64, 260, 1024, 4100])
def test_sliced_narrow_vocabulary(V):
    # slices of a few quads: tiles of 0 to 2 quads per warp, ragged everywhere
    D.set_option("verify_impl", 1)
    D.set_option("verify_groups", 1)
    B, G = 9, 3
    for T in (1.0, 0.0):
        ld, lt, x, u_acc, u_res = case(B, G, V, T, seed=V + int(T))
        n, y, c, fl = run_verify(ld, lt, x, None, u_acc, u_res, T)
        check_verify(ld, lt, x, None, u_acc, u_res, T, n, y, flags_gpu=fl)
        check_labels(ld, lt, T, c)
