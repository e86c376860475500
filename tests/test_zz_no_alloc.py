"""dspark_verify_noalloc: verification for callers that cannot hand the library device scratch
(for example a serving engine that has reserved nearly all HBM for its KV cache and forbids
further allocation while decoding, or plugin code given raw device pointers but no allocator).
It must give the same results as dspark_verify with a workspace, call after call, although
every call reuses the same fixed scratch array inside the library."""

import numpy as np
import pytest
import torch

from speculative_decoding_04_b200 import dspark as D
from speculative_decoding_04_b200 import inputs
from tests.parity import P_ATOL, P_RTOL, dev, draw_tokens, host, pm

pytestmark = pytest.mark.gpu


def _case(seed, B, G, V, T):
    wl = inputs.SINGLE_USER.with_(name="noalloc", B=B, gamma=G, V=V, T=T, seed=seed)
    ld, lt = inputs.logits(wl)
    u_draft, u_acc, u_res = inputs.uniforms(wl)
    x = draw_tokens(ld, u_draft, T)
    return ld, lt, x, u_acc, u_res


@pytest.mark.parametrize("T", [1.0, 0.0])
def test_noalloc_matches_workspace_verify_twice_in_a_row(T):
    B, G, V = 12, 6, 30000
    L = np.array([6, 0, 3, 5, 1, 6, 2, 4, 6, 6, 0, 1], dtype=np.int32)
    for call, seed in enumerate((21, 22)):   # two calls in a row on the shared scratch
        ld, lt, x, u_acc, u_res = _case(seed, B, G, V, T)
        args = (pm(ld), dev(lt), dev(x), dev(L) if call else None, dev(u_acc), dev(u_res), T)
        n0, y0, c0, f0 = D.verify(*args, want_c_star=True)
        # outputs prepared by the caller: the no-allocation call itself allocates nothing
        n1 = torch.empty(B, dtype=torch.int32, device="cuda")
        y1 = torch.empty((B, G + 1), dtype=torch.int32, device="cuda")
        c1 = torch.empty((B, G), dtype=torch.float32, device="cuda")
        f1 = torch.zeros(B, dtype=torch.int32, device="cuda")
        D.verify_noalloc(*args, n_acc=n1, y_out=y1, c_star=c1, flags=f1)
        torch.cuda.synchronize()
        assert np.array_equal(host(n1), host(n0))
        assert np.array_equal(host(y1), host(y0))
        assert np.array_equal(host(f1), host(f0))
        c0, c1 = host(c0).astype(np.float64), host(c1).astype(np.float64)
        assert np.all(np.abs(c1 - c0) <= P_RTOL * np.abs(c0) + P_ATOL)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    B, G, V = 4097, 1, 64
    ld = torch.zeros((G, B, V), device="cuda")
    lt = torch.zeros((B, G + 1, V), device="cuda")
    x = torch.zeros((B, G), dtype=torch.int32, device="cuda")
    u = torch.zeros((B, G), device="cuda")
    with pytest.raises(D.DsparkError) as e:
        D.verify_noalloc(ld, lt, x, None, u, u[:, 0].contiguous(), 1.0)
    assert e.value.status == D.EINVAL and "4096" in str(e.value)
