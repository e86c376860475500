"""The stored tiny-workload fixture still matches the (pinned) oracle."""
import json
import os

import numpy as np

import oracle as O
from speculative_decoding_04_b200 import inputs

HERE = os.path.dirname(os.path.abspath(__file__))


def test_tiny_fixture_matches_oracle():
    with open(os.path.join(HERE, "golden", "tiny_round.json")) as f:
        g = json.load(f)
    wl = inputs.TINY
    d = inputs.full_inputs(wl)
    x, ld, _ = O.markov_draft(d["U"], d["W1"], d["W2"], d["x0"], d["u_draft"], wl.T)
    assert x.tolist() == g["x"]
    assert abs(float(ld.astype(np.float64).sum()) - g["ld_sum"]) < 1e-6
    n_acc, y, _ = O.verify(ld, d["lt"], x, None, d["u_acc"], d["u_res"], wl.T)
    assert n_acc.tolist() == g["n_acc"] and y.tolist() == g["y"]
    np.testing.assert_allclose(O.tv_labels(ld, d["lt"][:, :wl.gamma], wl.T), g["c_star"], rtol=1e-12)
    sch = O.prefix_schedule(d["c"], d["sps"], wl.D_max)
    assert sch["L"].tolist() == g["schedule_L"] and sch["D"] == g["schedule_D"]
