"""Write tests/golden/tiny_round.json from the oracle alone.

The pages print no numeric worked example of the round, so the stored values
here are regression fixtures of the oracle (which is pinned separately by
tests/test_oracle_pins.py).  This script imports only the oracle and the
seeded input generator.  Run from the repository root:

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
from speculative_decoding_04_b200 import inputs  # noqa: E402


def main():
    wl = inputs.TINY
    d = inputs.full_inputs(wl)
    x, ld, alts = O.markov_draft(d["U"], d["W1"], d["W2"], d["x0"], d["u_draft"], wl.T)
    n_acc, y, _ = O.verify(ld, d["lt"], x, None, d["u_acc"], d["u_res"], wl.T)
    c_star = O.tv_labels(ld, d["lt"][:, :wl.gamma], wl.T)
    sch = O.prefix_schedule(d["c"], d["sps"], wl.D_max, O.SCHED_ARGMAX)
    n_s, y_s, _ = O.verify(ld, d["lt"], x, sch["L"], d["u_acc"], d["u_res"], wl.T)
    out = {
        "workload": "tiny: B=2, gamma=4, V=1024, r=16, T=1.0, fp32 weights, seed 0",
        "source": "oracle (tests/golden/make_golden.py)",
        "x": x.tolist(),
        "ld_sum": float(ld.astype(np.float64).sum()),
        "n_acc": n_acc.tolist(),
        "y": y.tolist(),
        "c_star": c_star.tolist(),
        "schedule_L": sch["L"].tolist(),
        "schedule_theta": sch["theta"],
        "schedule_D": sch["D"],
        "scheduled_n_acc": n_s.tolist(),
        "scheduled_y": y_s.tolist(),
        "near_ties": len(alts),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_round.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
