"""Writes oracle_tiny.json: the f64 oracle's outputs on tiny seeded problems.

Every stored value comes from ``oracle/`` alone (inputs from the seeded
generators of ``workloads.py``).  The file pins the oracle against accidental
change: ``tests/test_oracle_golden.py`` recomputes each case and compares.  A
deliberate change to the oracle's arithmetic regenerates it (run this script)
and says in its commit message which passage of the pages justifies it.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from selective_state_space_14_b200 import workloads as W  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json")


def cases():
    """name -> dict of f64 output arrays, for the tiny problems."""
    res = {}
    p = W.m1_problem(1, 2, 3, 7, io="f32", seed=101, ngroups=1, bias=True, with_h0=True)
    a = oracle.m1_problem_args(p)
    res["m1_fwd"] = oracle.m1_fwd(**a)
    res["m1_bwd"] = oracle.m1_bwd(dout=p.dout.as_f64(), **a)
    m = W.m3_problem(1, 7, 2, 3, 4, ngroups=1, nangles=2, io="f32", seed=102, with_h0=True)
    ma = oracle.m3_problem_args(m)
    res["m3_fwd"] = oracle.m3_fwd(**ma)
    res["m3_bwd"] = oracle.m3_bwd(dout=m.dout.as_f64(), **ma)
    rng = np.random.default_rng(103)
    x = rng.standard_normal((1, 2, 9))
    w = rng.standard_normal((2, 4)) / 2.0
    b = rng.standard_normal(2)
    xs0 = rng.standard_normal((1, 2, 3))
    u, xs = oracle.conv1d_fwd(x, w, bias=b, xs0=xs0)
    res["conv1d_fwd"] = dict(u=u, xs_final=xs)
    res["conv1d_bwd"] = oracle.conv1d_bwd(x, w, rng.standard_normal((1, 2, 9)), bias=b, xs0=xs0)
    q = W.m3disc_problem(1, 5, 2, 3, 8, nangles=2, io="f32", seed=104, A_floor=0.2)
    raw = {k: getattr(q, k).as_f64() for k in ("dd_dt", "dd_a", "trap", "angles", "B_raw",
                                                "C_raw")}
    kw = dict(dt_bias=q.dt_bias.astype(np.float64), A_floor=q.A_floor, eps=q.eps)
    res["m3_discretize"] = oracle.m3_discretize(**raw, **kw)
    g = np.random.default_rng(105)
    up = dict(dalpha=g.standard_normal((1, 5, 2)), dbeta=g.standard_normal((1, 5, 2)),
              dgamma=g.standard_normal((1, 5, 2)), dtheta=g.standard_normal((1, 5, 2, 2)),
              dB=g.standard_normal((1, 5, 1, 8)), dC=g.standard_normal((1, 5, 1, 8)))
    res["m3_discretize_bwd"] = oracle.m3_discretize_bwd(**raw, **up, **kw)
    return res


def main():
    out = {name: {k: {"shape": list(np.shape(v)), "values": [float(f"{e:.17g}") for e in
                                                              np.ravel(v)]}
                  for k, v in r.items() if v is not None}
           for name, r in cases().items()}
    with open(OUT, "w") as f:
        json.dump(out, f, indent=1, sort_keys=True)
        f.write("\n")
    print(f"wrote {OUT}")


if __name__ == "__main__":
    main()
