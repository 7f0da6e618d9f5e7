"""Writes oracle_tiny.json: the fp64 oracle on a tiny seeded case (calls only oracle/)."""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
import oracle  # noqa: E402


def case():
    rng = np.random.default_rng(20260101)
    T, dk, dv = 7, 3, 2
    q = rng.standard_normal((1, 1, T, dk))
    k = rng.standard_normal((1, 1, T, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, 1, T, dv))
    b = rng.uniform(0.1, 0.9, (1, 1, T))
    a = rng.uniform(0.4, 1.0, (1, 1, T))
    s0 = rng.standard_normal((1, 1, dk, dv))
    return q, k, v, b, a, s0


def main():
    q, k, v, b, a, s0 = case()
    o_c, s_c = oracle.gdn_forward(q, k, v, b, a, state_in=s0)
    o_b, s_b = oracle.gdn_forward(q, k, v, b, a, state_in=s0, bidi=True)
    out = {"inputs": {n: x.tolist() for n, x in zip(("q", "k", "v", "beta", "decay", "state0"),
                                                      (q, k, v, b, a, s0))},
           "causal": {"o": o_c.tolist(), "state": s_c.tolist()},
           "bidi": {"o": o_b.tolist(), "state": s_b.tolist()}}
    json.dump(out, open(os.path.join(HERE, "oracle_tiny.json"), "w"), indent=0)


if __name__ == "__main__":
    main()
