"""Helpers shared by the GPU parity tests (test-side only)."""
import numpy as np
import torch

# rel-L2 tolerances: fp32 inputs 1e-5, bf16 inputs (fp32 state) 1e-2.
TOL = {"fp32": 1e-5, "bf16": 1e-2}


def rel_l2(x, ref):
    """||x - ref||_2 / ||ref||_2 over the flattened tensors, accumulated in fp64
    (the metric the librediffusion PR #21 page, "Validation", argues for)."""
    x = np.asarray(x, dtype=np.float64).ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    den = np.linalg.norm(ref)
    num = np.linalg.norm(x - ref)
    if den == 0.0:
        return float(num)
    return float(num / den)


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def to_dev(inp, device="cuda"):
    out = {}
    for name in ("q", "k", "v", "beta", "decay", "state0"):
        t = getattr(inp, name)
        out[name] = None if t is None else t.to(device)
    return out


def oracle_forward(oracle_mod, inp, bidi):
    return oracle_mod.gdn_forward(f64(inp.q), f64(inp.k), f64(inp.v), f64(inp.beta),
                                  f64(inp.decay),
                                  None if inp.state0 is None else f64(inp.state0), bidi=bidi)


def assert_finite_bounded(o, bound=1e6):
    o = np.asarray(o)
    assert np.isfinite(o).all(), "non-finite values"
    assert np.abs(o).max() < bound
