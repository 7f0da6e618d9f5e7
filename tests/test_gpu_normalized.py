"""GPU parity of the normalised read-out (gdn_forward_normalized) against the
fp64 oracle (oracle.gdn_forward_normalized), element by element (rel-L2), for
o, the kv state and the z state: causal and bidirectional, with and without a
given z state, both value widths, ragged sequence ends.  Normalised linear
attention is used with non-negative (ReLU-featured) queries and keys, which
keeps z.q away from zero; the inputs here take |q| and |k| of the usual recipe
(unit norm and bf16 values unchanged)."""
import numpy as np
import pytest
import torch

from gated_delta_rule_149_b200 import gdn_device_status, gdn_forward_normalized
from gated_delta_rule_149_b200.inputs import make_custom
from parity_util import TOL, assert_finite_bounded, f64, rel_l2

pytestmark = pytest.mark.gpu


def nonneg(inp):
    inp.q = inp.q.abs()
    inp.k = inp.k.abs()
    return inp


def check(oracle_mod, inp, bidi, z0=None, eps=1e-6):
    o_ref, kv_ref, z_ref = oracle_mod.gdn_forward_normalized(
        f64(inp.q), f64(inp.k), f64(inp.v), f64(inp.beta), f64(inp.decay),
        state_in=None if inp.state0 is None else f64(inp.state0),
        state_z_in=None if z0 is None else f64(z0), eps=eps, bidi=bidi)
    dev = lambda t: None if t is None else t.cuda()
    o, kv, z = gdn_forward_normalized(dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.beta), dev(inp.decay),
                                      dev(inp.state0), dev(z0), eps=eps, bidi=bidi)
    gdn_device_status()
    o, kv, z = f64(o), f64(kv), f64(z)
    assert_finite_bounded(o)
    tol = TOL["bf16"]
    for name, x, ref in (("o", o, o_ref), ("state_kv", kv, kv_ref), ("state_z", z, z_ref)):
        e = rel_l2(x, ref)
        assert e <= tol, f"{name} rel-L2 {e:.3e} > {tol} (bidi={bidi})"


@pytest.mark.parametrize("T", [64, 333, 1000])
@pytest.mark.parametrize("bidi", [False, True])
def test_normalized_small(oracle_mod, T, bidi):
    inp = nonneg(make_custom(1, 2, T, 128, 128, dtype="bf16", seed=4000 + T, bidi=bidi, state0=True))
    check(oracle_mod, inp, bidi)


@pytest.mark.parametrize("dv", [64, 128])
def test_normalized_given_z_state(oracle_mod, dv):
    inp = nonneg(make_custom(2, 2, 500, 128, dv, dtype="bf16", seed=61 + dv, state0=True))
    g = torch.Generator().manual_seed(63)
    z0 = torch.rand(2, 2, 128, generator=g) * 0.1
    check(oracle_mod, inp, False, z0=z0)
    check(oracle_mod, inp, True, z0=z0, eps=1e-3)
