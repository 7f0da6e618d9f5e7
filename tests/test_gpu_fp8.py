"""GPU parity of the fp8 (E4M3) entry point (gdn_forward_fp8) against the fp64
oracle on the same codes and scales (oracle.gdn_forward_fp8: the recurrence on
exactly dequantised inputs), element by element (rel-L2): causal and
bidirectional, both value widths, ragged sequence ends, a given state, and a
full-size streaming call.  The codes come from the usual input recipe,
quantised per (batch, head) with scale max|x| / 448."""
import pytest

from gated_delta_rule_149_b200 import gdn_device_status, gdn_forward_fp8
from gated_delta_rule_149_b200.inputs import WORKLOADS, make_custom, make_inputs, quantize_e4m3
from parity_util import TOL, assert_finite_bounded, f64, rel_l2

pytestmark = pytest.mark.gpu


def check(oracle_mod, inp, bidi):
    (q8, sq), (k8, sk), (v8, sv) = (quantize_e4m3(x) for x in (inp.q, inp.k, inp.v))
    o_ref, s_ref = oracle_mod.gdn_forward_fp8(q8.numpy(), k8.numpy(), v8.numpy(), f64(sq), f64(sk), f64(sv),
                                              f64(inp.beta), f64(inp.decay),
                                              state_in=None if inp.state0 is None else f64(inp.state0), bidi=bidi)
    dev = lambda t: None if t is None else t.cuda()
    o, s = gdn_forward_fp8(dev(q8), dev(k8), dev(v8), dev(sq), dev(sk), dev(sv), dev(inp.beta), dev(inp.decay),
                           dev(inp.state0), bidi=bidi)
    gdn_device_status()
    o, s = f64(o), f64(s)
    assert_finite_bounded(o)
    e_o, e_s = rel_l2(o, o_ref), rel_l2(s, s_ref)
    assert e_o <= TOL["bf16"], f"o rel-L2 {e_o:.3e}"
    assert e_s <= TOL["bf16"], f"state rel-L2 {e_s:.3e}"


@pytest.mark.parametrize("T", [64, 257, 1000])
@pytest.mark.parametrize("bidi", [False, True])
def test_fp8_small(oracle_mod, T, bidi):
    check(oracle_mod, make_custom(1, 2, T, 128, 128, dtype="bf16", seed=5000 + T, bidi=bidi, state0=True), bidi)


@pytest.mark.parametrize("dv", [64, 128])
def test_fp8_heads_and_widths(oracle_mod, dv):
    check(oracle_mod, make_custom(2, 3, 300, 128, dv, dtype="bf16", seed=71 + dv, state0=True), False)


def test_fp8_streaming_call_full_size(oracle_mod):
    check(oracle_mod, make_inputs(WORKLOADS["causal_chunk_480p"]), False)
