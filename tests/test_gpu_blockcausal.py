"""GPU parity of the frame-block causal read-out (gdn_forward_blockcausal)
against the fp64 oracle (oracle.gdn_forward_blockcausal), element by element
(rel-L2): blocks of one chunk, of ragged chunk counts (frames of 100 and 1560
tokens, not multiples of 64), a single block, one-token blocks, a given
initial state, both value widths, several heads, slow decay, and the 480p
streaming workload at full size with its latent frames as blocks."""
import pytest

from gated_delta_rule_149_b200 import gdn_device_status, gdn_forward, gdn_forward_blockcausal
from gated_delta_rule_149_b200.inputs import WORKLOADS, make_custom, make_inputs
from parity_util import TOL, assert_finite_bounded, f64, rel_l2, to_dev

pytestmark = pytest.mark.gpu


def check(oracle_mod, inp, block):
    o_ref, s_ref = oracle_mod.gdn_forward_blockcausal(
        f64(inp.q), f64(inp.k), f64(inp.v), f64(inp.beta), f64(inp.decay), block,
        state_in=None if inp.state0 is None else f64(inp.state0))
    d = to_dev(inp)
    o, s = gdn_forward_blockcausal(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"], block=block)
    gdn_device_status()
    o, s = f64(o), f64(s)
    assert_finite_bounded(o)
    tol = TOL[inp.wl.dtype]
    e_o, e_s = rel_l2(o, o_ref), rel_l2(s, s_ref)
    assert e_o <= tol, f"o rel-L2 {e_o:.3e} > {tol} (block={block})"
    assert e_s <= tol, f"state rel-L2 {e_s:.3e} > {tol} (block={block})"


@pytest.mark.parametrize("T,block", [(640, 64), (600, 100), (600, 600), (256, 128), (1200, 300)])
def test_blockcausal_small(oracle_mod, T, block):
    inp = make_custom(1, 2, T, 128, 128, dtype="bf16", seed=3000 + T + block, state0=True)
    check(oracle_mod, inp, block)


@pytest.mark.parametrize("dv", [64, 128])
def test_blockcausal_heads_and_widths(oracle_mod, dv):
    inp = make_custom(2, 3, 500, 128, dv, dtype="bf16", seed=51 + dv, tokens_per_frame=100)
    check(oracle_mod, inp, 100)


def test_blockcausal_one_token_blocks_is_the_causal_scan(oracle_mod):
    inp = make_custom(1, 2, 96, 128, 128, dtype="bf16", seed=57, state0=True)
    check(oracle_mod, inp, 1)
    d = to_dev(inp)
    o1, s1 = gdn_forward(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"])
    o2, s2 = gdn_forward_blockcausal(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"], block=1)
    gdn_device_status()
    assert rel_l2(f64(o2), f64(o1)) < 5e-3
    assert rel_l2(f64(s2), f64(s1)) < 5e-3


def test_blockcausal_slow_decay(oracle_mod):
    inp = make_custom(1, 2, 2000, 128, 128, dtype="bf16", seed=59, decay_shift=-4.0, state0=True)
    check(oracle_mod, inp, 250)


def test_blockcausal_streaming_workload_full_size(oracle_mod):
    """causal_chunk_480p (3 latent frames of 30x52 tokens, 16 heads), frames as blocks."""
    wl = WORKLOADS["causal_chunk_480p"]
    check(oracle_mod, make_inputs(wl), wl.tokens_per_frame)
