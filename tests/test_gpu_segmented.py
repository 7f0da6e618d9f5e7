"""GPU parity of the segment-parallel causal scan (gdn_forward_segmented)
against the fp64 oracle, element by element (rel-L2), and against the plain
chunkwise call: the segmented result is the same causal scan, so both must meet
the bf16 bar against the oracle.  Covers ragged sequence ends, segment counts
that do and do not divide the chunk count, one and two segments (plain call),
more segments than chunks, a given initial state, both value widths, several
heads, and the streaming workloads at full size."""
import numpy as np
import pytest

from gated_delta_rule_149_b200 import gdn_device_status, gdn_forward, gdn_forward_segmented
from gated_delta_rule_149_b200.inputs import WORKLOADS, make_custom, make_inputs
from parity_util import TOL, assert_finite_bounded, f64, oracle_forward, rel_l2, to_dev

pytestmark = pytest.mark.gpu


def run_segmented(inp, n_segments):
    d = to_dev(inp)
    o, s = gdn_forward_segmented(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"],
                                 n_segments=n_segments)
    gdn_device_status()
    return f64(o), f64(s)


def check(oracle_mod, inp, n_segments, ref=None):
    o_ref, s_ref = ref if ref is not None else oracle_forward(oracle_mod, inp, False)
    o, s = run_segmented(inp, n_segments)
    assert_finite_bounded(o)
    e_o, e_s = rel_l2(o, o_ref), rel_l2(s, s_ref)
    tol = TOL[inp.wl.dtype]
    assert e_o <= tol, f"o rel-L2 {e_o:.3e} > {tol} (n_segments={n_segments})"
    assert e_s <= tol, f"state rel-L2 {e_s:.3e} > {tol} (n_segments={n_segments})"
    return e_o, e_s


@pytest.mark.parametrize("T", [200, 1000, 1601])
@pytest.mark.parametrize("n_segments", [1, 2, 3, 4, 7])
def test_segmented_small(oracle_mod, T, n_segments):
    inp = make_custom(1, 2, T, 128, 128, dtype="bf16", seed=2000 + T, state0=True)
    check(oracle_mod, inp, n_segments)


@pytest.mark.parametrize("dv", [64, 128])
def test_segmented_heads_and_widths(oracle_mod, dv):
    inp = make_custom(2, 3, 800, 128, dv, dtype="bf16", seed=31 + dv, state0=True,
                      tokens_per_frame=100)
    check(oracle_mod, inp, 5)


def test_segmented_zero_state_and_more_segments_than_chunks(oracle_mod):
    inp = make_custom(1, 2, 300, 128, 128, dtype="bf16", seed=41)   # 5 chunks
    ref = oracle_forward(oracle_mod, inp, False)
    for n in (5, 9, 100):
        check(oracle_mod, inp, n, ref)


def test_segmented_slow_decay_carries_state_across_segments(oracle_mod):
    """a ~ 0.98 per token: the state entering late segments depends strongly on
    early ones, so a wrong transition or combine would show."""
    inp = make_custom(1, 2, 3000, 128, 128, dtype="bf16", seed=43, decay_shift=-4.0, state0=True)
    assert float(inp.decay.mean()) > 0.95
    check(oracle_mod, inp, 6)


def test_segmented_matches_plain_call():
    inp = make_custom(1, 4, 2000, 128, 128, dtype="bf16", seed=47, state0=True)
    d = to_dev(inp)
    o1, s1 = gdn_forward(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"])
    o2, s2 = gdn_forward_segmented(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"],
                                   n_segments=5)
    gdn_device_status()
    assert rel_l2(f64(o2), f64(o1)) < 5e-3
    assert rel_l2(f64(s2), f64(s1)) < 5e-3


@pytest.mark.parametrize("name", ["causal_chunk_480p", "rollout_480p_5x"])
def test_segmented_streaming_workloads_full_size(oracle_mod, name):
    """The streaming workloads' calls (3 latent frames of 30x52 tokens, 16 and
    20 heads) at full size, with the segment count the benchmark uses."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl)
    if wl.n_chunks > 1:   # rollout: its first chunk is one such call
        inp = make_custom(wl.B, wl.H, wl.T, wl.dk, wl.dv, dtype=wl.dtype, seed=wl.seed,
                          tokens_per_frame=wl.tokens_per_frame, decay_shift=wl.decay_shift,
                          state0=True)
    check(oracle_mod, inp, 5)
