"""GPU parity on the five named workloads at their full sizes.

The GPU runs each workload exactly as the benchmark launches it (one call over
the whole batch).  The oracle checks every output and state for the four
smaller workloads, and a sample of whole heads (every token of each sampled
head, both directions, and its two final states) for the 720p bidirectional
one, where a full fp64 run would take minutes."""
import numpy as np
import pytest
import torch

from gated_delta_rule_149_b200 import gdn_device_status, gdn_forward, gdn_rollout
from gated_delta_rule_149_b200.inputs import WORKLOADS, make_inputs
from parity_util import TOL, assert_finite_bounded, f64, oracle_forward, rel_l2, to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

RECURRENT_BF16 = False   # False: the chunkwise tensor-core kernel serves bf16


def _fwd(inp, bidi):
    d = to_dev(inp)
    rec = inp.wl.dtype == "fp32" or RECURRENT_BF16
    o, s = gdn_forward(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"], bidi=bidi,
                       recurrent=rec)
    gdn_device_status()
    return o, s


def test_causal_fp32_small(oracle_mod):
    inp = make_inputs(WORKLOADS["causal_fp32_small"])
    o, s = _fwd(inp, False)
    o_ref, s_ref = oracle_forward(oracle_mod, inp, False)
    assert rel_l2(f64(o), o_ref) <= TOL["fp32"]
    assert rel_l2(f64(s), s_ref) <= TOL["fp32"]


def test_causal_chunk_480p(oracle_mod):
    inp = make_inputs(WORKLOADS["causal_chunk_480p"])
    o, s = _fwd(inp, False)
    o_ref, s_ref = oracle_forward(oracle_mod, inp, False)
    assert_finite_bounded(f64(o))
    assert rel_l2(f64(o), o_ref) <= TOL["bf16"]
    assert rel_l2(f64(s), s_ref) <= TOL["bf16"]


def test_rollout_480p_5x(oracle_mod):
    inp = make_inputs(WORKLOADS["rollout_480p_5x"])
    d = to_dev(inp)
    o, s, cs = gdn_rollout(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"],
                           recurrent=RECURRENT_BF16, chunk_states=True)
    gdn_device_status()
    o_ref, s_ref, cs_ref = oracle_mod.gdn_rollout(f64(inp.q), f64(inp.k), f64(inp.v),
                                                  f64(inp.beta), f64(inp.decay), f64(inp.state0))
    for c in range(inp.wl.n_chunks):
        assert rel_l2(f64(o[c]), o_ref[c]) <= TOL["bf16"], f"chunk {c}"
        assert rel_l2(f64(cs[c]), cs_ref[c]) <= TOL["bf16"], f"chunk {c} state"
    assert rel_l2(f64(s), s_ref) <= TOL["bf16"]


def test_bidi_clip_480p(oracle_mod):
    inp = make_inputs(WORKLOADS["bidi_clip_480p"])
    o, s = _fwd(inp, True)
    o_ref, s_ref = oracle_forward(oracle_mod, inp, True)
    assert rel_l2(f64(o), o_ref) <= TOL["bf16"]
    assert rel_l2(f64(s), s_ref) <= TOL["bf16"]


SAMPLED_HEADS = [0, 13, 17, 31]   # flat b*H + h of the B=2, H=16 batch


def test_bidi_720p_sampled_heads(oracle_mod):
    wl = WORKLOADS["bidi_720p"]
    inp = make_inputs(wl)
    o, s = _fwd(inp, True)
    o = o.reshape(wl.B * wl.H, wl.T, wl.dv)
    s = s.reshape(2, wl.B * wl.H, wl.dk, wl.dv)
    # all outputs finite and bounded (|o_t| <= sum of contraction-bounded terms)
    assert torch.isfinite(o.float()).all()
    assert float(o.float().abs().max()) < 1e3
    sub = make_inputs(wl, heads=SAMPLED_HEADS)
    assert torch.equal(sub.q[0, 1], inp.q.reshape(wl.B * wl.H, wl.T, wl.dk)[SAMPLED_HEADS[1]])
    o_ref, s_ref = oracle_forward(oracle_mod, sub, True)
    for j, hd in enumerate(SAMPLED_HEADS):
        e_o = rel_l2(f64(o[hd]), o_ref[0, j])
        assert e_o <= TOL["bf16"], f"head {hd}: o rel-L2 {e_o:.3e}"
        for d in range(2):
            e_s = rel_l2(f64(s[d, hd]), s_ref[d, 0, j])
            assert e_s <= TOL["bf16"], f"head {hd} dir {d}: state rel-L2 {e_s:.3e}"
