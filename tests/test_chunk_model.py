"""The chunkwise algebra the CUDA kernel implements, checked against the token
oracle on the CPU: exact in fp64 (up to rounding), and within the bf16
tolerance when tensor-core operands are rounded to bf16 as in the kernel."""
import numpy as np
import pytest

from chunk_model import bf16_round, chunk_forward
from gated_delta_rule_149_b200.inputs import make_custom
from parity_util import f64, rel_l2


def _case(T, dk, dv, seed, bidi, shift=2.0, state0=True, dtype="fp32"):
    inp = make_custom(1, 2, T, dk, dv, dtype=dtype, seed=seed, bidi=bidi, decay_shift=shift,
                      state0=state0)
    return [f64(x) for x in (inp.q, inp.k, inp.v, inp.beta, inp.decay)], f64(inp.state0)


@pytest.mark.parametrize("T", [1, 63, 64, 65, 130, 200])
@pytest.mark.parametrize("bidi", [False, True])
def test_chunk_algebra_exact(oracle_mod, T, bidi):
    (q, k, v, b, a), s0 = _case(T, 16, 8, T, bidi, shift=-1.0)
    o_ref, s_ref = oracle_mod.gdn_forward(q, k, v, b, a, state_in=s0, bidi=bidi)
    o, s = chunk_forward(q, k, v, b, a, state_in=s0, bidi=bidi)
    assert rel_l2(o, o_ref) < 1e-11 and rel_l2(s, s_ref) < 1e-11


@pytest.mark.parametrize("shift", [2.0, -4.0])
def test_chunk_algebra_bf16_operands_within_tolerance(oracle_mod, shift):
    (q, k, v, b, a), s0 = _case(300, 128, 64, 3, True, shift=shift, dtype="bf16")
    o_ref, s_ref = oracle_mod.gdn_forward(q, k, v, b, a, state_in=s0, bidi=True)
    o, s = chunk_forward(q, k, v, b, a, state_in=s0, bidi=True, operand_round=bf16_round, f32=True)
    e_o, e_s = rel_l2(bf16_round(o), o_ref), rel_l2(s, s_ref)
    assert e_o < 5e-3 and e_s < 5e-3, (e_o, e_s)
