"""GPU parity: the CUDA path, called through the C ABI, against the fp64 oracle
on the same seeded inputs (element by element, rel-L2 over o and states).

Small shapes that span several 64-token chunks plus ragged tails, every mode,
every supported head size, and the edge cases (T = 1, T < 64, state in ==
state out, zero inputs, slow decay)."""
import contextlib

import numpy as np
import pytest
import torch

from gated_delta_rule_149_b200 import gdn, gdn_device_status, gdn_forward, gdn_rollout
from gated_delta_rule_149_b200.inputs import WORKLOADS, make_custom, make_inputs
from parity_util import TOL, assert_finite_bounded, f64, oracle_forward, rel_l2, to_dev

pytestmark = pytest.mark.gpu

# which kernels serve bf16 inputs: the default choice by shape (the pooled
# chunkwise kernel for dk = dv = 128, the single-CTA one otherwise), the
# single-CTA chunkwise kernel for every shape, and the token-by-token
# cross-check kernel
BF16_KERNELS = ["pool", "single", "recurrent"]


@contextlib.contextmanager
def use_kernel(kernel):
    gdn.debug_kernel_select(1 if kernel == "single" else 0)
    try:
        yield kernel == "recurrent"
    finally:
        gdn.debug_kernel_select(0)


def run_gpu(inp, bidi, kernel):
    d = to_dev(inp)
    with use_kernel(kernel) as recurrent:
        o, s = gdn_forward(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"],
                           bidi=bidi, recurrent=recurrent)
        gdn_device_status()
    return f64(o), f64(s)


def check(oracle_mod, inp, bidi, kernel, tol=None):
    tol = tol or TOL[inp.wl.dtype]
    o_ref, s_ref = oracle_forward(oracle_mod, inp, bidi)
    o, s = run_gpu(inp, bidi, kernel)
    assert_finite_bounded(o)
    e_o, e_s = rel_l2(o, o_ref), rel_l2(s, s_ref)
    assert e_o <= tol, f"o rel-L2 {e_o:.3e} > {tol}"
    assert e_s <= tol, f"state rel-L2 {e_s:.3e} > {tol}"
    if bidi:
        for d in range(2):
            e = rel_l2(s[d], s_ref[d])
            assert e <= tol, f"state[{d}] rel-L2 {e:.3e}"
    return e_o, e_s


@pytest.mark.parametrize("T", [1, 5, 63, 64, 65, 200])
@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("bidi", [False, True])
def test_fp32_small(oracle_mod, T, d, bidi):
    inp = make_custom(1, 2, T, d, d, dtype="fp32", seed=T * 7 + d, bidi=bidi, decay_shift=0.0,
                      state0=True)
    check(oracle_mod, inp, bidi, "recurrent")


@pytest.mark.parametrize("dk,dv", [(32, 64), (128, 32), (96, 128)])
def test_fp32_rectangular(oracle_mod, dk, dv):
    inp = make_custom(2, 1, 77, dk, dv, dtype="fp32", seed=dk + dv, state0=True, decay_shift=0.0)
    check(oracle_mod, inp, False, "recurrent")


@pytest.mark.parametrize("kernel", BF16_KERNELS)
@pytest.mark.parametrize("T", [1, 17, 64, 65, 191, 256, 1000])
@pytest.mark.parametrize("bidi", [False, True])
def test_bf16_small(oracle_mod, kernel, T, bidi):
    inp = make_custom(1, 3, T, 128, 128, dtype="bf16", seed=1000 + T, bidi=bidi, state0=True)
    check(oracle_mod, inp, bidi, kernel)


@pytest.mark.parametrize("kernel", BF16_KERNELS)
@pytest.mark.parametrize("dv", [64, 128])
def test_bf16_dv(oracle_mod, kernel, dv):
    inp = make_custom(2, 2, 300, 128, dv, dtype="bf16", seed=dv, state0=True)
    check(oracle_mod, inp, False, kernel)
    check(oracle_mod, inp, True, kernel)


@pytest.mark.parametrize("kernel", BF16_KERNELS)
def test_bf16_slow_decay_long(oracle_mod, kernel):
    """a ~ 0.98 per token: the state carries across many chunks."""
    inp = make_custom(1, 2, 3000, 128, 128, dtype="bf16", seed=5, decay_shift=-4.0, state0=True)
    assert float(inp.decay.mean()) > 0.95
    check(oracle_mod, inp, False, kernel)
    check(oracle_mod, inp, True, kernel)


@pytest.mark.parametrize("kernel", BF16_KERNELS)
def test_bf16_fast_decay(oracle_mod, kernel):
    """a ~ 2^-11 per token in the first 250 tokens, ~0.9 after: the early
    chunks decay by far more than 2^-120 within a half chunk, so the kernel
    cannot split their decay ratios into row and column factors and takes each
    ratio as one exponential; the later chunks take the factorised form."""
    inp = make_custom(1, 2, 500, 128, 128, dtype="bf16", seed=8, decay_shift=8.0, state0=True)
    slow = make_custom(1, 2, 500, 128, 128, dtype="bf16", seed=9, decay_shift=-2.0)
    inp.decay[..., 250:] = slow.decay[..., 250:]
    assert float(inp.decay[..., :250].max()) < 0.05
    check(oracle_mod, inp, False, kernel)
    check(oracle_mod, inp, True, kernel)


@pytest.mark.parametrize("kernel,dv", [("single", 64), ("single", 128), ("pool", 128)])
def test_bf16_bidi_more_ctas_than_sms(oracle_mod, kernel, dv):
    """More scans than fit on the GPU at once.  Single-CTA kernel: 160 CTAs on 148
    SMs, so the order in which the two scans reach an output tile is decided at
    run time instead of in advance.  Pooled kernel: 80 heads (160 chains) run as
    successive launches of as many heads as fit beside the preparation workers."""
    heads = 160 // (2 * (dv // 64)) if kernel == "single" else 80
    inp = make_custom(1, heads, 333, 128, dv, dtype="bf16", seed=11 + dv, bidi=True)
    check(oracle_mod, inp, True, kernel)


@pytest.mark.parametrize("kernel", BF16_KERNELS)
def test_bf16_no_decay_unit_gates(oracle_mod, kernel):
    """a = 1, b = 1: the pure delta rule, the hardest case for carried error."""
    inp = make_custom(1, 2, 500, 128, 128, dtype="bf16", seed=6, state0=True)
    inp.decay.fill_(1.0)
    inp.beta.fill_(1.0)
    check(oracle_mod, inp, False, kernel)


@pytest.mark.parametrize("kernel", BF16_KERNELS)
@pytest.mark.parametrize("bidi", [False, True])
def test_bf16_decay_slightly_above_one(oracle_mod, kernel, bidi):
    # the gates' precondition is decay in (0, 1]; growth up to 1 + 1e-3 per token
    # keeps every within-chunk decay product a normal float and is computed as written
    inp = make_custom(1, 2, 333, 128, 128, dtype="bf16", seed=14, bidi=bidi, state0=True)
    g = torch.Generator().manual_seed(15)
    inp.decay.copy_(1.0 + 1e-3 * torch.rand(inp.decay.shape, generator=g))
    assert float(inp.decay.min()) > 1.0
    check(oracle_mod, inp, bidi, kernel)


@pytest.mark.parametrize("kernel", BF16_KERNELS)
def test_bf16_zero_inputs_keep_zero(kernel):
    inp = make_custom(1, 2, 130, 128, 128, dtype="bf16", seed=7)
    d = to_dev(inp)
    z = torch.zeros_like(d["v"])
    with use_kernel(kernel) as rec:
        o, s = gdn_forward(d["q"], d["k"], z, d["beta"], d["decay"], None, bidi=True, recurrent=rec)
        gdn_device_status()
    assert torch.count_nonzero(o) == 0 and torch.count_nonzero(s) == 0


@pytest.mark.parametrize("kernel", BF16_KERNELS)
def test_state_in_place(oracle_mod, kernel):
    """state_in and state_out may be the same buffer."""
    inp = make_custom(1, 4, 150, 128, 128, dtype="bf16", seed=8, state0=True)
    o_ref, s_ref = oracle_forward(oracle_mod, inp, False)
    d = to_dev(inp)
    st = d["state0"].clone()
    with use_kernel(kernel) as rec:
        o, s = gdn_forward(d["q"], d["k"], d["v"], d["beta"], d["decay"], st, state_out=st, recurrent=rec)
        gdn_device_status()
    assert s.data_ptr() == st.data_ptr()
    assert rel_l2(f64(o), o_ref) <= TOL["bf16"]
    assert rel_l2(f64(st), s_ref) <= TOL["bf16"]


def test_recurrent_fp32_config_causal_small(oracle_mod):
    inp = make_inputs(WORKLOADS["causal_fp32_small"])
    e_o, e_s = check(oracle_mod, inp, False, "recurrent")
    assert e_o < 1e-5 and e_s < 1e-5


@pytest.mark.parametrize("kernel", BF16_KERNELS)
def test_bidi_equals_two_causal_calls(kernel):
    """GPU self-consistency: BIDI = CAUSAL(x) + flip(CAUSAL(flip(x)))."""
    inp = make_custom(1, 3, 333, 128, 128, dtype="bf16", seed=9, bidi=True)
    d = to_dev(inp)
    fl = lambda x: x.flip(2).contiguous()
    with use_kernel(kernel) as rec:
        o_bi, s_bi = gdn_forward(d["q"], d["k"], d["v"], d["beta"], d["decay"], None, bidi=True,
                                 recurrent=rec)
        o_f, s_f = gdn_forward(d["q"], d["k"], d["v"], d["beta"], d["decay"], None, recurrent=rec)
        o_r, s_r = gdn_forward(fl(d["q"]), fl(d["k"]), fl(d["v"]), fl(d["beta"]), fl(d["decay"]), None,
                               recurrent=rec)
        gdn_device_status()
    ref = f64(o_f) + f64(o_r)[:, :, ::-1]
    assert rel_l2(f64(o_bi), ref) < 5e-3
    assert rel_l2(f64(s_bi[0]), f64(s_f)) < 1e-5
    assert rel_l2(f64(s_bi[1]), f64(s_r)) < 1e-5


@pytest.mark.parametrize("kernel", BF16_KERNELS)
def test_rollout_equals_single_call(oracle_mod, kernel):
    """Chunked rollout vs the oracle, and vs one GPU call over the whole sequence."""
    n, Tc = 3, 150
    full = make_custom(1, 2, n * Tc, 128, 128, dtype="bf16", seed=10, state0=True)
    ch = make_custom(1, 2, Tc, 128, 128, dtype="bf16", seed=10, state0=True, n_chunks=n)
    assert torch.equal(ch.q[1], full.q[:, :, Tc:2 * Tc])
    d = to_dev(ch)
    df = to_dev(full)
    with use_kernel(kernel) as rec:
        o, s, cs = gdn_rollout(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"],
                               recurrent=rec, chunk_states=True)
        o1, s1 = gdn_forward(df["q"], df["k"], df["v"], df["beta"], df["decay"], df["state0"],
                             recurrent=rec)
        gdn_device_status()
    o_ref, s_ref, cs_ref = oracle_mod.gdn_rollout(f64(ch.q), f64(ch.k), f64(ch.v), f64(ch.beta),
                                                  f64(ch.decay), f64(ch.state0))
    for c in range(n):
        assert rel_l2(f64(o[c]), o_ref[c]) <= TOL["bf16"]
        assert rel_l2(f64(cs[c]), cs_ref[c]) <= TOL["bf16"]
    assert rel_l2(f64(s), s_ref) <= TOL["bf16"]
    o_cat = torch.cat([o[c] for c in range(n)], dim=2)
    assert rel_l2(f64(o_cat), f64(o1)) < 5e-3
    assert rel_l2(f64(s), f64(s1)) < 1e-3


def test_rollout_without_chunk_states(oracle_mod):
    n, Tc = 4, 40
    ch = make_custom(1, 2, Tc, 64, 64, dtype="fp32", seed=11, state0=True, n_chunks=n,
                     decay_shift=0.0)
    d = to_dev(ch)
    o, s, _ = gdn_rollout(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"],
                          recurrent=True)
    o_ref, s_ref, _ = oracle_mod.gdn_rollout(f64(ch.q), f64(ch.k), f64(ch.v), f64(ch.beta),
                                             f64(ch.decay), f64(ch.state0))
    assert rel_l2(f64(o), o_ref) <= TOL["fp32"]
    assert rel_l2(f64(s), s_ref) <= TOL["fp32"]


def test_host_buffer_entry(oracle_mod):
    inp = make_custom(1, 2, 100, 64, 64, dtype="fp32", seed=12, state0=True, decay_shift=0.0)
    from gated_delta_rule_149_b200 import gdn_forward_host
    pin = lambda t: t.pin_memory()
    o, s = gdn_forward_host(pin(inp.q), pin(inp.k), pin(inp.v), pin(inp.beta), pin(inp.decay),
                            pin(inp.state0))
    o_ref, s_ref = oracle_forward(oracle_mod, inp, False)
    assert rel_l2(f64(o), o_ref) <= TOL["fp32"]
    assert rel_l2(f64(s), s_ref) <= TOL["fp32"]
