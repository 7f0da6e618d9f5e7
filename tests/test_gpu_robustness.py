"""Bounded device waits and co-residency of the chunkwise kernels.

1. A wait that runs out: with the wait limit lowered to 50 ms and scan 0's
   state chain of the pooled kernel told to wait for a slot sequence value
   nothing writes, the kernel records a timeout in the device error word and
   returns (no hang); gdn_device_status reports GDN_ERR_DEVICE_TIMEOUT, and the
   next normal call on the same context matches the oracle.  Causal and
   bidirectional bf16 calls, and a causal fp8 call (the fp8 instantiation).
2. Co-residency: the kernels whose CTAs wait for one another are launched
   cooperatively, so a call made while another stream keeps every SM busy with
   matrix products still finishes correctly (no wait runs out), and so do the
   products.
"""
import time

import pytest
import torch

from gated_delta_rule_149_b200 import gdn, gdn_device_status, gdn_forward, gdn_forward_fp8
from gated_delta_rule_149_b200.gdn import GDNError
from gated_delta_rule_149_b200.inputs import make_custom, quantize_e4m3
from parity_util import TOL, f64, oracle_forward, rel_l2, to_dev

pytestmark = pytest.mark.gpu

GDN_ERR_DEVICE_TIMEOUT = -5


def _check_parity(oracle_mod, inp, bidi, o, s):
    o_ref, s_ref = oracle_forward(oracle_mod, inp, bidi)
    e_o, e_s = rel_l2(f64(o), o_ref), rel_l2(f64(s), s_ref)
    assert e_o <= TOL["bf16"], f"o rel-L2 {e_o:.3e}"
    assert e_s <= TOL["bf16"], f"state rel-L2 {e_s:.3e}"


@pytest.mark.parametrize("bidi,fp8", [(False, False), (True, False), (False, True)])
def test_wait_runs_out_and_the_next_call_is_correct(oracle_mod, bidi, fp8):
    torch.cuda.set_device(0)
    inp = make_custom(1, 2, 1024, 128, 128, dtype="bf16", seed=31, bidi=bidi, state0=True)
    d = to_dev(inp)
    gdn_device_status()   # start from a clear error word
    gdn.debug_wait_limit(50_000_000)
    gdn.debug_stall(3)
    try:
        t0 = time.perf_counter()
        if fp8:   # the fp8 instantiation (its code widening runs in both CTA kinds)
            codes = [quantize_e4m3(x) for x in (inp.q, inp.k, inp.v)]
            gdn_forward_fp8(*(c.cuda() for c, _ in codes), *(sc.cuda() for _, sc in codes), d["beta"],
                            d["decay"], d["state0"])
        else:
            gdn_forward(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"], bidi=bidi)
        with pytest.raises(GDNError) as err:
            gdn_device_status()
        elapsed = time.perf_counter() - t0
    finally:
        gdn.debug_stall(-1)
        gdn.debug_wait_limit(0)
    assert err.value.code == GDN_ERR_DEVICE_TIMEOUT
    assert elapsed < 20.0, f"the aborted call took {elapsed:.1f} s"
    gdn_device_status()   # cleared by the read above
    o, s = gdn_forward(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"], bidi=bidi)
    gdn_device_status()
    _check_parity(oracle_mod, inp, bidi, o, s)


@pytest.mark.parametrize("kernel,dv", [("pool", 128), ("single", 64)])
def test_cooperative_call_beside_a_busy_stream(oracle_mod, kernel, dv):
    torch.cuda.set_device(0)
    inp = make_custom(1, 4, 4000, 128, dv, dtype="bf16", seed=32, bidi=True, state0=True)
    d = to_dev(inp)
    g = torch.Generator(device="cuda").manual_seed(5)
    a = torch.randn(4096, 4096, device="cuda", dtype=torch.bfloat16, generator=g)
    b = torch.randn(4096, 4096, device="cuda", dtype=torch.bfloat16, generator=g)
    ref = a @ b
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    outs = []
    gdn.debug_kernel_select(1 if kernel == "single" else 0)
    try:
        with torch.cuda.stream(side):
            for _ in range(40):           # tens of milliseconds of products on every SM
                outs.append(a @ b)
        o, s = gdn_forward(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"], bidi=True)
        gdn_device_status()
    finally:
        gdn.debug_kernel_select(0)
    torch.cuda.synchronize()
    _check_parity(oracle_mod, inp, True, o, s)
    for c in outs:
        assert torch.equal(c, ref)
