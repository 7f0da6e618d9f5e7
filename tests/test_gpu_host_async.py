"""gdn_forward_host_async: host-buffer calls in flight on two streams at once,
as a streaming loop uses them (chunk i+1 uploads while chunk i runs and
downloads).  Every call's result must equal the oracle within the bf16 bar and
the device entry point's result on the same inputs (same kernel: the states
bit for bit), with no call's staging buffers or outputs mixed with another's;
bidirectional calls included, whose kernels the library runs one after another."""
import pytest
import torch

from gated_delta_rule_149_b200 import gdn_device_status, gdn_forward, gdn_forward_host_async
from gated_delta_rule_149_b200.inputs import make_custom
from parity_util import TOL, f64, oracle_forward, rel_l2, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bidi", [False, True])
def test_two_streams_in_flight(oracle_mod, bidi):
    torch.cuda.set_device(0)
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    calls = []
    for n in range(4):   # different inputs per call, alternating streams
        inp = make_custom(1, 3, 700 + 64 * n, 128, 128, dtype="bf16", seed=80 + n, bidi=bidi, state0=True)
        host = {m: getattr(inp, m).pin_memory() for m in ("q", "k", "v", "beta", "decay", "state0")}
        calls.append((inp, host))
    outs = []
    for n, (inp, h) in enumerate(calls):
        o, s = gdn_forward_host_async(h["q"], h["k"], h["v"], h["beta"], h["decay"], h["state0"], bidi=bidi,
                                      stream=streams[n % 2])
        outs.append((o, s))
    for st in streams:
        st.synchronize()
    gdn_device_status()
    for (inp, _), (o, s) in zip(calls, outs):
        o_ref, s_ref = oracle_forward(oracle_mod, inp, bidi)
        assert rel_l2(f64(o), o_ref) <= TOL["bf16"]
        assert rel_l2(f64(s), s_ref) <= TOL["bf16"]
        d = to_dev(inp)
        o_dev, s_dev = gdn_forward(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"], bidi=bidi)
        torch.cuda.synchronize()
        assert torch.equal(s, s_dev.cpu())
        assert rel_l2(f64(o), f64(o_dev)) <= 1e-3
