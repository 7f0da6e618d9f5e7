"""The library's workspace pool: scratch reserved by one call stays reserved
across a synchronise (so the next call maps nothing), calls of the same shape
reuse it without growing it, and gdn_workspace_release hands it back, after
which calls reserve again and give the same results."""
import pytest
import torch

from gated_delta_rule_149_b200 import (gdn_device_status, gdn_forward, gdn_forward_fp8,
                                       gdn_workspace_release, gdn_workspace_reserved)
from gated_delta_rule_149_b200.inputs import make_custom, quantize_e4m3
from parity_util import f64, rel_l2, to_dev

pytestmark = pytest.mark.gpu


def test_pool_keeps_reuses_and_releases():
    torch.cuda.set_device(0)
    inp = make_custom(1, 4, 1000, 128, 128, dtype="bf16", seed=61, bidi=True, state0=True)
    d = to_dev(inp)
    (q8, sq), (k8, sk), (v8, sv) = (quantize_e4m3(x) for x in (inp.q, inp.k, inp.v))
    q8, k8, v8, sq, sk, sv = (t.cuda() for t in (q8, k8, v8, sq, sk, sv))

    def call():
        o1, s1 = gdn_forward(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"], bidi=True)
        o2, s2 = gdn_forward_fp8(q8, k8, v8, sq, sk, sv, d["beta"], d["decay"], d["state0"], bidi=True)
        gdn_device_status()
        return o1, s1, o2, s2

    first = call()
    torch.cuda.synchronize()
    held = gdn_workspace_reserved()
    # the fp8 call alone needs its three bf16 copies: 2 B * 4 heads * 1000 tokens * 384
    assert held >= 2 * 4 * 1000 * (128 + 128 + 128)
    for _ in range(3):
        call()
        torch.cuda.synchronize()
        assert gdn_workspace_reserved() == held   # kept across synchronise, not grown

    gdn_workspace_release()
    assert gdn_workspace_reserved() == 0
    again = call()
    assert gdn_workspace_reserved() > 0
    for a, b in zip(first, again):
        assert rel_l2(f64(b), f64(a)) <= 1e-3
    # the states do not depend on the order of the two directions' output adds
    assert torch.equal(first[1], again[1]) and torch.equal(first[3], again[3])
