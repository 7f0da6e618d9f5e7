"""gdn_forward_noalloc: the entry point for callers that cannot allocate device
memory while they run the library (plugins whose host framework owns all device
memory, streaming loops that must never wait on an allocator).  Its one piece
of scratch, the bidirectional arrival counters, lives in a fixed static device
array instead of a stream-ordered allocation.

The test calls it through the C ABI twice in a row (the second call reuses the
array the first one left behind) and checks each result against gdn_forward on
the same inputs.  It lives in its own file, collected last, and needs nothing
from the other tests, so it passes alone in a fresh process as well."""
import ctypes

import pytest
import torch

from gated_delta_rule_149_b200 import gdn, gdn_device_status, gdn_forward
from gated_delta_rule_149_b200.inputs import make_custom
from parity_util import TOL, f64, rel_l2

pytestmark = pytest.mark.gpu

CASES = [  # (seed, H, T, bidi): two bidirectional calls of different shapes, then a causal one
    (21, 4, 1000, True),
    (22, 3, 333, True),
    (23, 2, 200, False),
]


def _noalloc(lib, d, o, s_out, bidi, stream):
    B, H, T, dk = d["q"].shape
    dv = d["v"].shape[-1]
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    rc = lib.gdn_forward_noalloc(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["beta"]),
                                 ptr(d["decay"]), ptr(d["state0"]), ptr(s_out), ptr(o),
                                 B, H, T, dk, dv, 1 if bidi else 0,
                                 ctypes.c_void_p(stream.cuda_stream))
    assert rc == 0, lib.gdn_last_error().decode()


def test_noalloc_matches_gdn_forward_on_calls_in_a_row():
    torch.cuda.set_device(0)
    lib = gdn.load_library()
    stream = torch.cuda.current_stream()
    runs = []
    for seed, H, T, bidi in CASES:
        inp = make_custom(1, H, T, 128, 128, dtype="bf16", seed=seed, bidi=bidi, state0=True)
        d = {n: getattr(inp, n).cuda() for n in ("q", "k", "v", "beta", "decay", "state0")}
        o_ref, s_ref = gdn_forward(d["q"], d["k"], d["v"], d["beta"], d["decay"], d["state0"],
                                   bidi=bidi)
        o = torch.full_like(o_ref, float("nan"))
        s = torch.full_like(s_ref, float("nan"))
        runs.append((d, o_ref, s_ref, o, s, bidi))
    torch.cuda.synchronize()
    for d, _, _, o, s, bidi in runs:          # the entry point, call after call
        _noalloc(lib, d, o, s, bidi, stream)
    gdn_device_status()
    for d, o_ref, s_ref, o, s, bidi in runs:
        assert rel_l2(f64(o), f64(o_ref)) <= TOL["bf16"]
        assert rel_l2(f64(s), f64(s_ref)) <= TOL["bf16"]
        # same kernel, same inputs: the states are bit-identical, the outputs
        # differ at most by which direction's partial was rounded first
        assert torch.equal(s, s_ref)
        assert rel_l2(f64(o), f64(o_ref)) < 5e-3
