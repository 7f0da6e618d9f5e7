"""gdn_forward_noalloc: the entry point for callers that cannot allocate device
memory while they run the library (plugins whose host framework owns all device
memory, streaming loops that must never wait on an allocator).  Its one piece
of scratch, the bidirectional arrival counters, lives in a fixed static device
array instead of a stream-ordered allocation.

The test calls it through the C ABI several times in a row (each call reuses
the array the previous one left behind), compares every result with the fp64
oracle on the same seeded inputs, and checks that nothing was allocated: the
library's workspace pool stays empty and torch's allocator sees no change.
One bidirectional case has more CTAs than the GPU has SMs (the writer order is
then decided at run time).  The file is collected last and needs nothing from
the other tests, so it passes alone in a fresh process as well."""
import ctypes

import pytest
import torch

from gated_delta_rule_149_b200 import gdn, gdn_device_status, gdn_workspace_release, gdn_workspace_reserved
from gated_delta_rule_149_b200.inputs import make_custom
from parity_util import TOL, f64, oracle_forward, rel_l2

pytestmark = pytest.mark.gpu


def _cases():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    # the single-CTA kernel runs (dv / 64) x 2 x B*H CTAs for a bidirectional call
    wide_heads = sms // 4 + 1
    return [  # (seed, H, T, bidi)
        (21, 4, 1000, True),
        (22, 3, 333, True),
        (24, wide_heads, 130, True),   # 4 * wide_heads > SM count
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


def test_noalloc_matches_the_oracle_and_allocates_nothing(oracle_mod):
    torch.cuda.set_device(0)
    lib = gdn.load_library()
    stream = torch.cuda.current_stream()
    runs = []
    for seed, H, T, bidi in _cases():
        inp = make_custom(1, H, T, 128, 128, dtype="bf16", seed=seed, bidi=bidi, state0=True)
        o_ref, s_ref = oracle_forward(oracle_mod, inp, bidi)
        d = {n: getattr(inp, n).cuda() for n in ("q", "k", "v", "beta", "decay", "state0")}
        o = torch.full(inp.v.shape, float("nan"), dtype=inp.v.dtype, device="cuda")
        s = torch.full(s_ref.shape, float("nan"), dtype=torch.float32, device="cuda")
        runs.append((d, o_ref, s_ref, o, s, bidi))
    torch.cuda.synchronize()
    gdn_workspace_release()
    assert gdn_workspace_reserved() == 0
    before = torch.cuda.memory_allocated()
    for d, _, _, o, s, bidi in runs:          # the entry point, call after call
        _noalloc(lib, d, o, s, bidi, stream)
    gdn_device_status()
    assert gdn_workspace_reserved() == 0, "the allocation-free entry point reserved workspace"
    assert torch.cuda.memory_allocated() == before
    for d, o_ref, s_ref, o, s, bidi in runs:
        e_o, e_s = rel_l2(f64(o), o_ref), rel_l2(f64(s), s_ref)
        assert e_o <= TOL["bf16"], f"o rel-L2 {e_o:.3e} (H={d['q'].shape[1]}, bidi={bidi})"
        assert e_s <= TOL["bf16"], f"state rel-L2 {e_s:.3e} (H={d['q'].shape[1]}, bidi={bidi})"
