"""The benchmark's in-run parity check on CPU: its head sampling, reshapes and
rel-L2 against the oracle.  Fed the oracle's own full result (as fp32, the
form a GPU result has) it must pass; a mistake planted in a sampled head of
that result must fail it.  Planted mistakes live here, on the CPU side only."""
import argparse

import numpy as np
import torch

import bench
import oracle
from gated_delta_rule_149_b200.inputs import make_custom


def full_oracle(inp, bidi):
    f = lambda t: t.double().numpy()
    return oracle.gdn_forward(f(inp.q), f(inp.k), f(inp.v), f(inp.beta), f(inp.decay),
                              None if inp.state0 is None else f(inp.state0), bidi=bidi)


def test_sampled_parity_passes_on_the_oracle_and_catches_a_planted_error(oracle_mod):
    args = argparse.Namespace(normalized=False, block=0)
    for bidi in (False, True):
        inp = make_custom(2, 3, 130, 32, 32, dtype="fp32", seed=5, bidi=bidi, state0=True)
        o_ref, s_ref = full_oracle(inp, bidi)
        o_dev, s_dev = torch.from_numpy(o_ref).float(), torch.from_numpy(s_ref).float()
        r = bench.sampled_parity(args, inp.wl, inp, o_dev, s_dev)
        assert r["checked"] and r["pass"], r
        assert r["rel_l2_o"] < 1e-6 and r["rel_l2_state"] < 1e-6

        bad = o_dev.clone()
        bad[1, 2, 7] += 10.0                        # the last head is sampled
        assert not bench.sampled_parity(args, inp.wl, inp, bad, s_dev)["pass"]
        bad_s = s_dev.clone()
        if bidi:
            bad_s[1, 0, 0] *= -1.0                  # the first head's reverse-scan state
        else:
            bad_s[0, 0] *= -1.0
        assert not bench.sampled_parity(args, inp.wl, inp, o_dev, bad_s)["pass"]


def test_normalised_read_out_is_reported_unchecked():
    args = argparse.Namespace(normalized=True, block=0)
    inp = make_custom(1, 2, 64, 32, 32, dtype="fp32", seed=6)
    r = bench.sampled_parity(args, inp.wl, inp, None, None)
    assert r["checked"] is False and r["why"]


def test_fp8_and_frame_block_forms(oracle_mod):
    from gated_delta_rule_149_b200.inputs import quantize_e4m3
    f = lambda t: t.double().numpy()
    inp = make_custom(1, 2, 128, 32, 32, dtype="bf16", seed=7, bidi=True, state0=True)
    (q8, sq), (k8, sk), (v8, sv) = (quantize_e4m3(x) for x in (inp.q, inp.k, inp.v))
    o_ref, s_ref = oracle.gdn_forward_fp8(q8.numpy(), k8.numpy(), v8.numpy(), f(sq), f(sk), f(sv), f(inp.beta),
                                          f(inp.decay), state_in=f(inp.state0), bidi=True)
    args = argparse.Namespace(normalized=False, block=0)
    r = bench.sampled_parity(args, inp.wl, inp, torch.from_numpy(o_ref).float(), torch.from_numpy(s_ref).float(),
                             fp8=(q8, k8, v8, sq, sk, sv))
    assert r["pass"] and r["rel_l2_o"] < 1e-6, r
    # the same result checked as a plain bf16 call fails: the check uses the fp8 definition
    assert bench.sampled_parity(args, inp.wl, inp, torch.from_numpy(o_ref).float(),
                                torch.from_numpy(s_ref).float())["rel_l2_o"] > 1e-3

    inp = make_custom(1, 2, 120, 32, 32, dtype="fp32", seed=8, state0=True)
    o_ref, s_ref = oracle.gdn_forward_blockcausal(f(inp.q), f(inp.k), f(inp.v), f(inp.beta), f(inp.decay), 40,
                                                  state_in=f(inp.state0))
    args = argparse.Namespace(normalized=False, block=40)
    r = bench.sampled_parity(args, inp.wl, inp, torch.from_numpy(o_ref).float(), torch.from_numpy(s_ref).float())
    assert r["pass"], r


def test_algorithmic_bytes_and_source_hash():
    import bench
    from gated_delta_rule_149_b200.inputs import WORKLOADS
    wl = WORKLOADS["bidi_720p"]
    b16, b8 = bench.algorithmic_bytes(wl), bench.algorithmic_bytes(wl, fp8=True)
    # bf16: 2 directions x ((2 dk + dv) x 2 B + 8 B of gates) + dv x 2 B of o, per token-head, plus states
    states = wl.B * wl.H * wl.dk * wl.dv * 4 * 2
    assert b16 == wl.B * wl.H * wl.T * (2 * ((2 * 128 + 128) * 2 + 8) + 128 * 2) + states
    # fp8 codes: q, k, v at one byte, o still bf16
    assert b16 - b8 == wl.B * wl.H * wl.T * 2 * (2 * 128 + 128)
    # the hash covers the kernel that ran, and ignores comments
    assert bench.kernel_source_sha("pool") != bench.kernel_source_sha("single")
    assert bench.kernel_source_sha("pool") == bench.kernel_source_sha("pool")
