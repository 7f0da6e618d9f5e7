"""The seeded input recipe, checked against its stated readings (CPU only):
the workloads' shapes and token counts (latent grids of 30x52 and 45x80
tokens per frame), the gate distributions (beta = sigmoid(N(0,1)); decay =
exp(-softplus(N(0,1) + shift)), per token or constant over each latent frame),
L2-normalised q and k, the initial state's standard deviation 0.02,
determinism, the rollout being one sequence cut into chunks, and sampled heads
being exactly the full draw's heads."""

import pytest
import torch

from gated_delta_rule_149_b200.inputs import WORKLOADS, make_custom, make_inputs


def test_workload_table():
    expect = {  # name: (token*heads per call or rollout, frames x tokens per frame)
        "causal_fp32_small": (512, None),
        "causal_chunk_480p": (74880, (3, 30 * 52)),
        "rollout_480p_5x": (468000, (3, 30 * 52)),
        "bidi_clip_480p": (524160, (21, 30 * 52)),
        "bidi_720p": (2419200, (21, 45 * 80)),
    }
    for name, (th, frames) in expect.items():
        wl = WORKLOADS[name]
        assert wl.token_heads == th
        if frames is not None:
            assert wl.T == frames[0] * frames[1]
    assert WORKLOADS["bidi_720p"].bidi and WORKLOADS["bidi_clip_480p"].bidi
    assert WORKLOADS["rollout_480p_5x"].n_chunks == 5
    assert WORKLOADS["causal_fp32_small"].dtype == "fp32"


def logit(b):
    b = b.double()
    return torch.log(b / (1 - b))


def decay_raw(decay, shift):
    """Inverts decay = exp(-softplus(raw + shift)) in fp64."""
    sp = -torch.log(decay.double())
    return torch.log(torch.expm1(sp)) - shift


def near_standard_normal(x, tol):
    x = x.flatten().double()
    assert abs(float(x.mean())) < tol and abs(float(x.std()) - 1.0) < tol


@pytest.mark.parametrize("per_frame", [False, True])
def test_recipe(per_frame):
    tpf = 500 if per_frame else 0
    inp = make_custom(2, 4, 2000, 64, 32, dtype="bf16", seed=11, decay_shift=2.0, tokens_per_frame=tpf,
                      state0=True)
    assert inp.q.dtype == inp.k.dtype == inp.v.dtype == torch.bfloat16
    assert inp.beta.dtype == inp.decay.dtype == inp.state0.dtype == torch.float32
    assert inp.q.shape == (2, 4, 2000, 64) and inp.v.shape == (2, 4, 2000, 32)
    for x in (inp.q, inp.k):   # unit rows up to the bf16 rounding
        n = x.float().norm(dim=-1)
        assert float((n - 1).abs().max()) < 1e-2
    assert bool(((inp.beta > 0) & (inp.beta < 1)).all()) and bool(((inp.decay > 0) & (inp.decay < 1)).all())
    near_standard_normal(logit(inp.beta), 0.03)
    raw = decay_raw(inp.decay, 2.0)
    if per_frame:
        frames = raw.reshape(2, 4, 4, 500)
        assert float((frames - frames[..., :1]).abs().max()) < 1e-4   # one draw per frame
        near_standard_normal(frames[..., 0], 0.5)                       # 32 draws only
    else:
        near_standard_normal(raw, 0.03)
    assert abs(float(inp.state0.std()) - 0.02) < 0.001 and abs(float(inp.state0.mean())) < 0.001
    v = inp.v.float()
    assert abs(float(v.mean())) < 0.02 and abs(float(v.std()) - 1.0) < 0.02


def test_streaming_workload_draws():
    inp = make_inputs(WORKLOADS["causal_chunk_480p"])
    raw = decay_raw(inp.decay, 2.0).reshape(1, 16, 3, 1560)
    assert float((raw - raw[..., :1]).abs().max()) < 1e-4
    assert abs(float(inp.state0.std()) - 0.02) < 0.0005
    assert make_inputs(WORKLOADS["causal_fp32_small"]).state0 is None


def test_deterministic_and_seeded():
    a = make_custom(1, 2, 300, 32, 32, seed=5, state0=True)
    b = make_custom(1, 2, 300, 32, 32, seed=5, state0=True)
    c = make_custom(1, 2, 300, 32, 32, seed=6, state0=True)
    for n in ("q", "k", "v", "beta", "decay", "state0"):
        assert torch.equal(getattr(a, n), getattr(b, n))
        assert not torch.equal(getattr(a, n), getattr(c, n))


def test_rollout_is_one_sequence_in_chunks():
    roll = make_custom(1, 2, 100, 32, 32, seed=9, n_chunks=3, tokens_per_frame=50, state0=True)
    one = make_custom(1, 2, 300, 32, 32, seed=9, n_chunks=1, tokens_per_frame=50, state0=True)
    for n in ("q", "k", "v", "beta", "decay"):
        r, o = getattr(roll, n), getattr(one, n)
        for c in range(3):
            assert torch.equal(r[c], o[:, :, 100 * c:100 * (c + 1)])
    assert torch.equal(roll.state0, one.state0)


def test_sampled_heads_are_the_full_draws_heads():
    wl = WORKLOADS["causal_fp32_small"]
    full = make_inputs(wl)
    part = make_inputs(wl, heads=[1])
    assert torch.equal(part.q[0, 0], full.q[0, 1]) and torch.equal(part.decay[0, 0], full.decay[0, 1])
