"""Seeded synthetic inputs for the GDN recurrence (shared by tests, bench, smoke).

This module draws random numbers and shapes them like the pages' video-latent
workloads; it holds none of the recurrence's arithmetic.  Every tensor is made
on the CPU with a ``torch.Generator`` seeded per workload, in this fixed draw
order: q, k, v, beta_raw, decay_raw, state0.

Recipe (all draws N(0, 1) in fp32 unless stated):
  * q, k  -> L2-normalised per token (no epsilon), then cast to the input dtype
             (bf16 with round-to-nearest-even, or kept fp32);
  * v     -> cast to the input dtype;
  * beta  =  sigmoid(beta_raw), per token and head, fp32;
  * decay =  exp(-softplus(decay_raw + shift)), fp32, drawn per token or per
             latent frame; a per-frame value is repeated for every token of the
             frame (the gates stay per token at the library boundary);
  * state0 = 0.02 * N(0, 1) (standard deviation 0.02) or absent (zero state).

Token counts follow the latent grids of the pages' clips: 480x832 video gives
30x52 = 1560 latent tokens per frame, 720p gives 45x80 = 3600.
"""
from dataclasses import dataclass, field
from typing import Optional

import torch


@dataclass
class Workload:
    name: str
    B: int
    H: int
    T: int                      # tokens per call (per chunk for a rollout)
    dk: int
    dv: int
    dtype: str                  # "bf16" or "fp32"
    bidi: bool = False
    n_chunks: int = 1           # > 1: streaming rollout of n_chunks causal chunks
    tokens_per_frame: int = 0   # > 0: decay drawn per frame
    decay_shift: float = 0.0
    state0: bool = False
    seed: int = 0
    note: str = ""

    @property
    def token_heads(self) -> int:
        return self.B * self.H * self.T * self.n_chunks


# The five workloads the benchmark and the parity tests use.
WORKLOADS = {
    "causal_fp32_small": Workload(
        "causal_fp32_small", B=1, H=2, T=256, dk=32, dv=32, dtype="fp32",
        note="4 frames x 8x8 tokens, gates per token, zero state"),
    "causal_chunk_480p": Workload(
        "causal_chunk_480p", B=1, H=16, T=4680, dk=128, dv=128, dtype="bf16",
        tokens_per_frame=1560, decay_shift=2.0, state0=True,
        note="3 latent frames x 30x52 tokens, decay per frame, state0 std 0.02"),
    "rollout_480p_5x": Workload(
        "rollout_480p_5x", B=1, H=20, T=4680, dk=128, dv=128, dtype="bf16",
        n_chunks=5, tokens_per_frame=1560, decay_shift=2.0, state0=True,
        note="5 causal chunks of 3 frames x 1560 tokens, state carried"),
    "bidi_clip_480p": Workload(
        "bidi_clip_480p", B=1, H=16, T=32760, dk=128, dv=128, dtype="bf16", bidi=True,
        decay_shift=2.0, note="21 latent frames x 1560 tokens, gates per token"),
    "bidi_720p": Workload(
        "bidi_720p", B=2, H=16, T=75600, dk=128, dv=128, dtype="bf16", bidi=True,
        tokens_per_frame=3600, decay_shift=2.0,
        note="21 latent frames x 45x80 tokens, decay per frame, beta per token"),
}


@dataclass
class GDNInputs:
    wl: Workload
    q: torch.Tensor             # [B,H,T,dk] (rollout: [n,B,H,Tc,dk])
    k: torch.Tensor
    v: torch.Tensor             # [.., dv]
    beta: torch.Tensor          # [B,H,T] fp32 (rollout: [n,B,H,Tc])
    decay: torch.Tensor         # same shape as beta
    state0: Optional[torch.Tensor] = None   # [B,H,dk,dv] fp32
    extra: dict = field(default_factory=dict)


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def _l2norm_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


def make_inputs(wl: Workload, heads: Optional[list] = None) -> GDNInputs:
    """Draws the workload's tensors on the CPU.

    For a rollout one sequence of n_chunks*T tokens is drawn and sliced into
    chunk-major tensors, so the chunked run can be compared with a single scan.
    ``heads`` (a list of flat b*H+h indices) keeps only those heads after the
    full draw, so a sampled check sees exactly the full run's values.
    """
    g = torch.Generator(device="cpu").manual_seed(wl.seed)
    B, H, dk, dv = wl.B, wl.H, wl.dk, wl.dv
    T = wl.T * wl.n_chunks
    dt = torch_dtype(wl.dtype)

    q = _l2norm_rows(torch.randn(B, H, T, dk, generator=g)).to(dt)
    k = _l2norm_rows(torch.randn(B, H, T, dk, generator=g)).to(dt)
    v = torch.randn(B, H, T, dv, generator=g).to(dt)
    beta = torch.sigmoid(torch.randn(B, H, T, generator=g))
    if wl.tokens_per_frame > 0:
        assert T % wl.tokens_per_frame == 0
        n_frames = T // wl.tokens_per_frame
        raw = torch.randn(B, H, n_frames, generator=g)
        decay = torch.exp(-torch.nn.functional.softplus(raw + wl.decay_shift))
        decay = decay.repeat_interleave(wl.tokens_per_frame, dim=-1)
    else:
        raw = torch.randn(B, H, T, generator=g)
        decay = torch.exp(-torch.nn.functional.softplus(raw + wl.decay_shift))
    state0 = (0.02 * torch.randn(B, H, dk, dv, generator=g)) if wl.state0 else None

    if heads is not None:
        idx = torch.as_tensor(heads, dtype=torch.long)

        def pick(x):
            return x.reshape(B * H, *x.shape[2:])[idx].unsqueeze(0).contiguous()
        q, k, v, beta, decay = map(pick, (q, k, v, beta, decay))
        if state0 is not None:
            state0 = pick(state0)

    if wl.n_chunks > 1:
        n, Tc = wl.n_chunks, wl.T

        def chunks(x):  # [B,H,n*Tc,...] -> [n,B,H,Tc,...]
            Bx, Hx = x.shape[0], x.shape[1]
            y = x.reshape(Bx, Hx, n, Tc, *x.shape[3:])
            perm = (2, 0, 1, 3) + tuple(range(4, y.dim()))
            return y.permute(*perm).contiguous()
        q, k, v, beta, decay = map(chunks, (q, k, v, beta, decay))

    return GDNInputs(wl, q.contiguous(), k.contiguous(), v.contiguous(),
                     beta.contiguous(), decay.contiguous(),
                     None if state0 is None else state0.contiguous())


def make_custom(B, H, T, dk, dv, dtype="bf16", seed=0, bidi=False, decay_shift=2.0,
                tokens_per_frame=0, state0=False, n_chunks=1) -> GDNInputs:
    """Same recipe for an arbitrary shape (parity sweeps and edge cases)."""
    wl = Workload(f"custom_B{B}H{H}T{T}dk{dk}dv{dv}{dtype}", B=B, H=H, T=T, dk=dk, dv=dv,
                  dtype=dtype, bidi=bidi, n_chunks=n_chunks,
                  tokens_per_frame=tokens_per_frame, decay_shift=decay_shift,
                  state0=state0, seed=seed)
    return make_inputs(wl)


def quantize_e4m3(x: torch.Tensor):
    """Per-(batch, head) scaled fp8 E4M3 codes of a [B,H,T,d] tensor: scale =
    max|x| / 448 over the head (1 for an all-zero head), codes = the nearest
    E4M3 value of x / scale.  Returns (uint8 codes, fp32 scales [B,H])."""
    xf = x.to(torch.float32)
    amax = xf.abs().amax(dim=(2, 3))
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    codes = (xf / scale[:, :, None, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()
