"""ctypes wrapper around the fp64 C oracle (test infrastructure only).

Inputs are numpy arrays in the library's layouts; they are converted to
contiguous float64 before the call, and results come back as float64.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_gdn_forward.argtypes = [dp] * 8 + [ctypes.c_int] * 7
        lib.oracle_gdn_forward.restype = ctypes.c_int
        lib.oracle_gdn_rollout.argtypes = [dp] * 9 + [ctypes.c_int] * 7
        lib.oracle_gdn_rollout.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(x):
    if x is None:
        return None
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads():
    return max(1, os.cpu_count() or 1)


def gdn_forward(q, k, v, beta, decay, state_in=None, bidi=False, n_threads=None):
    """q,k [B,H,T,dk]; v [B,H,T,dv]; beta, decay [B,H,T]; state_in [B,H,dk,dv] or None.

    Returns (o [B,H,T,dv], state_out [B,H,dk,dv] causal or [2,B,H,dk,dv] bidi).
    """
    q, k, v, beta, decay = map(_f64, (q, k, v, beta, decay))
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and v.shape[:3] == (B, H, T)
    assert beta.shape == (B, H, T) and decay.shape == (B, H, T)
    s_in = None if state_in is None else _f64(state_in)
    if s_in is not None:
        assert s_in.shape == (B, H, dk, dv)
    o = np.zeros((B, H, T, dv), dtype=np.float64)
    s_out = np.zeros(((2,) if bidi else ()) + (B, H, dk, dv), dtype=np.float64)
    rc = load().oracle_gdn_forward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(decay), _ptr(s_in), _ptr(s_out),
        _ptr(o), B, H, T, dk, dv, 1 if bidi else 0, n_threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_gdn_forward failed ({rc})")
    return o, s_out


def gdn_rollout(q, k, v, beta, decay, state_in=None, n_threads=None):
    """Chunk-major inputs q,k [n,B,H,Tc,dk]; v [n,B,H,Tc,dv]; gates [n,B,H,Tc].

    Returns (o [n,B,H,Tc,dv], state_out [B,H,dk,dv], chunk_states [n,B,H,dk,dv]).
    """
    q, k, v, beta, decay = map(_f64, (q, k, v, beta, decay))
    n, B, H, Tc, dk = q.shape
    dv = v.shape[-1]
    s_in = None if state_in is None else _f64(state_in)
    o = np.zeros((n, B, H, Tc, dv), dtype=np.float64)
    s_out = np.zeros((B, H, dk, dv), dtype=np.float64)
    cs = np.zeros((n, B, H, dk, dv), dtype=np.float64)
    rc = load().oracle_gdn_rollout(
        _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(decay), _ptr(s_in), _ptr(s_out),
        _ptr(cs), _ptr(o), B, H, n, Tc, dk, dv, n_threads or default_threads())
    if rc != 0:
        raise RuntimeError(f"oracle_gdn_rollout failed ({rc})")
    return o, s_out, cs


def gdn_forward_blockcausal(q, k, v, beta, decay, block, state_in=None, n_threads=None):
    """Frame-block causal read-out (test infrastructure only).

    Reading (the LongSANA page, "PR feature": a causal linear-attention KV
    cache carried across video chunks; here every token of a frame sees its
    whole frame and every earlier frame): the state runs token by token as in
    gdn_forward, and every token t of block f (tokens [f*block, (f+1)*block))
    is read out with the state after the whole block:
        o_t = H_{(f+1)*block - 1}^T q_t.
    q,k [B,H,T,dk], v [B,H,T,dv], gates [B,H,T]; T a multiple of block.
    Returns (o [B,H,T,dv], final state [B,H,dk,dv]).  The state after each
    block comes from the token-by-token scan, run block by block with the
    state carried (bitwise the single scan); the read-out is a matrix product.
    """
    q, k, v, beta, decay = map(_f64, (q, k, v, beta, decay))
    B, H, T, dk = q.shape
    assert block >= 1 and T % block == 0
    state = None if state_in is None else _f64(state_in)
    o = np.zeros(v.shape, dtype=np.float64)
    for f in range(T // block):
        sl = slice(f * block, (f + 1) * block)
        cut = lambda x: np.ascontiguousarray(x[:, :, sl])
        _, state = gdn_forward(cut(q), cut(k), cut(v), cut(beta), cut(decay), state_in=state,
                               n_threads=n_threads)
        o[:, :, sl] = np.einsum("bhtk,bhkv->bhtv", q[:, :, sl], state)
    return o, state


def gdn_forward_normalized(q, k, v, beta, decay, state_in=None, state_z_in=None, eps=1e-6,
                           bidi=False, n_threads=None):
    """Normalised read-out with a z state (test infrastructure only).

    Reading (the librediffusion PR #21 review names a state_z next to
    state_kv in its bidirectional kernel, with no formula): z is the same
    gated delta recurrence driven by a constant value of 1,
        z_t = a_t (I - b_t k_t k_t^T) z_{t-1} + b_t k_t,
    and o_t = (S_t q_t) / (z_t . q_t + eps).  Bidirectional: numerators and
    denominators are each summed over the two scan directions (as gdn_forward
    sums o), then divided.  z runs token by token through the same oracle scan
    with a one-column value of ones.
    Returns (o [B,H,T,dv], state_kv, state_z [B,H,dk] (bidi: [2,B,H,dk])).
    """
    q, k, v, beta, decay = map(_f64, (q, k, v, beta, decay))
    B, H, T, dk = q.shape
    num, s_kv = gdn_forward(q, k, v, beta, decay, state_in=state_in, bidi=bidi, n_threads=n_threads)
    ones = np.ones((B, H, T, 1))
    z_in = None if state_z_in is None else _f64(state_z_in)[..., None]
    den, s_z = gdn_forward(q, k, ones, beta, decay, state_in=z_in, bidi=bidi, n_threads=n_threads)
    return num / (den + eps), s_kv, s_z[..., 0]


def decode_e4m3(codes):
    """fp8 E4M3 bytes -> float64 (test infrastructure only), from the format's
    definition: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits;
    exponent field 0 holds subnormals m/8 * 2^-6; S.1111.111 is NaN (no
    infinities); the largest finite value is 448."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 0xF) & (m == 7), np.nan, val)
    return sign * val


def gdn_forward_fp8(q8, k8, v8, q_scale, k_scale, v_scale, beta, decay, state_in=None, bidi=False,
                    n_threads=None):
    """fp8 (E4M3) q, k, v with one fp32 scale per (batch, head) (test
    infrastructure only): the inputs are x = scale * decode(x8), exactly, and
    the recurrence is gdn_forward on them."""
    deq = lambda x8, s: decode_e4m3(x8) * np.asarray(s, dtype=np.float64)[:, :, None, None]
    return gdn_forward(deq(q8, q_scale), deq(k8, k_scale), deq(v8, v_scale), beta, decay,
                       state_in=state_in, bidi=bidi, n_threads=n_threads)
