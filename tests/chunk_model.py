"""Chunkwise (C = 64) restatement of the GDN recurrence, in numpy (test-side).

Not the oracle: a step-by-step model of what the chunkwise CUDA kernel
computes, used to check the block algebra (WY/UT form, reverse direction,
ragged tails) against the token oracle on the CPU, and to predict the error
that bf16 operands add.  Shared with nothing on the CUDA side.

Per chunk of C tokens (positions p = 0..C-1 of tokens 64c + p; positions past
T are identity tokens: k = q = v = 0, beta = 0, log decay = 0), in scan order
(forward: p ascending; reverse: p descending), with H the dk x dv state S^T:
  g_p = log a_p,  G_p = sum of g over positions up to p in scan order,
  gamma_p = exp(G_p),  G_end = G at the chunk's last scan position,
  A_ij = b_i exp(G_i - G_j) (k_i . k_j)  if j strictly before i, else 0
  P_ij = exp(G_i - G_j) (q_i . k_j)       if j before or at i, else 0
  T    = (I + A)^-1
  W    = T diag(b gamma) K,   U~ = T diag(b) V
  U    = U~ - W H_prev
  O    = diag(gamma) Q H_prev + P U
  H    = gamma_end H_prev + sum_j exp(G_end - G_j) k_j u_j^T
"""
import numpy as np

C = 64


def bf16_round(x):
    """Round-to-nearest-even to bfloat16, returned as float64."""
    x = np.asarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    u = ((u + rounding) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def _ident(x):
    return np.asarray(x, dtype=np.float64)


def chunk_scan(q, k, v, beta, decay, h0=None, reverse=False, operand_round=None,
               f32=False):
    """One head.  q,k [T,dk]; v [T,dv]; beta, decay [T].  Returns (o [T,dv], H [dk,dv]).

    operand_round: None (exact fp64 model) or a rounding function applied
    where the kernel feeds a tensor-core operand (P, T1, T2, W, gamma*Q, H, U, U-bar).
    f32: round the fp32 intermediates (gates, accumulations) to float32.
    """
    rnd = operand_round or _ident
    f = (lambda x: np.asarray(x, dtype=np.float32).astype(np.float64)) if f32 else _ident
    T, dk = k.shape
    dv = v.shape[1]
    H = np.zeros((dk, dv)) if h0 is None else np.array(h0, dtype=np.float64)
    o = np.zeros((T, dv))
    n_chunks = (T + C - 1) // C
    order = range(n_chunks - 1, -1, -1) if reverse else range(n_chunks)
    for c in order:
        lo = c * C
        n = min(C, T - lo)
        K = np.zeros((C, dk)); Q = np.zeros((C, dk)); V = np.zeros((C, dv))
        b = np.zeros(C); g = np.zeros(C)
        K[:n] = k[lo:lo + n]; Q[:n] = q[lo:lo + n]; V[:n] = v[lo:lo + n]
        b[:n] = beta[lo:lo + n]
        g[:n] = f(np.log(f(decay[lo:lo + n])))
        # logical (scan) order l -> physical position p
        perm = np.arange(C)[::-1] if reverse else np.arange(C)
        G = np.zeros(C)
        acc = 0.0
        for p in perm:
            acc = f(acc + g[p])
            G[p] = acc
        G_end = G[perm[-1]]
        gamma = f(np.exp(G))
        rank = np.empty(C, dtype=int)
        rank[perm] = np.arange(C)           # scan position of each physical p
        before = rank[None, :] < rank[:, None]      # [i, j]: j strictly before i
        upto = rank[None, :] <= rank[:, None]
        E = f(np.exp(np.where(upto, G[:, None] - G[None, :], -np.inf)))
        KK = f(K @ K.T)
        QK = f(Q @ K.T)
        A = f(np.where(before, b[:, None] * E * KK, 0.0))
        P = rnd(np.where(upto, E * QK, 0.0))
        Tm = f(np.linalg.inv(np.eye(C) + A))
        T1 = rnd(Tm * (b * gamma)[None, :])
        T2 = rnd(Tm * b[None, :])
        W = rnd(f(T1 @ K))
        Ut = f(T2 @ V)
        Hb = rnd(H)
        U = f(Ut - W @ Hb)
        gQ = rnd(gamma[:, None] * Q)
        Ur = rnd(U)
        O = f(gQ @ Hb + P @ Ur)
        ebar = f(np.exp(G_end - G))
        Ubar = rnd(ebar[:, None] * U)
        H = f(f(np.exp(G_end)) * H + K.T @ Ubar)
        o[lo:lo + n] = O[:n]
    return o, H


def chunk_forward(q, k, v, beta, decay, state_in=None, bidi=False, **kw):
    """Batch version, [B,H,T,*] layouts, same conventions as the oracle."""
    B, Hh, T, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, Hh, T, dv))
    s = np.zeros(((2,) if bidi else ()) + (B, Hh, dk, dv))
    for bi in range(B):
        for h in range(Hh):
            h0 = None if state_in is None else state_in[bi, h]
            of, sf = chunk_scan(q[bi, h], k[bi, h], v[bi, h], beta[bi, h], decay[bi, h], h0, **kw)
            if bidi:
                orv, sr = chunk_scan(q[bi, h], k[bi, h], v[bi, h], beta[bi, h], decay[bi, h],
                                     None, reverse=True, **kw)
                o[bi, h] = of + orv
                s[0, bi, h], s[1, bi, h] = sf, sr
            else:
                o[bi, h] = of
                s[bi, h] = sf
    return o, s
