"""Pins for the fp64 CPU oracle: results the definition fixes independently.

The pages never print a numeric GDN example (the librediffusion PR #21 page,
"Validation", reports only a ~1e-7 rel-L2 self-check), so the oracle is pinned
by closed forms and brute force instead:

* orthonormal keys: the delta rule's erase term vanishes and the recurrence is
  gated causal linear attention, computed here by an O(T^2) double sum;
* a = b = 1 with orthonormal keys: plain causal linear attention;
* b = 0: the state only decays (product of gates);
* k = v = 0: the same, with any b;
* b = 1 and a unit key: the write overwrites, so S_t k_t = v_t;
* T = 1: the one-token closed form with the dk x dk matrix (I - b k k^T);
* tiny T, d: the full product expansion with explicit dk x dk factors, and an
  exact rational evaluation of the definition;
* bidirectional = forward + re-reversed forward on the reversed sequence;
* a rollout split at arbitrary points = one scan (bitwise);
* the final state is affine in the initial one (the segment transition);
* the frame-block read-out: blocks of one token = the causal scan; one block
  with orthonormal keys = its closed form; tiny cases by brute force;
* the normalised read-out: its closed form with orthonormal keys, z against its
  written-out recurrence, linearity in v, the bidirectional sums;
* fp8 inputs: the E4M3 decoder against the format's fixed codes and torch's
  float8 type for all 256 codes; the fp8 entry = the forward on exact
  dequantised inputs;
* the contraction bound ||H_t|| <= a_t ||H_{t-1}|| + b_t ||v_t|| for unit keys.
Each pin is chosen so that a dropped term, a wrong sign or index, or a
transposed state would fail at least one of them.
"""
from fractions import Fraction

import numpy as np
import pytest

RNG = np.random.default_rng(1234)


def rand_unit(n, d, rng=RNG):
    x = rng.standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def batch(x):
    """[T, ...] -> [1, 1, T, ...]"""
    return np.asarray(x, dtype=np.float64)[None, None]


def orthonormal_rows(n, d, rng=RNG):
    qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    return qm[:n]


# ----------------------------------------------------------------------------
# Reductions to linear attention
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("dk,dv,T", [(8, 5, 8), (16, 16, 11), (32, 7, 32)])
def test_orthonormal_keys_equal_gated_linear_attention(oracle_mod, dk, dv, T):
    k = orthonormal_rows(T, dk)
    q = RNG.standard_normal((T, dk))
    v = RNG.standard_normal((T, dv))
    a = RNG.uniform(0.3, 1.0, T)
    b = RNG.uniform(0.1, 1.0, T)
    o, s = oracle_mod.gdn_forward(batch(q), batch(k), batch(v), batch(b), batch(a))
    # o_t = sum_{s<=t} (prod_{r=s+1..t} a_r) b_s (k_s . q_t) v_s
    ref = np.zeros((T, dv))
    for t in range(T):
        for s_ in range(t + 1):
            ref[t] += np.prod(a[s_ + 1:t + 1]) * b[s_] * (k[s_] @ q[t]) * v[s_]
    np.testing.assert_allclose(o[0, 0], ref, rtol=0, atol=1e-12)
    # final state H = S^T = sum_s (prod_{r>s} a_r) b_s k_s v_s^T
    Href = sum(np.prod(a[s_ + 1:]) * b[s_] * np.outer(k[s_], v[s_]) for s_ in range(T))
    np.testing.assert_allclose(s[0, 0], Href, rtol=0, atol=1e-12)


def test_a1_b1_orthonormal_is_plain_causal_linear_attention(oracle_mod):
    T, dk, dv = 12, 16, 9
    k = orthonormal_rows(T, dk)
    q = RNG.standard_normal((T, dk))
    v = RNG.standard_normal((T, dv))
    o, _ = oracle_mod.gdn_forward(batch(q), batch(k), batch(v), batch(np.ones(T)), batch(np.ones(T)))
    scores = np.tril(q @ k.T)            # [t, s] = q_t . k_s for s <= t
    np.testing.assert_allclose(o[0, 0], scores @ v, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# Gates alone
# ----------------------------------------------------------------------------

def test_beta_zero_only_decays(oracle_mod):
    T, dk, dv = 20, 6, 5
    q = RNG.standard_normal((T, dk))
    k = RNG.standard_normal((T, dk))
    v = RNG.standard_normal((T, dv))
    a = RNG.uniform(0.5, 1.0, T)
    H0 = RNG.standard_normal((dk, dv))
    o, s = oracle_mod.gdn_forward(batch(q), batch(k), batch(v), batch(np.zeros(T)), batch(a),
                                  state_in=batch(H0))
    cum = np.cumprod(a)
    np.testing.assert_allclose(o[0, 0], cum[:, None] * (q @ H0), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(s[0, 0], cum[-1] * H0, rtol=1e-13, atol=1e-15)


def test_zero_kv_decays_state_by_gate_product(oracle_mod):
    T, dk, dv = 17, 4, 6
    q = RNG.standard_normal((T, dk))
    a = RNG.uniform(0.2, 1.0, T)
    b = RNG.uniform(0.0, 1.0, T)
    H0 = RNG.standard_normal((dk, dv))
    o, s = oracle_mod.gdn_forward(batch(q), batch(np.zeros((T, dk))), batch(np.zeros((T, dv))),
                                  batch(b), batch(a), state_in=batch(H0))
    cum = np.cumprod(a)
    np.testing.assert_allclose(o[0, 0], cum[:, None] * (q @ H0), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(s[0, 0], cum[-1] * H0, rtol=1e-13, atol=1e-15)


# ----------------------------------------------------------------------------
# Erase / overwrite
# ----------------------------------------------------------------------------

def test_beta_one_unit_key_overwrites(oracle_mod):
    """With b_t = 1 and |k_t| = 1, S_t k_t = v_t whatever came before.

    Reading it through the output: q_t = k_t gives o_t = S_t k_t = v_t.
    """
    T, dk, dv = 40, 8, 5
    k = rand_unit(T, dk)
    v = RNG.standard_normal((T, dv))
    a = RNG.uniform(0.1, 1.0, T)
    H0 = RNG.standard_normal((dk, dv))
    o, _ = oracle_mod.gdn_forward(batch(k), batch(k), batch(v), batch(np.ones(T)), batch(a),
                                  state_in=batch(H0))
    np.testing.assert_allclose(o[0, 0], v, rtol=0, atol=1e-13)


# ----------------------------------------------------------------------------
# Closed forms with explicit dk x dk factors
# ----------------------------------------------------------------------------

def test_single_token_closed_form(oracle_mod):
    dk, dv = 7, 4
    q, k = RNG.standard_normal(dk), RNG.standard_normal(dk)
    v = RNG.standard_normal(dv)
    a, b = 0.7, 0.45
    H0 = RNG.standard_normal((dk, dv))
    o, s = oracle_mod.gdn_forward(batch(q[None]), batch(k[None]), batch(v[None]),
                                  batch([b]), batch([a]), state_in=batch(H0))
    S0 = H0.T                                      # dv x dk
    S1 = a * S0 @ (np.eye(dk) - b * np.outer(k, k)) + b * np.outer(v, k)
    np.testing.assert_allclose(s[0, 0], S1.T, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(o[0, 0, 0], S1 @ q, rtol=1e-14, atol=1e-14)


def _expansion(q, k, v, a, b, H0):
    """H_T = P_{1..T} H_0 + sum_s P_{s+1..T} b_s k_s v_s^T with
    P_{i..j} = A_j ... A_i, A_t = a_t (I - b_t k_t k_t^T), in the H = S^T frame."""
    T, dk = k.shape
    A = [a[t] * (np.eye(dk) - b[t] * np.outer(k[t], k[t])) for t in range(T)]

    def P(i, j):  # product A_j ... A_i (later tokens on the left); identity if i > j
        m = np.eye(dk)
        for t in range(i, j + 1):
            m = A[t] @ m
        return m

    outs, Hs = [], []
    for t in range(T):
        H = P(0, t) @ H0 + sum(P(s + 1, t) @ (b[s] * np.outer(k[s], v[s])) for s in range(t + 1))
        Hs.append(H)
        outs.append(H.T @ q[t])
    return np.array(outs), Hs[-1]


@pytest.mark.parametrize("T,dk,dv", [(1, 2, 3), (5, 3, 2), (8, 4, 4)])
def test_product_expansion(oracle_mod, T, dk, dv):
    q = RNG.standard_normal((T, dk))
    k = RNG.standard_normal((T, dk))
    v = RNG.standard_normal((T, dv))
    a = RNG.uniform(0.2, 1.0, T)
    b = RNG.uniform(0.0, 1.0, T)
    H0 = RNG.standard_normal((dk, dv))
    o, s = oracle_mod.gdn_forward(batch(q), batch(k), batch(v), batch(b), batch(a),
                                  state_in=batch(H0))
    o_ref, H_ref = _expansion(q, k, v, a, b, H0)
    np.testing.assert_allclose(o[0, 0], o_ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s[0, 0], H_ref, rtol=1e-12, atol=1e-13)


def test_exact_rational_tiny(oracle_mod):
    """The definition evaluated in exact rationals, S dv x dk, T = 3."""
    F = Fraction
    q = [[F(1, 2), F(-1, 3)], [F(2, 5), F(1, 1)], [F(-3, 4), F(1, 6)]]
    k = [[F(3, 5), F(4, 5)], [F(1, 1), F(0)], [F(-1, 2), F(1, 3)]]
    v = [[F(1), F(-2), F(1, 2)], [F(0), F(3, 2), F(-1)], [F(2, 3), F(1, 4), F(5, 7)]]
    a = [F(1, 2), F(9, 10), F(3, 4)]
    b = [F(1, 3), F(1), F(2, 5)]
    S0 = [[F(1, 10), F(-1, 5)], [F(0), F(1, 2)], [F(3, 8), F(1, 16)]]   # dv x dk
    dk, dv = 2, 3
    S = [row[:] for row in S0]
    outs = []
    for t in range(3):
        # S (I - b k k^T): entry (i,j) = sum_m S[i][m] * (delta_mj - b k_m k_j)
        SI = [[sum(S[i][m] * ((1 if m == j else 0) - b[t] * k[t][m] * k[t][j]) for m in range(dk))
               for j in range(dk)] for i in range(dv)]
        S = [[a[t] * SI[i][j] + b[t] * v[t][i] * k[t][j] for j in range(dk)] for i in range(dv)]
        outs.append([sum(S[i][j] * q[t][j] for j in range(dk)) for i in range(dv)])
    fq = np.array(q, dtype=np.float64)
    o, s = oracle_mod.gdn_forward(batch(fq), batch(np.array(k, dtype=float)),
                                  batch(np.array(v, dtype=float)), batch(np.array(b, dtype=float)),
                                  batch(np.array(a, dtype=float)),
                                  state_in=batch(np.array(S0, dtype=float).T))
    np.testing.assert_allclose(o[0, 0], np.array(outs, dtype=float), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(s[0, 0], np.array(S, dtype=float).T, rtol=1e-14, atol=1e-15)


# ----------------------------------------------------------------------------
# Bidirectional and rollout structure
# ----------------------------------------------------------------------------

def _rand_case(B, H, T, dk, dv, rng=RNG):
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, H, T, dv))
    b = rng.uniform(0, 1, (B, H, T))
    a = rng.uniform(0.5, 1, (B, H, T))
    return q, k, v, b, a


def test_bidi_is_forward_plus_rereversed_reverse(oracle_mod):
    q, k, v, b, a = _rand_case(2, 3, 37, 8, 6)
    H0 = RNG.standard_normal((2, 3, 8, 6))
    o_bi, s_bi = oracle_mod.gdn_forward(q, k, v, b, a, state_in=H0, bidi=True)
    o_f, s_f = oracle_mod.gdn_forward(q, k, v, b, a, state_in=H0)
    flip = lambda x: np.ascontiguousarray(x[:, :, ::-1])
    o_r, s_r = oracle_mod.gdn_forward(flip(q), flip(k), flip(v), flip(b), flip(a))
    assert np.array_equal(o_bi, o_f + flip(o_r))
    assert np.array_equal(s_bi[0], s_f) and np.array_equal(s_bi[1], s_r)
    # the two directions really differ (the reverse scan is not a copy)
    assert not np.allclose(o_f, flip(o_r))


@pytest.mark.parametrize("cuts", [[1], [63, 64, 65], [10, 100, 133]])
def test_split_scan_equals_single_scan_bitwise(oracle_mod, cuts):
    T = 200
    q, k, v, b, a = _rand_case(1, 2, T, 8, 5)
    H0 = RNG.standard_normal((1, 2, 8, 5))
    o_full, s_full = oracle_mod.gdn_forward(q, k, v, b, a, state_in=H0)
    state, pieces = H0, []
    edges = [0] + cuts + [T]
    for lo, hi in zip(edges[:-1], edges[1:]):
        sl = lambda x: np.ascontiguousarray(x[:, :, lo:hi])
        o, state = oracle_mod.gdn_forward(sl(q), sl(k), sl(v), sl(b), sl(a), state_in=state)
        pieces.append(o)
    assert np.array_equal(np.concatenate(pieces, axis=2), o_full)
    assert np.array_equal(state, s_full)


def test_state_is_affine_in_the_initial_state(oracle_mod):
    """The segment-parallel scan rests on this: a segment's final state is
    P X + L for any initial state X, where P = prod_t a_t (I - b_t k_t k_t^T)
    (later tokens on the left) is the final state of the same segment run with
    v = 0 from the identity, and L its final state from zero."""
    T, dk, dv = 60, 6, 5
    q = RNG.standard_normal((T, dk))
    k = rand_unit(T, dk)
    v = RNG.standard_normal((T, dv))
    a = RNG.uniform(0.5, 1.0, T)
    b = RNG.uniform(0.0, 1.0, T)
    _, P = oracle_mod.gdn_forward(batch(q), batch(k), batch(np.zeros((T, dk))), batch(b), batch(a),
                                  state_in=batch(np.eye(dk)))
    P_ref = np.eye(dk)
    for t in range(T):
        P_ref = a[t] * (np.eye(dk) - b[t] * np.outer(k[t], k[t])) @ P_ref
    np.testing.assert_allclose(P[0, 0], P_ref, rtol=1e-12, atol=1e-14)
    _, L = oracle_mod.gdn_forward(batch(q), batch(k), batch(v), batch(b), batch(a))
    X = RNG.standard_normal((dk, dv))
    _, F = oracle_mod.gdn_forward(batch(q), batch(k), batch(v), batch(b), batch(a), state_in=batch(X))
    np.testing.assert_allclose(F[0, 0], P_ref @ X + L[0, 0], rtol=1e-11, atol=1e-13)


# ----------------------------------------------------------------------------
# Frame-block causal read-out
# ----------------------------------------------------------------------------

def test_blockcausal_block_one_is_the_causal_scan(oracle_mod):
    """Blocks of one token: every token is read out with its own state."""
    q, k, v, b, a = _rand_case(2, 2, 40, 6, 5)
    H0 = RNG.standard_normal((2, 2, 6, 5))
    o, s = oracle_mod.gdn_forward(q, k, v, b, a, state_in=H0)
    ob, sb = oracle_mod.gdn_forward_blockcausal(q, k, v, b, a, 1, state_in=H0)
    np.testing.assert_allclose(ob, o, rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(sb, s)


def test_blockcausal_one_block_orthonormal_keys_closed_form(oracle_mod):
    """One block over the whole sequence with orthonormal keys: the erase term
    vanishes, the final state is the decayed sum of b_s k_s v_s^T, and every
    token reads it out."""
    T, dk, dv = 12, 16, 5
    k = orthonormal_rows(T, dk)
    q = RNG.standard_normal((T, dk))
    v = RNG.standard_normal((T, dv))
    a = RNG.uniform(0.3, 1.0, T)
    b = RNG.uniform(0.1, 1.0, T)
    Hf = sum(np.prod(a[s_ + 1:]) * b[s_] * np.outer(k[s_], v[s_]) for s_ in range(T))
    o, s = oracle_mod.gdn_forward_blockcausal(batch(q), batch(k), batch(v), batch(b), batch(a), T)
    np.testing.assert_allclose(s[0, 0], Hf, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(o[0, 0], q @ Hf, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("T,block", [(6, 2), (6, 3), (8, 4)])
def test_blockcausal_product_expansion(oracle_mod, T, block):
    """Brute force: every state from the explicit dk x dk product expansion,
    each token read out with the state at the end of its block."""
    dk, dv = 3, 2
    q = RNG.standard_normal((T, dk))
    k = RNG.standard_normal((T, dk))
    v = RNG.standard_normal((T, dv))
    a = RNG.uniform(0.2, 1.0, T)
    b = RNG.uniform(0.0, 1.0, T)
    H0 = RNG.standard_normal((dk, dv))
    states = []
    H = H0
    for t in range(T):
        H = a[t] * (np.eye(dk) - b[t] * np.outer(k[t], k[t])) @ H + b[t] * np.outer(k[t], v[t])
        states.append(H)
    ref = np.array([q[t] @ states[(t // block + 1) * block - 1] for t in range(T)])
    o, s = oracle_mod.gdn_forward_blockcausal(batch(q), batch(k), batch(v), batch(b), batch(a), block,
                                              state_in=batch(H0))
    np.testing.assert_allclose(o[0, 0], ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(s[0, 0], states[-1], rtol=1e-11, atol=1e-12)


# ----------------------------------------------------------------------------
# Normalised read-out (z state)
# ----------------------------------------------------------------------------

def test_normalized_orthonormal_keys_closed_form(oracle_mod):
    """Orthonormal keys: both states are decayed sums (no erase), so
    o_t = sum_s w_ts (k_s.q_t) v_s / (sum_s w_ts (k_s.q_t) + eps) with
    w_ts = b_s prod_{r=s+1..t} a_r, by a double sum."""
    T, dk, dv, eps = 10, 16, 4, 1e-3
    k = orthonormal_rows(T, dk)
    q = np.abs(RNG.standard_normal((T, dk)))
    v = RNG.standard_normal((T, dv))
    a = RNG.uniform(0.3, 1.0, T)
    b = RNG.uniform(0.1, 1.0, T)
    o, s_kv, s_z = oracle_mod.gdn_forward_normalized(batch(q), batch(k), batch(v), batch(b), batch(a), eps=eps)
    ref = np.zeros((T, dv))
    for t in range(T):
        w = [b[s_] * np.prod(a[s_ + 1:t + 1]) * (k[s_] @ q[t]) for s_ in range(t + 1)]
        ref[t] = sum(w[s_] * v[s_] for s_ in range(t + 1)) / (sum(w) + eps)
    np.testing.assert_allclose(o[0, 0], ref, rtol=1e-11, atol=1e-12)
    z_ref = sum(b[s_] * np.prod(a[s_ + 1:]) * k[s_] for s_ in range(T))
    np.testing.assert_allclose(s_z[0, 0], z_ref, rtol=1e-12, atol=1e-13)


def test_normalized_z_is_the_recurrence_with_unit_values(oracle_mod):
    """z against its recurrence written out with the dk x dk factor, from a
    given initial z; and a value scale passes straight through the read-out."""
    T, dk, dv = 9, 5, 3
    q = RNG.standard_normal((T, dk))
    k = rand_unit(T, dk)
    v = RNG.standard_normal((T, dv))
    a = RNG.uniform(0.2, 1.0, T)
    b = RNG.uniform(0.0, 1.0, T)
    z0 = RNG.standard_normal(dk)
    z = z0.copy()
    for t in range(T):
        z = a[t] * (np.eye(dk) - b[t] * np.outer(k[t], k[t])) @ z + b[t] * k[t]
    o, _, s_z = oracle_mod.gdn_forward_normalized(batch(q), batch(k), batch(v), batch(b), batch(a),
                                                   state_z_in=z0[None, None], eps=0.5)
    np.testing.assert_allclose(s_z[0, 0], z, rtol=1e-12, atol=1e-13)
    o3, _, _ = oracle_mod.gdn_forward_normalized(batch(q), batch(k), batch(3 * v), batch(b), batch(a),
                                                 state_z_in=z0[None, None], eps=0.5)
    np.testing.assert_allclose(o3, 3 * o, rtol=1e-12, atol=1e-13)


def test_normalized_bidi_sums_numerators_and_denominators(oracle_mod):
    q, k, v, b, a = _rand_case(1, 2, 30, 6, 4)
    q = np.abs(q)
    eps = 1e-2
    o, s_kv, s_z = oracle_mod.gdn_forward_normalized(q, k, v, b, a, eps=eps, bidi=True)
    num, _ = oracle_mod.gdn_forward(q, k, v, b, a, bidi=True)
    den, _ = oracle_mod.gdn_forward(q, k, np.ones(v.shape[:3] + (1,)), b, a, bidi=True)
    np.testing.assert_array_equal(o, num / (den + eps))
    assert s_z.shape == (2, 1, 2, 6)


# ----------------------------------------------------------------------------
# fp8 (E4M3) inputs
# ----------------------------------------------------------------------------

def test_e4m3_decoder_known_codes(oracle_mod):
    """Codes fixed by the format: 1.0, -2.0, the largest finite value 448, the
    smallest subnormal 2^-9, the largest subnormal 7/8 * 2^-6, 0.5, zero, NaN."""
    codes = [0x38, 0xC0, 0x7E, 0x01, 0x07, 0x30, 0x00, 0x7F, 0xFF]
    ref = [1.0, -2.0, 448.0, 2.0 ** -9, 7 / 8 * 2.0 ** -6, 0.5, 0.0]
    got = oracle_mod.decode_e4m3(codes)
    np.testing.assert_array_equal(got[:7], ref)
    assert np.isnan(got[7]) and np.isnan(got[8])


def test_e4m3_decoder_matches_torch_float8_for_every_code(oracle_mod):
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle_mod.decode_e4m3(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    np.testing.assert_array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])


def test_fp8_forward_is_the_forward_on_dequantised_inputs(oracle_mod):
    """With power-of-two scales the dequantised values are exact, so the fp8
    entry equals gdn_forward on them bitwise; a per-head scale of v scales o."""
    rng = np.random.default_rng(77)
    B, H, T, dk, dv = 1, 2, 20, 8, 4
    q8, k8, v8 = (rng.integers(0, 0x7E, (B, H, T, d), dtype=np.uint8) for d in (dk, dk, dv))
    sq, sk, sv = (np.full((B, H), 2.0 ** -6) for _ in range(3))
    b = rng.uniform(0, 1, (B, H, T))
    a = rng.uniform(0.5, 1, (B, H, T))
    o, s = oracle_mod.gdn_forward_fp8(q8, k8, v8, sq, sk, sv, b, a)
    dq = lambda x: oracle_mod.decode_e4m3(x) * 2.0 ** -6
    o_ref, s_ref = oracle_mod.gdn_forward(dq(q8), dq(k8), dq(v8), b, a)
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(s, s_ref)
    o2, _ = oracle_mod.gdn_forward_fp8(q8, k8, v8, sq, sk, 4 * sv, b, a)
    np.testing.assert_allclose(o2, 4 * o, rtol=1e-12, atol=1e-14)


def test_rollout_entry_equals_single_scan_bitwise(oracle_mod):
    n, Tc = 4, 30
    q, k, v, b, a = _rand_case(1, 3, n * Tc, 6, 4)
    H0 = RNG.standard_normal((1, 3, 6, 4))
    o_full, s_full = oracle_mod.gdn_forward(q, k, v, b, a, state_in=H0)
    cm = lambda x: np.ascontiguousarray(
        x.reshape(x.shape[0], x.shape[1], n, Tc, *x.shape[3:]).transpose(2, 0, 1, 3, *range(4, x.ndim + 1)))
    o, s, cs = oracle_mod.gdn_rollout(cm(q), cm(k), cm(v), cm(b), cm(a), state_in=H0)
    assert np.array_equal(o, cm(o_full))
    assert np.array_equal(s, s_full)
    assert np.array_equal(cs[-1], s_full)


# ----------------------------------------------------------------------------
# Contraction invariant
# ----------------------------------------------------------------------------

def test_contraction_bound_per_token(oracle_mod):
    """Unit keys, b in [0,1], a in (0,1]: ||H_t||_F <= a_t ||H_{t-1}||_F + b_t ||v_t||."""
    T, dk, dv = 60, 8, 6
    q, k, v, b, a = _rand_case(1, 1, T, dk, dv)
    H0 = RNG.standard_normal((1, 1, dk, dv))
    # rollout with one-token chunks exposes every intermediate state
    cm = lambda x: np.ascontiguousarray(np.moveaxis(x, 2, 0)[:, :, :, None])
    _, _, cs = oracle_mod.gdn_rollout(cm(q), cm(k), cm(v), cm(b), cm(a), state_in=H0)
    prev = np.linalg.norm(H0[0, 0])
    for t in range(T):
        cur = np.linalg.norm(cs[t, 0, 0])
        assert cur <= a[0, 0, t] * prev + b[0, 0, t] * np.linalg.norm(v[0, 0, t]) + 1e-12
        prev = cur


def test_threads_do_not_change_bits(oracle_mod):
    q, k, v, b, a = _rand_case(2, 4, 50, 8, 8)
    o1, s1 = oracle_mod.gdn_forward(q, k, v, b, a, bidi=True, n_threads=1)
    o8, s8 = oracle_mod.gdn_forward(q, k, v, b, a, bidi=True, n_threads=8)
    assert np.array_equal(o1, o8) and np.array_equal(s1, s8)


def test_oracle_regression_record(oracle_mod):
    """The oracle still reproduces its committed tiny record (tests/golden)."""
    import json
    import os
    rec = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "oracle_tiny.json")))
    inp = {n: np.array(x) for n, x in rec["inputs"].items()}
    args = [inp[n] for n in ("q", "k", "v", "beta", "decay")]
    o, s = oracle_mod.gdn_forward(*args, state_in=inp["state0"])
    np.testing.assert_allclose(o, np.array(rec["causal"]["o"]), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(s, np.array(rec["causal"]["state"]), rtol=1e-14, atol=1e-15)
    o, s = oracle_mod.gdn_forward(*args, state_in=inp["state0"], bidi=True)
    np.testing.assert_allclose(o, np.array(rec["bidi"]["o"]), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(s, np.array(rec["bidi"]["state"]), rtol=1e-14, atol=1e-15)
