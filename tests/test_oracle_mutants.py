"""The oracle's pins catch plausible mistakes.

Each case below plants one mistake in a copy of the oracle's C source (on the
CPU only: a temporary library, never the product), and checks that at least
one pin of tests/test_oracle_pins.py then fails.  The unmodified source must
pass every pin (test_oracle_pins.py checks that)."""
import ctypes
import os
import subprocess
import tempfile

import pytest

import test_oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "gdn_oracle.c")

UPDATE = "*sij = a * (*sij - b * y[i] * kt[j]) + b * vt[i] * kt[j];"
MUTANTS = {
    "decayed write": (UPDATE, "*sij = a * (*sij - b * y[i] * kt[j]) + a * b * vt[i] * kt[j];"),
    "dropped erase": (UPDATE, "*sij = a * *sij + b * vt[i] * kt[j];"),
    "erase sign": (UPDATE, "*sij = a * (*sij + b * y[i] * kt[j]) + b * vt[i] * kt[j];"),
    "dropped decay": (UPDATE, "*sij = (*sij - b * y[i] * kt[j]) + b * vt[i] * kt[j];"),
    "erase uses q": ("acc += S[(size_t)i * dk + j] * kt[j];\n            y[i] = acc;",
                     "acc += S[(size_t)i * dk + j] * qt[j];\n            y[i] = acc;"),
    "output uses k": ("acc += S[(size_t)i * dk + j] * qt[j];\n            if (J->accumulate)",
                      "acc += S[(size_t)i * dk + j] * kt[j];\n            if (J->accumulate)"),
    "reverse not re-reversed": ("double *ot = J->o + (size_t)t * dv;",
                                "double *ot = J->o + (size_t)s * dv;"),
    "state_in not transposed": ("S[(size_t)i * dk + j] = J->h0[(size_t)j * dv + i];",
                                "S[(size_t)i * dk + j] = J->h0[(size_t)i * dk + j];"),
    "state_in in reverse scan": ("J->h0 = (dir == 0 && state_in)", "J->h0 = (state_in)"),
}


def build_mutant(name, tmpdir):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name!r} not found exactly once"
    path_c = os.path.join(tmpdir, "mutant.c")
    path_so = os.path.join(tmpdir, "libmutant.so")
    open(path_c, "w").write(src.replace(old, new))
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-pthread", path_c, "-o", path_so],
                   check=True)
    lib = ctypes.CDLL(path_so)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_gdn_forward.argtypes = [dp] * 8 + [ctypes.c_int] * 7
    lib.oracle_gdn_forward.restype = ctypes.c_int
    lib.oracle_gdn_rollout.argtypes = [dp] * 9 + [ctypes.c_int] * 7
    lib.oracle_gdn_rollout.restype = ctypes.c_int
    return lib


PIN_CALLS = [
    lambda m: pins.test_orthonormal_keys_equal_gated_linear_attention(m, 8, 5, 8),
    lambda m: pins.test_a1_b1_orthonormal_is_plain_causal_linear_attention(m),
    lambda m: pins.test_beta_zero_only_decays(m),
    lambda m: pins.test_zero_kv_decays_state_by_gate_product(m),
    lambda m: pins.test_beta_one_unit_key_overwrites(m),
    lambda m: pins.test_single_token_closed_form(m),
    lambda m: pins.test_product_expansion(m, 5, 3, 2),
    lambda m: pins.test_exact_rational_tiny(m),
    lambda m: pins.test_bidi_is_forward_plus_rereversed_reverse(m),
    lambda m: pins.test_split_scan_equals_single_scan_bitwise(m, [63, 64, 65]),
    lambda m: pins.test_contraction_bound_per_token(m),
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(oracle_mod, name):
    import oracle.oracle as oo
    with tempfile.TemporaryDirectory() as tmp:
        lib = build_mutant(name, tmp)
        saved = oo._lib
        oo._lib = lib
        failed = []
        try:
            for k, call in enumerate(PIN_CALLS):
                try:
                    call(oracle_mod)
                except AssertionError:
                    failed.append(k)
        finally:
            oo._lib = saved
    assert failed, f"no pin catches the mutant {name!r}"
