"""The oracle's pins catch plausible mistakes (CPU only).

Each case copies ``oracle/kda_oracle.c`` to a temporary directory, plants one
mistake by text substitution (a transposed decay, a read before the write, a
dropped beta, a flipped sign, a wrong gate constant, ...), compiles it, swaps
it in for the real oracle and runs the pins of ``test_oracle.py``.  At least one
pin must fail for every mutant; the real oracle is restored afterwards.
"""
import ctypes
import os
import subprocess

import pytest

import oracle.oracle as ormod
import tests.test_oracle as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "kda_oracle.c")

MUTANTS = {
    "decay_scales_columns": (
        "const double alpha = exp(g[c]);\n        for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= alpha;",
        "for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= exp(g[j % dk]);"),
    "read_before_write": (
        "    /* S = Sbar + beta k (v - vhat)^T. */",
        "    for (int j = 0; j < dv; ++j) o[j] = 0.0;\n"
        "    for (int c = 0; c < dk; ++c) for (int j = 0; j < dv; ++j) o[j] += S[(size_t)c * dv + j] * q[c];\n"
        "    return;\n    /* S = Sbar + beta k (v - vhat)^T. */"),
    "beta_dropped": ("+= beta * k[c] * (v[j] - vhat[j])", "+= k[c] * (v[j] - vhat[j])"),
    "error_sign": ("(v[j] - vhat[j])", "(v[j] + vhat[j])"),
    "gmin_wrong": ("#define KDA_ORACLE_GMIN (-5.0)", "#define KDA_ORACLE_GMIN (-4.0)"),
    "gate_without_exp_A": ("oracle_sigmoid(exp(A[c]) * z[c])", "oracle_sigmoid(A[c] * z[c])"),
    "no_decay": ("const double alpha = exp(g[c]);", "const double alpha = 1.0 + 0.0 * g[c];"),
    "softplus_argument_negated": ("-oracle_softplus(exp(A[c]) * z[c])", "-oracle_softplus(-exp(A[c]) * z[c])"),
    "softplus_without_exp_A": ("-oracle_softplus(exp(A[c]) * z[c])", "-oracle_softplus(A[c] * z[c])"),
    "softplus_without_log": ("+ log1p(exp(-fabs(x)))", "+ exp(-fabs(x))"),
    "vhat_from_old_state": (
        "    /* vhat = Sbar^T k. */",
        "    for (int c = 0; c < dk; ++c) { const double a = exp(g[c]);"
        " for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] /= a; }\n    /* vhat = Sbar^T k. */"),
}

PIN_TESTS = [
    pins.test_gate_range_and_saturation_match_pages,
    pins.test_matches_product_form_and_unrolled_brute_force,
    pins.test_read_after_write_single_token,
    pins.test_alpha_one_reduces_to_delta_rule,
    pins.test_beta_zero_leaves_decayed_state,
    pins.test_decay_scales_rows_scalar_channel_via_lfilter,
    pins.test_per_step_write_identity,
    lambda: pins.test_chunkwise_form_equals_recurrence(16),
    pins.test_softplus_gate_closed_forms,
]


def _build_mutant(tmp_path, name):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert old in src, f"mutation anchor for {name} not found"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new, 1))
    so = tmp_path / f"{name}.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", str(path), "-o", str(so), "-lm"],
                   check=True)
    return str(so)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(tmp_path, name):
    real = ormod._load()
    lib = ctypes.CDLL(_build_mutant(tmp_path, name))
    for fn in ("kda_oracle_prefill", "kda_oracle_decode", "kda_oracle_gate", "kda_oracle_max_threads",
               "kda_oracle_prefill_gate", "kda_oracle_decode_gate", "kda_oracle_gate_kind",
               "kda_oracle_prefill_ckpt"):
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
        getattr(lib, fn).restype = getattr(real, fn).restype
    caught = []
    ormod._lib = lib
    try:
        for t in PIN_TESTS:
            try:
                t()
            except AssertionError:
                caught.append(getattr(t, "__name__", "chunkwise"))
    finally:
        ormod._lib = real
    assert caught, f"no pin caught mutant {name}"
