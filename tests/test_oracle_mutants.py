"""The oracle's pins are strong enough: each plausible mistake planted in a copy
of the oracle's C source (a dropped term, a wrong sign or index, swapped
operands) makes at least one pin fail.  CPU only; the mistakes are planted in
temporary copies, never in the committed oracle.
"""
import os
import subprocess
import tempfile

import pytest

import oracle
import test_oracle_backward_pins as bpins
import test_oracle_mimo_pins as mpins
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "ssd_oracle.c")

MUTANTS = {
    "transition sign": ("const double a = exp(dt * j->A[h]);", "const double a = exp(-dt * j->A[h]);"),
    "dropped D skip": ("const double yv = acc + j->D[h] * xt[p];", "const double yv = acc;"),
    "reversed conv taps": ("acc += w[k] * v;", "acc += w[3 - k] * v;"),
    "reversed conv history": ("else v = hist ? hist[s + 3] : 0.0;", "else v = hist ? hist[-s - 1] : 0.0;"),
    "wrong head->group map": ("const int g = h / (H / G);\n    const long cx",
                              "const int g = h % G;\n    const long cx"),
    "B and C swapped": ("Sp[n] = a * Sp[n] + dt * xt[p] * Bt[n];\n                acc += Sp[n] * Ct[n];",
                        "Sp[n] = a * Sp[n] + dt * xt[p] * Ct[n];\n                acc += Sp[n] * Bt[n];"),
    "read-out before update": ("Sp[n] = a * Sp[n] + dt * xt[p] * Bt[n];\n                acc += Sp[n] * Ct[n];",
                               "acc += Sp[n] * Ct[n];\n                Sp[n] = a * Sp[n] + dt * xt[p] * Bt[n];"),
    "missing dt bias": ("j->dt_raw[((size_t)b * L + t) * H + h] + j->dt_bias[h]",
                        "j->dt_raw[((size_t)b * L + t) * H + h]"),
    "input not scaled by dt": ("Sp[n] = a * Sp[n] + dt * xt[p] * Bt[n];", "Sp[n] = a * Sp[n] + xt[p] * Bt[n];"),
    "ungated output": ("= yv * o_silu(zv);", "= yv * zv;"),
    "conv bias dropped": ("double acc = b;", "double acc = 0.0;"),
    "decode roll stale": ("cs[0] = win[1];", "cs[0] = win[0];"),
    "decode missing D": ("const double yv = acc + D[h] * xt[p];", "const double yv = acc;"),
    "decode wrong B group": ("const double* Bt = u + HP + (size_t)g * N;", "const double* Bt = u + HP;"),
    "softplus branch wrong": ("if (v > 30.0) return v + log1p(exp(-v));", "if (v > 0.0) return v;"),
}

# mistakes in the backward (the adjoint recurrence and the conv backward)
BACKWARD_MUTANTS = {
    "adjoint not decayed": ("for (int i2 = 0; i2 < P * N; i2++) lam[i2] *= av[t];",
                            "for (int i2 = 0; i2 < P * N; i2++) lam[i2] *= 1.0;"),
    "read-out adjoint after the decay": ("lam[p * N + n] += g_[p] * Ct[n];", "lam[p * N + n] += 0.0 * Ct[n];"),
    "dC from the previous state": ("duC[t * N + n] += g_[p] * St[p * N + n];",
                                   "duC[t * N + n] += g_[p] * Sprev[p * N + n];"),
    "dB without dt": ("duB[t * N + n] += dtv[t] * xt[p] * lam[p * N + n];",
                      "duB[t * N + n] += xt[p] * lam[p * N + n];"),
    "decay term of ddt dropped": ("ddt[t] += dxB + lamS * av[t] * j->A[h];", "ddt[t] += dxB;"),
    "dA without dt": ("dA_h += lamS * av[t] * dtv[t];", "dA_h += lamS * av[t];"),
    "softplus derivative missing": ("const double v = ddt[t] * o_sigmoid(j->dt_raw[i] + j->dt_bias[h]);",
                                    "const double v = ddt[t];"),
    "silu derivative wrong": ("return s * (1.0 + v * (1.0 - s));", "return s;"),
    "gate gradient ungated": ("g_[p] = j->dy[yi] * o_silu(zv);", "g_[p] = j->dy[yi];"),
    "D skip gradient dropped": ("dux[t * P + p] += j->D[h] * g_[p];", "dux[t * P + p] += 0.0 * g_[p];"),
    "conv taps not flipped": ("long t = s + 3 - k;\n            if (t >= 0 && t < L) acc += w[k] * dv[t];",
                              "long t = s + k;\n            if (t >= 0 && t < L) acc += w[k] * dv[t];"),
    "conv bias gradient dropped": ("*db += dv[t];", "*db += 0.0;"),
    "history gradient misplaced": ("else if (d_hist) d_hist[s + 3] = acc;", "else if (d_hist) d_hist[-s - 1] = acc;"),
    "checkpoint off by one": ("if (t % RECOMP_SEG == 0) memcpy(", "if (t % RECOMP_SEG == 1) memcpy("),
}

# mistakes in the MIMO decode step
MIMO_MUTANTS = {
    "MIMO input from slot 0's B": ("in += xh[k * P + p] * Bg[k * N + n];", "in += xh[k * P + p] * Bg[n];"),
    "MIMO read-out from slot 0's C": ("acc += S[(size_t)p * N + n] * Cg[k * N + n];",
                                      "acc += S[(size_t)p * N + n] * Cg[n];"),
    "MIMO D skip from slot 0": ("const double yv = acc + D[h] * xh[k * P + p];", "const double yv = acc + D[h] * xh[p];"),
    "MIMO gate from slot 0": ("yv * o_silu(zh[k * P + p]);", "yv * o_silu(zh[p]);"),
    "MIMO input not scaled by dt": ("S[(size_t)p * N + n] = a * S[(size_t)p * N + n] + dt * in;",
                                    "S[(size_t)p * N + n] = a * S[(size_t)p * N + n] + in;"),
    "MIMO decay squared": ("S[(size_t)p * N + n] = a * S[(size_t)p * N + n] + dt * in;",
                           "S[(size_t)p * N + n] = a * a * S[(size_t)p * N + n] + dt * in;"),
}

PINS = [
    lambda: pins.test_conv_silu_matches_library_fir(True),
    lambda: pins.test_prefill_matches_quadratic_form(1, True),
    lambda: pins.test_prefill_quadratic_form_bf16_inputs_groups_of_three(),
    lambda: pins.test_closed_form_constant_inputs(-1.2, -2.5),
    lambda: pins.test_closed_form_constant_inputs(0.8, -0.6),
    lambda: pins.test_closed_form_constant_inputs(35.0, -0.01),
    lambda: pins.test_decode_steps_reproduce_prefill(True),
]


def _compile(src_text, out_dir, name):
    c = os.path.join(out_dir, name + ".c")
    so = os.path.join(out_dir, name + ".so")
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O1", "-shared", "-fPIC", "-pthread", "-o", so, c, "-lm"])
    return so


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for '{name}' not unique"
    with tempfile.TemporaryDirectory() as tmp:
        so = _compile(src.replace(old, new), tmp, "mutant")
        oracle.use_library(so)
        try:
            failed = 0
            for pin in PINS:
                try:
                    pin()
                except AssertionError:
                    failed += 1
            assert failed > 0, f"no pin caught the planted mistake '{name}'"
        finally:
            oracle.use_library(None)


def test_unmutated_copy_passes_every_pin():
    with tempfile.TemporaryDirectory() as tmp:
        so = _compile(open(SRC).read(), tmp, "clean")
        oracle.use_library(so)
        try:
            for pin in PINS + BACKWARD_PINS + MIMO_PINS:
                pin()
        finally:
            oracle.use_library(None)


BACKWARD_PINS = [
    lambda: bpins.test_directional_finite_differences(True, True),
    lambda: bpins.test_elementwise_finite_differences_of_parameters(),
    lambda: bpins.test_segment_recomputation_boundary(),
]


@pytest.mark.parametrize("name", sorted(BACKWARD_MUTANTS))
def test_planted_backward_mistake_is_caught(name):
    src = open(SRC).read()
    old, new = BACKWARD_MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for '{name}' not unique"
    with tempfile.TemporaryDirectory() as tmp:
        so = _compile(src.replace(old, new), tmp, "mutant")
        oracle.use_library(so)
        try:
            failed = 0
            for pin in BACKWARD_PINS:
                try:
                    pin()
                except AssertionError:
                    failed += 1
            assert failed > 0, f"no pin caught the planted mistake '{name}'"
        finally:
            oracle.use_library(None)


MIMO_PINS = [
    lambda: mpins.test_closed_form_over_steps(2),
    lambda: mpins.test_rank_one_is_the_mamba2_decode_without_conv(),
    lambda: mpins.test_slot_permutation(),
]


@pytest.mark.parametrize("name", sorted(MIMO_MUTANTS))
def test_planted_mimo_mistake_is_caught(name):
    src = open(SRC).read()
    old, new = MIMO_MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for '{name}' not unique"
    with tempfile.TemporaryDirectory() as tmp:
        so = _compile(src.replace(old, new), tmp, "mutant")
        oracle.use_library(so)
        try:
            failed = 0
            for pin in MIMO_PINS:
                try:
                    pin()
                except AssertionError:
                    failed += 1
            assert failed > 0, f"no pin caught the planted mistake '{name}'"
        finally:
            oracle.use_library(None)
