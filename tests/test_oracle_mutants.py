"""Every pin in test_oracle_pins must be able to catch a plausible mistake.

Each case below plants one mistake in a copy of the oracle's C source
(transposed state, flipped sign of the delta correction, decay applied to the
new write, reversed conv taps, missing SiLU, missing 1/sqrt(d_k), wrong gate
formulas, eps in the wrong place, off-by-one decay index), compiles it on the
CPU, and runs the pin suite against it: at least one pin must fail.  The
unmodified source must pass them all.  CPU only.
"""
import inspect

import pytest

import oracle
import test_oracle_pins as pins

MUTANTS = {
    "state_transposed_in_output": ("acc += S[(size_t)i * dk + j] * q[j];", "acc += S[(size_t)j * dk + i] * q[j];"),
    "delta_correction_sign": ("*s = a * (*s - be * Sk[i] * k[j]) + be * v[i] * k[j];",
                              "*s = a * (*s + be * Sk[i] * k[j]) + be * v[i] * k[j];"),
    "decay_on_new_write": ("*s = a * (*s - be * Sk[i] * k[j]) + be * v[i] * k[j];",
                           "*s = a * (*s - be * Sk[i] * k[j] + be * v[i] * k[j]);"),
    "no_delta_correction": ("*s = a * (*s - be * Sk[i] * k[j]) + be * v[i] * k[j];",
                            "*s = a * (*s) + be * v[i] * k[j];"),
    "conv_taps_reversed": ("u += (double)w[(size_t)c * 4 + j] *", "u += (double)w[(size_t)c * 4 + (3 - j)] *"),
    "conv_no_silu": ("out[(((size_t)b * T + t) * H + h) * d + i] = silu(u);",
                     "out[(((size_t)b * T + t) * H + h) * d + i] = u;"),
    "output_scale_missing": ("ot[i] = acc * scale;", "ot[i] = acc;"),
    "softplus_wrong": ("log1p(exp(-fabs(x)))", "log1p(exp(-x))"),
    "beta_sign": ("beta[idx] = 1.0 / (1.0 + exp(-(double)bgate[idx]));",
                  "beta[idx] = 1.0 / (1.0 + exp((double)bgate[idx]));"),
    "A_log_not_exponentiated": ("const double a = exp((double)A_log[h]);", "const double a = (double)A_log[h];"),
    "l2_eps_outside_sqrt": ("const double inv = 1.0 / sqrt(ss + eps);", "const double inv = 1.0 / (sqrt(ss) + eps);"),
    "rms_sum_not_mean": ("const double r = 1.0 / sqrt(ms / dv + eps);", "const double r = 1.0 / sqrt(ms + eps);"),
    "decay_index_shift": ("const double a = alpha[row], be = beta[row];",
                          "const double a = alpha[row >= (size_t)H ? row - H : row], be = beta[row];"),
    "output_before_update": [
        ("        /* S k */\n",
         "        for (int i = 0; i < dv; ++i) { double acc = 0.0;\n"
         "            for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * q[j];\n"
         "            o[row * dv + i] = acc * scale; }\n        /* S k */\n"),
        ("ot[i] = acc * scale;", "(void)ot; (void)acc;"),
    ],
}


def _pin_functions():
    out = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        params = inspect.signature(fn).parameters
        if "T" in params or "C" in params:
            out.append((name, lambda fn=fn: fn(T=65, C=64)))
        elif not params:
            out.append((name, fn))
    return out


def _failures(so_path):
    failed = []
    with oracle._swapped_library(so_path):
        for name, fn in _pin_functions():
            try:
                fn()
            except AssertionError:
                failed.append(name)
    return failed


def test_unmodified_source_passes_every_pin(tmp_path):
    so = oracle.compile_variant(oracle.source_text(), str(tmp_path / "clean.so"))
    assert _failures(so) == []


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistake_is_caught(mutant, tmp_path):
    src = oracle.source_text()
    edits = MUTANTS[mutant]
    for old, new in ([edits] if isinstance(edits, tuple) else edits):
        assert src.count(old) == 1, mutant
        src = src.replace(old, new)
    so = oracle.compile_variant(src, str(tmp_path / (mutant + ".so")))
    assert _failures(so), f"no pin catches {mutant}"
