"""Planted mistakes: each mutant of the oracle's C source must fail a pin.

A mutant is a textual edit of bq_oracle.c (a dropped term, a wrong sign or
index, a transposed operand, a wrong rounding rule), compiled on the CPU into a
temporary library and swapped in for the real oracle while the pin tests of
test_oracle.py run.  Every mutant keeps all memory accesses in bounds for the
shapes those tests use.
"""
import ctypes
import inspect
import json
import os
import subprocess

import pytest

import oracle
import test_oracle as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "bq_oracle.c")

MUTANTS = {
    "wscale_drops_kblock_index": ("(double)sa[m * Kb + kb] * (double)sw[nb * Kb + kb];",
                                  "(double)sa[m * Kb + kb] * (double)sw[nb * Kb + 0];"),
    "ascale_drops_kblock_index": ("acc += P * (double)sa[m * Kb + kb]",
                                  "acc += P * (double)sa[m * Kb]"),
    "drops_block_accumulation": ("acc += P * (double)sa", "acc = P * (double)sa"),
    "int8_product_sign": ("Pi += (int64_t)(int8_t)qa", "Pi -= (int64_t)(int8_t)qa"),
    "transposed_weight_operand": ("(int8_t)qw[n * ldw + k]", "(int8_t)qw[m * ldw + k]"),
    "multiply_instead_of_divide": ("float c = x[i] / s;", "float c = x[i] * s;"),
    "round_half_away": ("return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;\n}",
                        "return f + 1.0;\n}"),
    "int8_qmax_128": ("? 127.0f : 448.0f", "? 128.0f : 448.0f"),
    "e4m3_ties_down": ("else pick = (c % 2 == 0) ? c : c + 1;", "else pick = c;"),
    "e4m3_no_subnormals": ("if (e == 0) v = ldexp((double)m, -9);",
                           "if (e == 0) v = ldexp((double)m, -10);"),
    "seam_floor_not_ceil": ("return (seam + bn - 1) / bn + (n - seam) / bn;",
                            "return seam / bn + (n - seam) / bn;"),
    "silu_sign": ("g / (1.0 + exp(-g)) * u", "g / (1.0 + exp(g)) * u"),
    "combine_first_weight_only": ("(double)w[t * topk + j]", "(double)w[t * topk]"),
    "bias_dropped": ("if (bias) acc += bq_ref_bf16_to_double(bias[n]);", ""),
    "mx_scale_exponent_off_by_one": ("se = floor_log2(amax) - 8;", "se = floor_log2(amax) - 7;"),
    "mx_no_low_clamp": ("if (se < -127) se = -127;", ""),
    "mx_weight_scale_inverted": ("ldexp(1.0, (int)sw[n * G + g] - 127)",
                                 "ldexp(1.0, 127 - (int)sw[n * G + g])"),
    "mx_bias_dropped": ("if (bias != NULL) acc += bq_ref_bf16_to_double(bias[n]);", ""),
    "mx_act_scale_first_group_only": ("ldexp(1.0, (int)sa[m * G + g] - 127)",
                                      "ldexp(1.0, (int)sa[m * G] - 127)"),
    "route_ties_to_higher_index": ("if (!taken[e] && (best < 0 || p[e] > p[best])) best = e;",
                                   "if (!taken[e] && (best < 0 || p[e] >= p[best])) best = e;"),
    "route_not_renormalised": ("w[t * topk + j] = (float)(p[ids[t * topk + j]] / topsum);",
                               "w[t * topk + j] = (float)(p[ids[t * topk + j]]);"),
    "bf16_ties_up": ("else r = (fmod(f, 2.0) == 0.0) ? f : f + 1.0;\n    double res",
                     "else r = f + 1.0;\n    double res"),
}


def _pin_functions():
    out = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        out.append((name, fn, params))
    return out


def _run_all_pins(golden):
    """Run every pin; return the name of the first one that fails, or None."""
    for name, fn, params in _pin_functions():
        argnames = inspect.signature(fn).parameters
        cases = [{}]
        for p in params:
            names = [n.strip() for n in p.args[0].split(",")]
            cases = [dict(c, **dict(zip(names, v if len(names) > 1 else (v,))))
                     for c in cases for v in p.args[1]]
        for case in cases:
            kw = dict(case)
            if "golden" in argnames:
                kw["golden"] = golden
            try:
                fn(**kw)
            except (AssertionError, ValueError):
                return name
    return None


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_mutant_is_caught(mutant, tmp_path, golden, monkeypatch):
    old, new = MUTANTS[mutant]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique for {mutant}"
    path = tmp_path / "mut.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "mut.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", str(so), str(path), "-lm"])
    lib = oracle.configure(ctypes.CDLL(str(so)))
    monkeypatch.setattr(oracle, "_lib", lib)
    caught = _run_all_pins(golden)
    assert caught is not None, f"no pin catches mutant {mutant}"


def test_real_oracle_passes_all_pins(golden):
    assert _run_all_pins(golden) is None
