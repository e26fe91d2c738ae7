"""Mutation check of the oracle's pins: plausible mistakes planted in a copy of the oracle's
C source (a dropped scale, a wrong GQA head map, a causal off-by-one, a transposed V stride, a
missing normalisation, a wrong LSE, a wrong mean divisor, a wrong rounding mode, a window
off-by-one or a dropped window, a sink left out of the denominator or of an empty row, a gate
sample stride off by one, a strict gate threshold, an unsquared gate mean) must each be
caught by at least one pin. The planted copies are built in a temporary directory on the CPU;
the real oracle is untouched."""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

MUTANTS = {
    "dropped_scale": ("s[j] = a->scale * dot;", "s[j] = dot;"),
    "gqa_modulo_map": ("int64_t g = h / group;", "int64_t g = h % a->hk;"),
    "causal_off_by_one": ("const int64_t diag = i + a->sk - a->sq;", "const int64_t diag = i + a->sk - a->sq - 1;"),
    "causal_top_left": ("const int64_t diag = i + a->sk - a->sq;", "const int64_t diag = i;"),
    "v_stride_dqk": ("((bi * a->sk + lo + j) * a->hk + g) * a->dv;", "((bi * a->sk + lo + j) * a->hk + g) * a->dqk;"),
    "window_off_by_one": ("diag - a->window > lo) lo = diag - a->window;", "diag - a->window > lo) lo = diag - a->window + 1;"),
    "window_ignored": ("if (a->window >= 0 && diag", "if (0 && diag"),
    "sink_left_out_of_sum": ("if (has_sink) l += exp(sink - m);", "if (0) l += exp(sink - m);"),
    "empty_row_ignores_sink": ("*lse_out = has_sink ? sink : -INFINITY;", "*lse_out = -INFINITY;"),
    "gate_stride_off_by_one": ("const int64_t stride = (sk + 2047) / 2048;", "const int64_t stride = sk / 2048 + 1;"),
    "gate_strict_threshold": ("const int on = r >= threshold;", "const int on = r > threshold;"),
    "gate_mean_not_squared": ("num += mu[c] * mu[c];", "num += fabs(mu[c]);"),
    "no_normalisation": ("o_row[c] /= l;", "o_row[c] /= 1.0;"),
    "lse_without_max": ("*lse_out = m + log(l);", "*lse_out = log(l);"),
    "mean_divisor": ("double mean = sum / (double)sk;", "double mean = sum / (double)(sk - 1);"),
    "round_toward_zero": ("double r = nearbyint(ldexp(ax, -qexp));", "double r = trunc(ldexp(ax, -qexp));"),
    "max_skips_first": ("double m = s[0];", "double m = 0.0;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found: {old}"
    mut_src = tmp_path / "attn_oracle_mutant.c"
    mut_src.write_text(src.replace(old, new))
    out = str(tmp_path / f"liboracle_{name}.so")
    oracle.build(force=True, src=str(mut_src), out=out)
    lib = oracle.load_library(out)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
