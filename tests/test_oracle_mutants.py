"""Planted mistakes: copies of the oracle source with one plausible error each
(a dropped term, a wrong sign or offset, a swapped operand or index) must
each fail at least one pin.  This shows the pins can see such mistakes.
Compiled and run on the CPU only."""
import os
import tempfile

import pytest

from oracle import Oracle
from oracle.build import SRC, compile_to
from oracle_pins import PINS

MUTANTS = [
    ("drop_relu_bias", "      g += b;\n      h[j] = g > 0.0", "      g += 0.0;\n      h[j] = g > 0.0"),
    ("no_relu", "h[j] = g > 0.0 ? g : 0.0;", "h[j] = g;"),
    ("reglu_gate_up_swapped", "h[j] = (g > 0.0 ? g : 0.0) * u;", "h[j] = (u > 0.0 ? u : 0.0) * g;"),
    ("q4_nibble_swapped", "(k < 16) ? (byte & 0x0F) : (byte >> 4)", "(k < 16) ? (byte >> 4) : (byte & 0x0F)"),
    ("q4_offset", "(double)(q - 8) *", "(double)(q - 7) *"),
    ("half_exp_bias", "e - 15);", "e - 14);"),
    ("rms_mean_wrong", "sqrt(ss / d + 1e-6)", "sqrt(ss / (d - 1) + 1e-6)"),
    ("pred_bias_dropped", "z[j] = acc + (L->pbias ? (double)L->pbias[j] : 0.0);", "z[j] = acc;"),
    ("mask_sign", "z[j] > theta)", "z[j] < theta)"),
    ("compact_ignores_begin", "for (int j = begin < 0 ? 0 : begin; j < F; ++j)", "for (int j = 0; j < F; ++j)"),
    ("down_uses_up", "weight(L->wdt, L->wd, L->sd, d, j, i)", "weight(L->wdt, L->wu, L->su, d, j, i)"),
    ("hot_off_by_one", "for (int j = 0; j < H && j < F; ++j) rowset[j] = 1;",
     "for (int j = 0; j < H - 1 && j < F; ++j) rowset[j] = 1;"),
    ("residual_dropped", "x_out[i] = (double)x[i] + y[i];", "x_out[i] = y[i];"),
    ("p1_transposed_scale", "acc += weight(L->pdt, L->p1, NULL, d, k, i) * xh[i];",
     "acc += weight(L->pdt, L->p1, NULL, d, k, i) * xh[d - 1 - i];"),
    ("predict_evaluates_hot_as_cold", "if (j < L->H) { z[j] = INFINITY; continue; }", ""),
    ("relu2_not_squared", "if (L->act == OR_RELU2) h[j] = h[j] * h[j];", ""),
    ("relu2_squares_before_relu", "h[j] = g > 0.0 ? g : 0.0;\n      if (L->act == OR_RELU2) h[j] = h[j] * h[j];",
     "h[j] = g > 0.0 ? g : 0.0;\n      if (L->act == OR_RELU2) h[j] = g * g;"),
]


@pytest.mark.parametrize("name,orig,mut", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, orig, mut):
    src = open(SRC).read()
    assert src.count(orig) == 1, f"mutation anchor not unique/present: {name}"
    with tempfile.TemporaryDirectory() as td:
        path = os.path.join(td, "mutant.c")
        with open(path, "w") as f:
            f.write(src.replace(orig, mut))
        lib = os.path.join(td, f"liboracle_{name}.so")
        compile_to(path, lib)
        orc = Oracle(lib)
        failed = []
        for pin in PINS:
            try:
                pin(orc)
            except AssertionError:
                failed.append(pin.__name__)
        assert failed, f"planted mistake {name} passed every pin"
