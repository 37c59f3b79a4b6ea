"""The sparse-attention CPU oracle against its pins, and plausible mistakes
planted in copies of its source (on the CPU, never in the CUDA path)."""
import os

import pytest

from oracle import attention as att
from tests import attn_oracle_pins as pins

SRC = os.path.join(os.path.dirname(att.__file__), "si_attn_oracle.c")

MUTANTS = {
    "scale_dropped": ("s[j] = scale * dot;", "s[j] = dot;"),
    "not_normalised": ("const double p = exp(s[j] - smax) / z;", "const double p = exp(s[j] - smax);"),
    "lse_without_max": ("lse[r * H + h] = smax + log(z);", "lse[r * H + h] = log(z);"),
    "head_zero_only": ("const uint16_t* qh = q_rows + (r * H + h) * D;", "const uint16_t* qh = q_rows + (r * H) * D;"),
    "empty_row_lse_zero": ("lse[r * H + h] = -INFINITY;", "lse[r * H + h] = 0.0;"),
    "absw_signed": ("if (ah) ah[e] += p * fabs(v);", "if (ah) ah[e] += p * v;"),
    "batch_ignored": ("const uint16_t* vj = vcache + (b * T + sel[j]) * DV;",
                      "const uint16_t* vj = vcache + (sel[j]) * DV;"),
    "last_key_dropped": ("for (int64_t j = 0; j < k; ++j) {\n                if (sel[j] < 0) continue;\n                const double p",
                         "for (int64_t j = 0; j + 1 < k; ++j) {\n                if (sel[j] < 0) continue;\n                const double p"),
}


@pytest.fixture(scope="module")
def lib():
    return att.load_library()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(lib, pin):
    pin(lib)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    path = tmp_path / f"attn_mutant_{name}.c"
    path.write_text(src.replace(old, new))
    lib = att.load_library(att.build(str(path), str(tmp_path / f"libattn_mutant_{name}.so")))
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {name}"
