"""Plants plausible mistakes in copies of the CPU oracle (never in the CUDA
path) and checks that at least one pin catches each one."""
import os

import pytest

from oracle import oracle as orc
from tests import oracle_pins as pins

SRC = os.path.join(os.path.dirname(orc.__file__), "si_oracle.c")

MUTANTS = {
    "relu_dropped": ("double relu = dot > 0.0 ? dot : 0.0;", "double relu = dot;"),
    "w_before_relu": ("double relu = dot > 0.0 ? dot : 0.0;\n        score += (double)w_row[h] * relu;",
                      "double wd = (double)w_row[h] * dot;\n        score += wd > 0.0 ? wd : 0.0;"),
    "visibility_off_by_one": ("(s + 1) * m <= t + 1", "s * m <= t"),
    "visibility_strict": ("(s + 1) * m <= t + 1", "(s + 1) * m < t + 1"),
    "tie_to_higher_index": ("if (a->idx < b->idx) return -1;\n    if (a->idx > b->idx) return 1;",
                            "if (a->idx < b->idx) return 1;\n    if (a->idx > b->idx) return -1;"),
    "ascending_scores": ("if (a->score > b->score) return -1;\n    if (a->score < b->score) return 1;",
                         "if (a->score > b->score) return 1;\n    if (a->score < b->score) return -1;"),
    "q_transposed": ("q_row[(int64_t)h * D + d]", "q_row[(int64_t)d * H + h]"),
    "kc_batch_ignored": ("const uint16_t* kc_b = kc + b * T * D;", "const uint16_t* kc_b = kc;"),
    "last_head_dropped": ("for (int h = 0; h < H; ++h) {", "for (int h = 0; h < H - 1; ++h) {"),
    "padding_score_zero": ("out_score[r * k + j] = -INFINITY;", "out_score[r * k + j] = 0.0;"),
    "w_of_wrong_head": ("score += (double)w_row[h] * relu;", "score += (double)w_row[H - 1 - h] * relu;"),
    # the per-row meta that the acceptance rule's tie band and tolerance use
    "rank_k_off_by_one": ("(k - 1 < nvis) ? keys[k - 1].score : NAN", "(k < nvis) ? keys[k].score : NAN"),
    "rank_k1_off_by_one": ("(k < nvis) ? keys[k].score : NAN", "(k + 1 < nvis) ? keys[k + 1].score : NAN"),
    "rowmax_signed": ("if (fabs(sc) > rowmax) rowmax = fabs(sc);", "if (sc > rowmax) rowmax = sc;"),
    "rowmax_over_invisible_keys": (
        "if (fabs(sc) > rowmax) rowmax = fabs(sc);\n            }",
        "}\n            { double a = fabs(indexer_score(q_row, w_row, kc_b + s * D, H, D)); if (a > rowmax) rowmax = a; }"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    with open(SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    path = tmp_path / f"mutant_{name}.c"
    path.write_text(src.replace(old, new))
    so = orc.build(str(path), str(tmp_path / f"libmutant_{name}.so"))
    lib = orc.load_library(so)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {name}"
