"""Plant plausible mistakes in copies of the oracle; each must fail a pin.

The mutants are built from the oracle's C source in a temporary directory
(CPU only).  A mutant that passes every pin would mean the pins cannot tell
that mistake from the definition.
"""
import os

import pytest

import oracle
import oracle_pins

MUTANTS = {
    "tie_to_higher_index": ("if (a->index < b->index) return -1;\n    if (a->index > b->index) return 1;",
                            "if (a->index < b->index) return 1;\n    if (a->index > b->index) return -1;"),
    "ascending_sort": ("if (a->value > b->value) return -1;\n    if (a->value < b->value) return 1;",
                       "if (a->value > b->value) return 1;\n    if (a->value < b->value) return -1;"),
    "dropped_last_term": ("for (int64_t h = 0; h < H; ++h) {", "for (int64_t h = 0; h < H - 1; ++h) {"),
    "transposed_gate": ("acc[e] += xv * wr[e];", "acc[e] += xv * w[(e * H + h) % (H * E)];"),
    "wrong_row_offset": ("const uint16_t* x = hidden + t * H;", "const uint16_t* x = hidden + t;"),
    "softmax_sign": ("const double s = exp(row[j].value - m) / denom;",
                     "const double s = exp(m - row[j].value) / denom;"),
    "softmax_short_denominator": ("for (int j = 0; j < k; ++j) denom += exp(row[j].value - m);",
                                  "for (int j = 1; j < k; ++j) denom += exp(row[j].value - m);"),
    "softmax_over_k_plus_one": ("for (int j = 0; j < k; ++j) denom += exp(row[j].value - m);",
                                "for (int j = 0; j < k + (k < E); ++j) denom += exp(row[j].value - m);"),
    "gap_off_by_one": ("row[k - 1].value - row[k].value", "row[0].value - row[k].value"),
    "ids_off_by_one": ("ids[t * k + j] = row[j].index;", "ids[t * k + j] = row[j < k - 1 ? j + 1 : j].index;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    before, after = MUTANTS[name]
    src = open(oracle.SOURCE).read()
    assert src.count(before) == 1, f"mutation site for {name} not found exactly once"
    mutant_src = tmp_path / f"mutant_{name}.c"
    mutant_src.write_text(src.replace(before, after))
    lib = oracle.compile_oracle(str(mutant_src), str(tmp_path / f"libmutant_{name}.so"))
    mutant = oracle.Oracle(lib)
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"


def test_unmutated_copy_passes(tmp_path):
    lib = oracle.compile_oracle(oracle.SOURCE, str(tmp_path / "libcopy.so"))
    copy = oracle.Oracle(lib)
    for pin in oracle_pins.ALL_PINS:
        pin(copy)
    assert os.path.exists(lib)
