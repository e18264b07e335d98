"""CPU-only: plant plausible mistakes in copies of the oracle and check that
the pin battery catches every one of them.

Each mutant is a textual edit of the oracle's C source, compiled to a
temporary library; the real source is untouched. A mutant that no pin catches
would mean the pins cannot tell that mistake from the right arithmetic.
"""
import os
import shutil

import pytest

import oracle
from tests import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_ref.c")

MUTANTS = {
    "dropped_scale": ("srow[j] = scale * dot;", "srow[j] = dot;"),
    "causal_direction_flipped": ("if (causal && j > i + off) return 0;",
                                 "if (causal && j < i + off) return 0;"),
    "causal_diagonal_hidden": ("if (causal && j > i + off) return 0;",
                               "if (causal && j >= i + off) return 0;"),
    "causal_offset_dropped": ("if (causal && j > i + off) return 0;",
                              "if (causal && j > i) return 0;"),
    "kv_len_off_by_one": ("if (j >= kv_lim) return 0;", "if (j > kv_lim) return 0;"),
    "lse_log2": ("double lse = m + log(sum);", "double lse = m + log2(sum);"),
    "lse_missing_max": ("double lse = m + log(sum);", "double lse = log(sum);"),
    "wrong_key_row": ("const double *kj = K + (size_t)j * d;",
                      "const double *kj = K + (size_t)i * d;"),
    "wrong_value_row": ("const double *vj = V + (size_t)j * d;",
                        "const double *vj = V + (size_t)i * d;"),
    "unnormalised_weights": ("double p = exp(srow[j] - lse);",
                             "double p = exp(srow[j] - m);"),
    "max_not_subtracted_in_sum": ("sum += exp(srow[j] - m);", "sum += exp(srow[j]);"),
    "kv_head_modulo_instead_of_group": ("h / (H / Hkv)) * head;  /* K, V */",
                                        "h % Hkv) * head;  /* K, V */"),
}


def test_real_oracle_passes_every_pin():
    assert oracle_pins.failures(oracle.load()) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    before, after = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(before) == 1, f"mutation anchor not found: {before}"
    src = tmp_path / f"mut_{name}.c"
    src.write_text(text.replace(before, after))
    lib_path = str(tmp_path / f"mut_{name}.so")
    oracle.build(str(src), lib_path)
    failed = oracle_pins.failures(oracle.load(lib_path))
    assert failed, f"mutant {name} passed every pin"
