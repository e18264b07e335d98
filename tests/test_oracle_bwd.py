"""CPU-only: the backward oracle passes its pins, and every planted mistake
in a copy of it is caught by them (the real source is untouched)."""
import os
import shutil

import pytest

import oracle
from tests import oracle_bwd_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_ref.c")

MUTANTS = {
    "missing_D_term": ("const double ds = pij * (dprow[j] - D);",
                       "const double ds = pij * dprow[j];"),
    "D_sign_flipped": ("D += prow[j] * dot;", "D -= prow[j] * dot;"),
    "dK_missing_scale": ("dkj[t] += scale * ds * qi[t];", "dkj[t] += ds * qi[t];"),
    "dQ_missing_scale": ("dqi[t] += scale * ds * krow[t];", "dqi[t] += ds * krow[t];"),
    "dV_uses_dS": ("dvj[t] += pij * doi[t];", "dvj[t] += ds * doi[t];"),
    "dK_uses_wrong_query": ("dkj[t] += scale * ds * qi[t];", "dkj[t] += scale * ds * doi[t];"),
    "P_unnormalised": ("exp(prow[j] - m) / sum;", "exp(prow[j] - m);"),
    "dP_uses_key": ("dot += doi[t] * vrow[t];", "dot += doi[t] * K[(size_t)j * d + t];"),
    "group_sum_overwritten": (
        "for (int hq = hk * G; hq < (hk + 1) * G; ++hq) {\n"
        "            const size_t qbase = ((size_t)b * H + hq) * head;\n"
        "            for (size_t e = 0; e < head; ++e) {\n"
        "                Q[e] = bits ?",
        "for (int hq = hk * G; hq < (hk + 1) * G; ++hq) {\n"
        "            for (size_t e = 0; e < head; ++e) dK[e] = dV[e] = 0.0;\n"
        "            const size_t qbase = ((size_t)b * H + hq) * head;\n"
        "            for (size_t e = 0; e < head; ++e) {\n"
        "                Q[e] = bits ?"),
    "backward_mask_not_causal": ("if (!key_allowed(i, j, causal, kv_lim, 0)) {",
                                 "if (!key_allowed(i, j, 0, kv_lim, 0)) {"),
    "kv_rows_dK_missing_scale": ("aK[(size_t)r * d + t] += scale * ds * qi[t];",
                                 "aK[(size_t)r * d + t] += ds * qi[t];"),
    "kv_rows_dV_uses_dS": ("aV[(size_t)r * d + t] += pij * doi[t];",
                           "aV[(size_t)r * d + t] += ds * doi[t];"),
    "kv_rows_one_head_of_group": ("for (int hq = hk * G; hq < (hk + 1) * G; ++hq) {\n"
                                  "            const size_t qbase = ((size_t)b * H + hq) * head;\n"
                                  "            for (size_t e = 0; e < head; ++e) {\n"
                                  "                Q[e] = bf16_to_f64(qb[qbase + e]);\n"
                                  "                dO[e] = bf16_to_f64(dob[qbase + e]);\n"
                                  "            }\n#pragma omp parallel",
                                  "for (int hq = hk * G; hq < hk * G + 1; ++hq) {\n"
                                  "            const size_t qbase = ((size_t)b * H + hq) * head;\n"
                                  "            for (size_t e = 0; e < head; ++e) {\n"
                                  "                Q[e] = bf16_to_f64(qb[qbase + e]);\n"
                                  "                dO[e] = bf16_to_f64(dob[qbase + e]);\n"
                                  "            }\n#pragma omp parallel"),
}


def test_real_backward_oracle_passes_every_pin():
    assert oracle_bwd_pins.failures(oracle.load()) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_backward_mutant_is_caught(name, tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    before, after = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(before) == 1, f"mutation anchor not found: {before}"
    src = tmp_path / f"mut_{name}.c"
    src.write_text(text.replace(before, after))
    lib_path = str(tmp_path / f"mut_{name}.so")
    oracle.build(str(src), lib_path)
    failed = oracle_bwd_pins.failures(oracle.load(lib_path))
    assert failed, f"mutant {name} passed every pin"
