"""The pins catch plausible mistakes in the oracle.

Each case plants one mistake in a copy of ``oracle/h2o_oracle.c`` (on the
CPU, in a temporary library), runs pins of ``test_oracle_pins`` against it,
and requires at least one of them to fail: a pin set that a dropped term, a
flipped comparison or a wrong index survives would not pin anything."""
import ctypes
import os
import subprocess

import pytest

from oracle import oracle
import test_oracle_pins as pins

SRC = open(os.path.join(os.path.dirname(oracle.__file__), "h2o_oracle.c")).read()

MUTANTS = {
    "softmax scale dropped": ("const double scale = 1.0 / sqrt((double)d);\n\n    /* Step 1",
                              "const double scale = 1.0;\n\n    /* Step 1"),
    "diagonal masked": ("if (cand_pos[c] > P + i) { w[c] = 0.0; continue; }",
                        "if (cand_pos[c] >= P + i && c > 0) { w[c] = 0.0; continue; }"),
    "ties toward the older position": ("    return pos_a > pos_b;\n}", "    return pos_a < pos_b;\n}"),
    "old score not kept": ("for (int c = 0; c < n_cand; ++c) cand_score[c] += delta[c];",
                           "for (int c = 0; c < n_cand; ++c) cand_score[c] = delta[c];"),
    "one too few kept": ("kept[a] = (uint8_t)(above < C);", "kept[a] = (uint8_t)(above < C - 1);"),
    "free slots from the top": ("while (next_free < C && occupied[next_free]) ++next_free;",
                                "while (next_free < C && occupied[C - 1 - next_free]) ++next_free;"),
    "weights not normalised": ("double wc = exp(w[c] - m) / Z;", "double wc = exp(w[c] - m);"),
    "value row of the wrong key": ("vrow[c] = Vc + (size_t)cand_slot[c] * d;",
                                   "vrow[c] = Vc + (size_t)cand_slot[c > 0 ? c - 1 : c] * d;"),
}


# mistakes in the normalized policy, the insert-always variant and the backward
MUTANTS.update({
    "normalized: age off by one": ("cand_score[c] / (double)(t_after - cand_pos[c])",
                                   "cand_score[c] / (double)(t_after - cand_pos[c] + 1)"),
    "insert-always: the highest evicted": (
        "if (b != a && pos[b] >= 0 && ranks_above(phi[a], pos[a], phi[b], pos[b])) ++below;",
        "if (b != a && pos[b] >= 0 && ranks_above(phi[b], pos[b], phi[a], pos[a])) ++below;"),
    "insert-always: chunk token hidden from its own row": (
        "if (pos[j] < 0 || pos[j] > P + i) continue;\n                w[j] =",
        "if (pos[j] < 0 || pos[j] > P + i || (pos[j] == P + i && i > 0)) continue;\n                w[j] ="),
    "backward: row-sum term dropped": ("const double ds = p[j] * (dp[j] - pdp);", "const double ds = p[j] * dp[j];"),
    "backward: dV without the weights": ("gv[x] += p[j] * go[x];", "gv[x] += go[x];"),
    # the per-row checker used at full size
    "rows: a row does not see its own token": ("const int n_keys = C + i + 1;", "const int n_keys = C + i;"),
    "rows: KV head of the wrong group": ("const size_t bg = (size_t)b * Hkv + g;\n        const double *qrow",
                                         "const size_t bg = (size_t)b * Hkv + h % Hkv;\n        const double *qrow"),
})


def _battery():
    """Pins that together should fail for any of the mistakes above."""
    pins.test_hand_worked_example(None, "worked_example_c2_t2.json")
    pins.test_hand_worked_example(None, "worked_example_c2_t2_normalized.json")
    pins.test_oracle_matches_brute_force(None, 2, 4, 2, 8, 6, 3, 5, 1.0, False)
    pins.test_oracle_matches_brute_force(None, 1, 2, 1, 5, 4, 1, 9, 2.0, False)
    pins.test_oracle_matches_brute_force(None, 2, 4, 2, 8, 6, 3, 5, 1.0, True)
    pins.test_select_against_sort_with_planted_ties(None, 0)
    pins.test_insert_always_hand_worked_example(None)
    pins.test_insert_always_matches_brute_force(None, 2, 4, 2, 8, 6, 3, 5, 1.0)
    pins.test_backward_matches_torch_autograd(None)
    pins.test_rows_match_brute_force(None, 2, 4, 2, 8, 9, 4, 5)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path, monkeypatch, oracle_lib):
    old, new = MUTANTS[name]
    assert SRC.count(old) == 1, f"mutation site for '{name}' not found once"
    src = tmp_path / "mutant.c"
    src.write_text(SRC.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(so), str(src), "-lm"],
                   check=True)
    monkeypatch.setattr(oracle, "_lib", oracle.bind(ctypes.CDLL(str(so))))
    with pytest.raises((AssertionError, RuntimeError, ValueError)):
        _battery()


def test_unmutated_oracle_passes_the_battery(oracle_lib):
    _battery()
