"""The oracle's pins must fail when a plausible mistake is planted in the oracle.

Each case copies oracle/ to a temporary directory, plants one mistake in the
C source (dropped decay, wrong sign of the delta write, transposed recall,
read-out with the wrong vector, wrong head grouping, inverted decay mask,
missing cumulative decay in W, strict instead of inclusive output mask) or in
the Python functions (bfloat16 rounding with ties up or one bit short, a
reset that keeps the old state, a step not written back to its slot, conv
taps in reverse order, a conv state that is ignored, v normalised like q and
k), rebuilds it and runs tests/test_oracle_pins.py against the mutant.  At
least one pin must fail for every mutant.  Mistakes are planted in the oracle
on the CPU only.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "drop_decay": ("for (int64_t x = 0; x < Dv * Dk; ++x) S[x] *= a;\n            for (int64_t i = 0;",
                   "for (int64_t x = 0; x < Dv * Dk; ++x) S[x] *= 1.0;\n            for (int64_t i = 0;"),
    "sign_of_write": ("const double u = b * (vt[i] - r[i]);", "const double u = b * (vt[i] + r[i]);"),
    "transposed_recall": ("acc += S[i * Dk + d] * kt[d];\n                r[i] = acc;\n            }\n        }",
                          "acc += S[d * Dk + i] * kt[d];\n                r[i] = acc;\n            }\n        }"),
    "readout_with_key": ("acc += S[i * Dk + d] * qt[d];", "acc += S[i * Dk + d] * kt[d];"),
    "head_group_modulo": ("const int64_t j = h / (Hv / Hqk);", "const int64_t j = h % Hqk;"),
    "chunk_mask_inverted": ("val = GB(beta, r) * kk * exp(GREC(r) - gam[i]);",
                            "val = GB(beta, r) * kk * exp(gam[i] - GREC(r));"),
    "chunk_W_without_decay": ("GB(beta, i) *\n                                     exp(GREC(i)) * KR(i)[d];",
                              "GB(beta, i) *\n                                     1.0 * KR(i)[d];"),
    "chunk_recall_first_uses_gamma_r": (
        "(order == ORACLE_ORDER_ILLUSTRATIVE ? ((r) > 0 ? gam[(r) - 1] : 0.0) : gam[r])",
        "(gam[r])"),
    "chunk_output_mask_strict": ("for (int64_t i = 0; i <= r; ++i) {\n                                double qk",
                                 "for (int64_t i = 0; i < r; ++i) {\n                                double qk"),
}

# mistakes in the Python functions of oracle/__init__.py
MUTANTS_PY = {
    "bf16_ties_up": ("return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)",
                     "return np.ldexp(np.floor(np.ldexp(m, 8) + 0.5), e - 8)"),
    "bf16_seven_bits": ("return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)",
                        "return np.ldexp(np.rint(np.ldexp(m, 7)), e - 7)"),
    "slots_reset_ignored": ("states[rs != 0] = 0.0", "states[rs != 0] = states[rs != 0]"),
    "slots_not_written_back": ("    pool[idx] = new\n", "    pool[idx] = pool[idx]\n"),
    "conv_taps_reversed": ("y[cu[n] + t] += w[:, j] * ext[t + j]", "y[cu[n] + t] += w[:, 3 - j] * ext[t + j]"),
    "conv_state_ignored": ("st = np.zeros((N, 3, C)) if conv_state is None else _f64(conv_state)",
                           "st = np.zeros((N, 3, C))"),
    "conv_v_normalised": ("v = ys[2].reshape(T, Hv, Dv)", "v = l2_normalise_heads(ys[2], Hv, Dv)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS) + sorted(MUTANTS_PY))
def test_pins_catch_mutant(name, tmp_path):
    fname = "gdn_oracle.c" if name in MUTANTS else "__init__.py"
    src = open(os.path.join(ROOT, "oracle", fname)).read()
    old, new = MUTANTS[name] if name in MUTANTS else MUTANTS_PY[name]
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    work = tmp_path / "repo"
    shutil.copytree(os.path.join(ROOT, "oracle"), work / "oracle",
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    shutil.copytree(os.path.join(ROOT, "gated_deltanet_04_b200"), work / "gated_deltanet_04_b200",
                    ignore=shutil.ignore_patterns("*.so", "__pycache__", "csrc"))
    (work / "tests").mkdir()
    for f in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), work / "tests" / f)
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), work / "tests" / "golden")
    (work / "oracle" / fname).write_text(src.replace(old, new))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider",
                        "tests/test_oracle_pins.py"], cwd=work, capture_output=True, text=True,
                       timeout=600)
    tail = r.stdout.strip().splitlines()[-1] if r.stdout.strip() else r.stderr[-500:]
    assert r.returncode != 0 and "failed" in tail, f"mutant {name} survived: {tail}"
