"""Plant plausible mistakes in a copy of the oracle's C source and check that the
pins catch every one of them (CPU only; the real oracle is never modified)."""
import os
import subprocess

import pytest

from oracle import gdn_oracle as O
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(O.__file__), "gdn_oracle.c")

# (name, exact snippet in the source, replacement)
MUTANTS = [
    ("error_on_undecayed_state",  # the teaching scan's order: alpha*S + b (v - S k) k^T
     "            row[a] *= alpha;\n            sk += row[a] * kt[a];\n",
     "            sk += row[a] * kt[a];\n            row[a] *= alpha;\n"),
    ("no_decay", "            row[a] *= alpha;\n", ""),
    ("no_write_strength", "double u = b * (vt[i] - sk);", "double u = (vt[i] - sk);"),
    ("wrong_sign_correction", "for (int a = 0; a < dk; ++a) row[a] += u * kt[a];",
     "for (int a = 0; a < dk; ++a) row[a] -= u * kt[a];"),
    ("readout_before_update",
     "        token_update(S, dk, dv, alpha, b, kt, vt);\n        token_readout(S, dk, dv, P->scale, qt, P->o + ((size_t)t * HV + h) * dv);\n",
     "        token_readout(S, dk, dv, P->scale, qt, P->o + ((size_t)t * HV + h) * dv);\n        token_update(S, dk, dv, alpha, b, kt, vt);\n"),
    ("readout_with_key", "for (int a = 0; a < dk; ++a) acc += row[a] * qt[a];",
     "for (int a = 0; a < dk; ++a) acc += row[a] * qt[a] * 0.0 + row[a] * qt[(a + 1) % dk];"),
    ("wrong_head_map_sequential",
     "static void run_unit_sequential(const problem_t *P, int64_t n, int h, double *S) {\n    const int dk = P->dk, dv = P->dv, HK = P->HK, HV = P->HV;\n    const int c = h / (HV / HK);",
     "static void run_unit_sequential(const problem_t *P, int64_t n, int h, double *S) {\n    const int dk = P->dk, dv = P->dv, HK = P->HK, HV = P->HV;\n    const int c = h % HK;"),
    ("chunk_decay_ratio_inverted", "val = BETA(i) * exp(G[i] - G[j]) * kk;",
     "val = BETA(i) * exp(G[j] - G[i]) * kk;"),
    ("chunk_inverse_sign", "val -= A[(size_t)i * C + m] * T[(size_t)m * C + j];",
     "val += A[(size_t)i * C + m] * T[(size_t)m * C + j];"),
    ("chunk_missing_gamma_in_w",
     "acc += T[(size_t)i * C + j] * BETA(j) * exp(G[j]) * KR(j)[a];",
     "acc += T[(size_t)i * C + j] * BETA(j) * KR(j)[a];"),
    ("chunk_intra_includes_future", "for (int j = 0; j <= i; ++j) intra += mq[j] * U[(size_t)j * dv + e];",
     "for (int j = 0; j <= i && j < L; ++j) intra += mq[j] * U[(size_t)j * dv + e] * (j == i ? 0.0 : 1.0);"),
    ("chunk_state_decay_dropped", "double acc = exp(G[L - 1]) * S[(size_t)e * dk + a];",
     "double acc = S[(size_t)e * dk + a];"),
    ("chunk_state_transposed_u",
     "for (int j = 0; j < L; ++j) acc += U[(size_t)j * dv + e] * exp(G[L - 1] - G[j]) * KR(j)[a];",
     "for (int j = 0; j < L; ++j) acc += U[(size_t)j * dv + (e + 1) % dv] * exp(G[L - 1] - G[j]) * KR(j)[a];"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib_path = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                           str(mutated), "-o", str(lib_path), "-lm"])
    lib = O._load(str(lib_path))
    caught = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
        except ValueError:
            caught.append(pin.__name__)
    assert caught, f"no pin detects the planted mistake {name}"
