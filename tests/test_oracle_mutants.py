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


# Mistakes planted in the prologue (plain numpy): each replaces oracle.prologue
# for the duration of one test and must fail at least one prologue pin.
def _prologue_mutant(kind):
    import numpy as np
    real = O.prologue

    def mutant(q, k, g, beta, flags):
        q, k, g, beta = (O._f64(x) for x in (q, k, g, beta))
        if kind == "no_eps" and flags & O.PROLOGUE_NORM_K:
            k = k / np.sqrt(np.sum(k * k, axis=-1, keepdims=True))
            return real(q, k, g, beta, flags & ~O.PROLOGUE_NORM_K)
        if kind == "wrong_axis" and flags & O.PROLOGUE_NORM_Q:
            q = q / np.maximum(np.sqrt(np.sum(q * q, axis=0, keepdims=True)), 1e-12)
            return real(q, k, g, beta, flags & ~O.PROLOGUE_NORM_Q)
        if kind == "flags_swapped":
            f = flags & ~3
            f |= (O.PROLOGUE_NORM_K if flags & O.PROLOGUE_NORM_Q else 0)
            f |= (O.PROLOGUE_NORM_Q if flags & O.PROLOGUE_NORM_K else 0)
            return real(q, k, g, beta, f)
        if kind == "forget_gate_sign" and flags & O.PROLOGUE_GATE_LOGITS:
            qq, kk, _, bb = real(q, k, g, beta, flags)
            return qq, kk, -np.logaddexp(0.0, g), bb
        if kind == "write_gate_sign" and flags & O.PROLOGUE_GATE_LOGITS:
            qq, kk, gg, _ = real(q, k, g, beta, flags)
            return qq, kk, gg, np.exp(-np.logaddexp(0.0, beta))
        if kind == "gate_as_alpha" and flags & O.PROLOGUE_GATE_LOGITS:
            qq, kk, _, bb = real(q, k, g, beta, flags)   # alpha itself returned as g
            return qq, kk, np.exp(-np.logaddexp(0.0, -g)), bb
        if kind == "norms_ignored":
            return real(q, k, g, beta, flags & O.PROLOGUE_GATE_LOGITS)
        return real(q, k, g, beta, flags)
    return mutant


PROLOGUE_MUTANTS = ["no_eps", "wrong_axis", "flags_swapped", "forget_gate_sign",
                    "write_gate_sign", "gate_as_alpha", "norms_ignored"]


@pytest.mark.parametrize("kind", PROLOGUE_MUTANTS)
def test_prologue_pins_catch_mutant(monkeypatch, kind):
    import numpy as np
    monkeypatch.setattr(O, "prologue", _prologue_mutant(kind))
    caught = []
    with np.errstate(all="ignore"):
        for pin in ALL_PINS:
            if "prologue" not in pin.__name__:
                continue
            try:
                pin()
            except (AssertionError, ValueError):
                caught.append(pin.__name__)
    assert caught, f"no pin detects the planted prologue mistake {kind}"


# Mistakes planted in the per-row-decay step (plain numpy), each caught by a
# row-decay pin.
def _row_decay_mutant(kind):
    import numpy as np

    def mutant(q, k, v, g_rows, beta, state, scale=1.0):
        q, k, v, g_rows, beta = (O._f64(x) for x in (q, k, v, g_rows, beta))
        S = O._f64(state).copy()
        N, HK, dk = q.shape
        HV, dv = v.shape[1], v.shape[2]
        o = np.zeros((N, HV, dv))
        for n in range(N):
            for h in range(HV):
                c = h // (HV // HK)
                kt, qt = k[n, c], q[n, c]
                a = np.exp(g_rows[n, h])
                for i in range(dv):
                    row = S[n, h, i]
                    if kind == "decay_after_correction":
                        row = a[i] * (row + beta[n, h] * (v[n, h, i] - row @ kt) * kt)
                    elif kind == "decay_on_key_columns":
                        ac = np.resize(a, dk)
                        row = row * ac
                        row = row + beta[n, h] * (v[n, h, i] - row @ kt) * kt
                    elif kind == "first_row_decay_for_all":
                        row = row * a[0]
                        row = row + beta[n, h] * (v[n, h, i] - row @ kt) * kt
                    S[n, h, i] = row
                    o[n, h, i] = scale * (row @ qt)
        return o, S
    return mutant


@pytest.mark.parametrize("kind", ["decay_after_correction", "decay_on_key_columns",
                                  "first_row_decay_for_all"])
def test_row_decay_pins_catch_mutant(monkeypatch, kind):
    monkeypatch.setattr(O, "step_row_decay", _row_decay_mutant(kind))
    caught = []
    for pin in ALL_PINS:
        if "row_decay" not in pin.__name__:
            continue
        try:
            pin()
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin detects the planted row-decay mistake {kind}"


# Mistakes planted in the short convolution and the output gate (plain numpy),
# each caught by one of their pins.
def _conv_mutant(kind):
    import numpy as np

    def mutant(x, weight, bias=None, conv_state=None, cu_seqlens=None, activation="none"):
        x, w = O._f64(x), O._f64(weight)
        C, W = w.shape
        if cu_seqlens is None and x.ndim == 3:
            B, T = x.shape[0], x.shape[1]
            bounds = [(b * T, (b + 1) * T) for b in range(B)]
        else:
            cu = np.asarray(O._f64(cu_seqlens)).astype(np.int64)
            bounds = [(int(cu[i]), int(cu[i + 1])) for i in range(len(cu) - 1)]
        x = x.reshape(-1, C)
        N = len(bounds)
        hist = (np.zeros((N, W - 1, C)) if conv_state is None or kind == "state_ignored"
                else O._f64(conv_state).reshape(N, W - 1, C))
        b = np.zeros(C) if bias is None or kind == "bias_dropped" else O._f64(bias)
        y = np.zeros_like(x)
        new_state = np.zeros((N, W - 1, C))
        for n, (s0, s1) in enumerate(bounds):
            L = s1 - s0
            xs = np.concatenate([hist[n], x[s0:s1]], axis=0)
            acc = np.tile(b, (L, 1))
            for j in range(W):
                wj = w[:, W - 1 - j] if kind == "taps_reversed" else w[:, j]
                if kind == "one_token_late":
                    src = np.concatenate([np.zeros((1, C)), xs])[j:j + L]
                else:
                    src = xs[j:j + L]
                acc = acc + wj * src
            if activation == "silu":
                acc = (1.0 / (1.0 + np.exp(-acc))) if kind == "silu_as_sigmoid" else O.silu(acc)
            y[s0:s1] = acc
            new_state[n] = xs[:W - 1] if kind == "state_from_first_tokens" else xs[L:L + W - 1]
        return y, new_state
    return mutant


@pytest.mark.parametrize("kind", ["taps_reversed", "one_token_late", "state_ignored",
                                  "bias_dropped", "silu_as_sigmoid", "state_from_first_tokens"])
def test_conv_pins_catch_mutant(monkeypatch, kind):
    monkeypatch.setattr(O, "short_conv", _conv_mutant(kind))
    caught = []
    for pin in ALL_PINS:
        if "conv" not in pin.__name__ and "layer" not in pin.__name__:
            continue
        try:
            pin()
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin detects the planted convolution mistake {kind}"


@pytest.mark.parametrize("kind", ["tanh_gate", "one_minus_sigmoid", "gate_on_logit_only"])
def test_gate_pins_catch_mutant(monkeypatch, kind):
    import numpy as np

    def mutant(o, z):
        o, z = O._f64(o), O._f64(z)
        if kind == "tanh_gate":
            return o * np.tanh(z)
        if kind == "one_minus_sigmoid":
            return o * (1.0 - 1.0 / (1.0 + np.exp(-z)))
        return o + (1.0 / (1.0 + np.exp(-z)))
    monkeypatch.setattr(O, "output_gate", mutant)
    caught = []
    for pin in ALL_PINS:
        if "gate" not in pin.__name__ and "layer" not in pin.__name__:
            continue
        try:
            pin()
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin detects the planted gate mistake {kind}"
