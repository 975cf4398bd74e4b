"""Checks that pin the float64 oracle to facts fixed by the pages and by mathematics.

Each ``pin_*`` function takes an oracle library handle (``None`` = the normal
build) and raises AssertionError when the oracle disagrees.  They are run by
``test_oracle_pins.py`` against the real oracle and by
``test_oracle_mutants.py`` against deliberately broken copies, to show that a
plausible mistake (a dropped term, a wrong sign or index, the error term taken
before the decay, the read-out taken before the update, a transposed operand)
fails at least one of them.

Sources:
* worked examples: "Qwen3-Next" (sghael.github.io), section "Correcting a
  memory instead of adding to it" (fixtures under tests/golden/);
* head geometry 32 V / 16 QK / 128: model card "Qwen3-Next-80B-A3B-Instruct",
  section "Model Overview";
* the rule S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T, o_t = S_t q_t
  and its invariants: closed forms derived from it (stated per check).
"""
from __future__ import annotations

import math
import os

import numpy as np

from oracle import gdn_oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read_fixture(name):
    s0, rows = None, []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if parts[0] == "S0":
                s0 = float(parts[1])
            else:
                rows.append([float(x) for x in parts[1:]])
    return s0, np.array(rows)


def _rand_problem(rng, T, HK, HV, dk, dv, unit=True, g_range=(math.log(0.9), 0.0)):
    q = rng.standard_normal((1, T, HK, dk))
    k = rng.standard_normal((1, T, HK, dk))
    if unit:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, HV, dv))
    g = rng.uniform(*g_range, size=(1, T, HV))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((1, T, HV))))
    return q, k, v, g, beta


# ----------------------------------------------------------------------------
# Values printed on the pages
# ----------------------------------------------------------------------------
def pin_worked_example_delta(lib=None):
    s0, rows = _read_fixture("worked_example_delta.txt")
    T = len(rows)
    one = np.ones((1, T, 1, 1))
    g = rows[:, 0].reshape(1, T, 1)
    beta = rows[:, 1].reshape(1, T, 1)
    v = rows[:, 2].reshape(1, T, 1, 1)
    o, hT = O.prefill(one, one, v, g, beta, h0=np.full((1, 1, 1, 1), s0), lib=lib)
    assert np.array_equal(o.ravel(), rows[:, 3]), (o.ravel(), rows[:, 3])
    assert hT.ravel()[0] == rows[-1, 3]
    # the same through the chunked form and through decode steps
    oc, _ = O.prefill(one, one, v, g, beta, h0=np.full((1, 1, 1, 1), s0), chunked=True,
                      chunk=2, lib=lib)
    assert np.allclose(oc.ravel(), rows[:, 3], rtol=0, atol=1e-12)
    S = np.full((1, 1, 1, 1), s0)
    for t in range(T):
        ot, S = O.step(one[:, t], one[:, t], v[:, t], g[:, t], beta[:, t], S, lib=lib)
        assert ot.ravel()[0] == rows[t, 3]


def pin_worked_example_gated(lib=None):
    s0, rows = _read_fixture("worked_example_gated.txt")
    T = len(rows)
    one = np.ones((1, T, 1, 1))
    g = np.log(rows[:, 0]).reshape(1, T, 1)
    beta = rows[:, 1].reshape(1, T, 1)
    v = rows[:, 2].reshape(1, T, 1, 1)
    h0 = np.full((1, 1, 1, 1), s0)
    o, hT = O.prefill(one, one, v, g, beta, h0=h0, lib=lib)
    assert np.allclose(o.ravel(), rows[:, 3], rtol=0, atol=1e-14), o.ravel()
    oc, _ = O.prefill(one, one, v, g, beta, h0=h0, chunked=True, chunk=1, lib=lib)
    assert np.allclose(oc.ravel(), rows[:, 3], rtol=0, atol=1e-14), oc.ravel()
    ot, _ = O.step(one[:, 0], one[:, 0], v[:, 0], g[:, 0], beta[:, 0], h0, lib=lib)
    assert np.allclose(ot.ravel(), rows[0, 3], rtol=0, atol=1e-14)


# ----------------------------------------------------------------------------
# Closed forms and invariants of the rule
# ----------------------------------------------------------------------------
def pin_converges_closed_form(lib=None):
    """No decay, one repeated unit key: S_n k = v + (1-b)^n (S_0 k - v) (the page's
    example approaching the target 10), and directions orthogonal to k are never
    touched."""
    rng = np.random.default_rng(1)
    dk, dv, T, b = 5, 3, 12, 0.3
    kvec = rng.standard_normal(dk); kvec /= np.linalg.norm(kvec)
    qvec = rng.standard_normal(dk)
    vvec = rng.standard_normal(dv)
    S0 = rng.standard_normal((dv, dk))
    k = np.broadcast_to(kvec, (1, T, 1, dk)).copy()
    q = np.broadcast_to(qvec, (1, T, 1, dk)).copy()
    v = np.broadcast_to(vvec, (1, T, 1, dv)).copy()
    g = np.zeros((1, T, 1)); beta = np.full((1, T, 1), b)
    for chunked in (False, True):
        o, hT = O.prefill(q, k, v, g, beta, h0=S0[None, None], chunked=chunked, chunk=5, lib=lib)
        S = hT[0, 0]
        expect = vvec + (1 - b) ** T * (S0 @ kvec - vvec)
        assert np.allclose(S @ kvec, expect, atol=1e-12)
        perp = qvec - (qvec @ kvec) * kvec
        assert np.allclose(S @ perp, S0 @ perp, atol=1e-12)
        # o_t after the update: o_t = S_t q with S_t k following the same closed form
        for t in range(T):
            skt = vvec + (1 - b) ** (t + 1) * (S0 @ kvec - vvec)
            ot = S0 @ perp + skt * (qvec @ kvec)
            assert np.allclose(o[t, 0], ot, atol=1e-12)


def pin_identity_when_no_write(lib=None):
    """alpha = 1, beta = 0: S never changes and o_t = S_0 q_t."""
    rng = np.random.default_rng(2)
    q, k, v, g, beta = _rand_problem(rng, 9, 2, 4, 6, 5)
    g[:] = 0.0; beta[:] = 0.0
    h0 = rng.standard_normal((1, 4, 5, 6))
    for chunked in (False, True):
        o, hT = O.prefill(q, k, v, g, beta, h0=h0, chunked=chunked, chunk=4, lib=lib)
        assert np.allclose(hT, h0, atol=1e-13)
        for h in range(4):
            expect = q[0, :, h // 2, :] @ h0[0, h].T
            assert np.allclose(o[:, h], expect, atol=1e-13)


def pin_full_write_recalls_value(lib=None):
    """beta = 1 with a unit key: S_t k_t = v_t exactly, whatever the decay.  dk != dv
    so a transposed state fails; HK < HV so a wrong head map fails."""
    rng = np.random.default_rng(3)
    HK, HV, dk, dv, T = 2, 4, 4, 3, 7
    q, k, v, g, beta = _rand_problem(rng, T, HK, HV, dk, dv, g_range=(-1.0, 0.0))
    beta[:] = 1.0
    h0 = rng.standard_normal((1, HV, dv, dk))
    S = h0.copy()
    for t in range(T):
        _, S = O.step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], S, lib=lib)
        for h in range(HV):
            assert np.allclose(S[0, h] @ k[0, t, h // (HV // HK)], v[0, t, h], atol=1e-12)
    o, hT = O.prefill(q, k, v, g, beta, h0=h0, lib=lib)
    for h in range(HV):
        assert np.allclose(hT[0, h] @ k[0, -1, h // (HV // HK)], v[0, -1, h], atol=1e-12)
    assert np.allclose(hT, S, atol=1e-12)


def pin_full_decay_resets(lib=None):
    """alpha = 0 (g -> -inf): everything before is forgotten, S_t = b_t v_t k_t^T."""
    rng = np.random.default_rng(4)
    q, k, v, g, beta = _rand_problem(rng, 6, 1, 2, 5, 4)
    g[:] = -1.0e4  # exp underflows to exactly 0
    h0 = rng.standard_normal((1, 2, 4, 5))
    for chunked in (False, True):
        o, hT = O.prefill(q, k, v, g, beta, h0=h0, chunked=chunked, chunk=3, lib=lib)
        for h in range(2):
            S_last = beta[0, -1, h] * np.outer(v[0, -1, h], k[0, -1, 0])
            assert np.allclose(hT[0, h], S_last, atol=1e-13)
            for t in range(6):
                St = beta[0, t, h] * np.outer(v[0, t, h], k[0, t, 0])
                assert np.allclose(o[t, h], St @ q[0, t, 0], atol=1e-13)


def pin_orthonormal_keys_store(lib=None):
    """alpha = beta = 1 and the keys run through an orthonormal basis: after the
    writes S e_j = v_j for each written direction (a plain associative store)."""
    rng = np.random.default_rng(5)
    dk, dv = 6, 5
    # a random orthonormal basis, written in order
    Qb, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qb.T
    T = dk
    k = keys.reshape(1, T, 1, dk)
    q = rng.standard_normal((1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    g = np.zeros((1, T, 1)); beta = np.ones((1, T, 1))
    h0 = rng.standard_normal((1, 1, dv, dk))
    for chunked in (False, True):
        _, hT = O.prefill(q, k, v, g, beta, h0=h0, chunked=chunked, chunk=4, lib=lib)
        assert np.allclose(hT[0, 0] @ keys.T, v[0, :, 0].T, atol=1e-12)


def pin_norm_bound(lib=None):
    """For b in [0,1] and unit k, I - b k k^T has spectral norm <= 1, hence
    ||S_t||_2 <= a_t ||S_{t-1}||_2 + b_t ||v_t||."""
    rng = np.random.default_rng(6)
    q, k, v, g, beta = _rand_problem(rng, 30, 1, 1, 8, 8, g_range=(-0.3, 0.0))
    S = rng.standard_normal((1, 1, 8, 8))
    for t in range(30):
        prev = np.linalg.norm(S[0, 0], 2)
        _, S = O.step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], S, lib=lib)
        bound = math.exp(g[0, t, 0]) * prev + beta[0, t, 0] * np.linalg.norm(v[0, t, 0])
        assert np.linalg.norm(S[0, 0], 2) <= bound * (1 + 1e-12)


# ----------------------------------------------------------------------------
# Two independent forms must agree (brute force on tiny inputs)
# ----------------------------------------------------------------------------
def pin_chunked_equals_sequential(lib=None):
    rng = np.random.default_rng(7)
    for (T, HK, HV, dk, dv) in [(1, 1, 1, 1, 1), (13, 1, 2, 4, 4), (37, 2, 4, 8, 5),
                                (64, 1, 2, 8, 8), (50, 2, 2, 3, 7)]:
        q, k, v, g, beta = _rand_problem(rng, T, HK, HV, dk, dv, g_range=(-0.5, 0.0))
        h0 = rng.standard_normal((1, HV, dv, dk))
        o_ref, h_ref = O.prefill(q, k, v, g, beta, h0=h0, lib=lib)
        for C in (1, 2, 3, 4, 16, max(T, 1)):
            o, h = O.prefill(q, k, v, g, beta, h0=h0, chunked=True, chunk=C, lib=lib)
            assert np.allclose(o, o_ref, atol=1e-11, rtol=0), (T, C, np.abs(o - o_ref).max())
            assert np.allclose(h, h_ref, atol=1e-11, rtol=0), (T, C)


def pin_strong_decay_no_overflow(lib=None):
    """g = -30 on some tokens (decay e^-30): the chunked form must not overflow."""
    rng = np.random.default_rng(8)
    q, k, v, g, beta = _rand_problem(rng, 40, 1, 2, 6, 6)
    g[0, ::7, :] = -30.0
    g[0, 5, 1] = -80.0
    o_ref, h_ref = O.prefill(q, k, v, g, beta, lib=lib)
    o, h = O.prefill(q, k, v, g, beta, chunked=True, chunk=16, lib=lib)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(h))
    assert np.allclose(o, o_ref, atol=1e-11) and np.allclose(h, h_ref, atol=1e-11)


# ----------------------------------------------------------------------------
# Structure: packing, splitting, decode, linearity, head symmetry
# ----------------------------------------------------------------------------
def pin_varlen_equals_separate(lib=None):
    rng = np.random.default_rng(9)
    lens = [5, 1, 17, 9]
    HK, HV, dk, dv = 1, 2, 4, 3
    parts = [_rand_problem(rng, L, HK, HV, dk, dv) for L in lens]
    h0 = rng.standard_normal((len(lens), HV, dv, dk))
    cat = [np.concatenate([p[i] for p in parts], axis=1) for i in range(5)]
    cu = np.concatenate([[0], np.cumsum(lens)])
    for chunked in (False, True):
        o, hT = O.prefill(*cat, h0=h0, cu_seqlens=cu, chunked=chunked, chunk=4, lib=lib)
        for n, p in enumerate(parts):
            on, hn = O.prefill(*p, h0=h0[n:n + 1], chunked=False, lib=lib)
            assert np.allclose(o[cu[n]:cu[n + 1]], on, atol=1e-12)
            assert np.allclose(hT[n], hn[0], atol=1e-12)


def pin_split_resume(lib=None):
    """prefill(T1) then prefill(T2, h0 = hT1) equals prefill(T1 + T2)."""
    rng = np.random.default_rng(10)
    q, k, v, g, beta = _rand_problem(rng, 23, 2, 4, 5, 5)
    h0 = rng.standard_normal((1, 4, 5, 5))
    o, hT = O.prefill(q, k, v, g, beta, h0=h0, lib=lib)
    a = [x[:, :10] for x in (q, k, v, g, beta)]
    b = [x[:, 10:] for x in (q, k, v, g, beta)]
    o1, h1 = O.prefill(*a, h0=h0, lib=lib)
    o2, h2 = O.prefill(*b, h0=h1, chunked=True, chunk=4, lib=lib)
    assert np.allclose(np.concatenate([o1, o2]), o, atol=1e-12)
    assert np.allclose(h2, hT, atol=1e-12)


def pin_decode_equals_prefill(lib=None):
    rng = np.random.default_rng(11)
    q, k, v, g, beta = _rand_problem(rng, 11, 2, 4, 6, 6)
    h0 = rng.standard_normal((1, 4, 6, 6))
    o, hT = O.prefill(q, k, v, g, beta, h0=h0, chunked=True, chunk=4, lib=lib)
    S = h0
    for t in range(11):
        ot, S = O.step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], S, lib=lib)
        assert np.allclose(ot[0], o[t], atol=1e-12)
    assert np.allclose(S, hT, atol=1e-12)


def pin_linear_in_values_and_state(lib=None):
    """For fixed q, k, g, beta the map (V, h0) -> (O, hT) is linear."""
    rng = np.random.default_rng(12)
    q, k, v1, g, beta = _rand_problem(rng, 15, 1, 2, 4, 4)
    v2 = rng.standard_normal(v1.shape)
    h1 = rng.standard_normal((1, 2, 4, 4)); h2 = rng.standard_normal((1, 2, 4, 4))
    a, b = 0.7, -1.3
    oa, ha = O.prefill(q, k, v1, g, beta, h0=h1, lib=lib)
    ob, hb = O.prefill(q, k, v2, g, beta, h0=h2, lib=lib)
    oc, hc = O.prefill(q, k, a * v1 + b * v2, g, beta, h0=a * h1 + b * h2, chunked=True,
                       chunk=4, lib=lib)
    assert np.allclose(oc, a * oa + b * ob, atol=1e-12)
    assert np.allclose(hc, a * ha + b * hb, atol=1e-12)


def pin_swap_value_heads(lib=None):
    """The two value heads of one query/key head are interchangeable."""
    rng = np.random.default_rng(13)
    q, k, v, g, beta = _rand_problem(rng, 12, 1, 2, 4, 4)
    h0 = rng.standard_normal((1, 2, 4, 4))
    o, hT = O.prefill(q, k, v, g, beta, h0=h0, lib=lib)
    o2, h2 = O.prefill(q, k, v[:, :, ::-1], g[:, :, ::-1], beta[:, :, ::-1],
                       h0=h0[:, ::-1], lib=lib)
    assert np.allclose(o2, o[:, ::-1], atol=1e-13)
    assert np.allclose(h2, hT[:, ::-1], atol=1e-13)


def pin_scale_multiplies_readout(lib=None):
    rng = np.random.default_rng(14)
    q, k, v, g, beta = _rand_problem(rng, 8, 1, 1, 4, 4)
    o1, h1 = O.prefill(q, k, v, g, beta, lib=lib)
    o2, h2 = O.prefill(q, k, v, g, beta, scale=0.25, lib=lib)
    assert np.allclose(o2, 0.25 * o1, atol=1e-14) and np.allclose(h2, h1, atol=1e-14)


def pin_verify_equals_prefill_of_drafts(lib=None):
    """Checking K drafts at once gives, for every draft j, the outputs and the
    state that a chunked prefill (the independent WY form) of the first j+1
    drafts gives from the same start state."""
    rng = np.random.default_rng(15)
    N, K, HK, HV, d = 3, 5, 2, 4, 6
    probs = [_rand_problem(rng, K, HK, HV, d, d) for _ in range(N)]
    q, k, v, g, beta = (np.concatenate([p_[i] for p_ in probs]) for i in range(5))
    S0 = rng.standard_normal((N, HV, d, d))
    o, states = O.verify(q, k, v, g, beta, S0, scale=0.5, lib=lib)
    assert o.shape == (N, K, HV, d) and states.shape == (N, K, HV, d, d)
    for n in range(N):
        for j in range(K):
            op, hp = O.prefill(q[n:n + 1, :j + 1], k[n:n + 1, :j + 1], v[n:n + 1, :j + 1],
                               g[n:n + 1, :j + 1], beta[n:n + 1, :j + 1], h0=S0[n:n + 1],
                               scale=0.5, chunked=True, chunk=2, lib=lib)
            assert np.allclose(o[n, j], op[j], atol=1e-12)
            assert np.allclose(states[n, j], hp[0], atol=1e-12)


def pin_commit_rolls_back_to_accepted_prefix(lib=None):
    rng = np.random.default_rng(16)
    N, K, HV, d = 3, 4, 2, 5
    probs = [_rand_problem(rng, K, 1, HV, d, d) for _ in range(N)]
    q, k, v, g, beta = (np.concatenate([p_[i] for p_ in probs]) for i in range(5))
    S0 = rng.standard_normal((N, HV, d, d))
    _, states = O.verify(q, k, v, g, beta, S0, lib=lib)
    accepted = [0, 2, K]
    S = O.commit(states, accepted, S0)
    assert np.array_equal(S[0], S0[0])
    for n in (1, 2):
        _, hp = O.prefill(q[n:n + 1, :accepted[n]], k[n:n + 1, :accepted[n]],
                          v[n:n + 1, :accepted[n]], g[n:n + 1, :accepted[n]],
                          beta[n:n + 1, :accepted[n]], h0=S0[n:n + 1], lib=lib)
        assert np.allclose(S[n], hp[0], atol=1e-12)


# ----------------------------------------------------------------------------
# The input prologue (L2-normalised keys and queries, sigmoid gates)
# ----------------------------------------------------------------------------
def pin_prologue_normalises_rows(lib=None):
    """Normalised rows have unit length and point along the raw row; each flag
    touches only its own tensor; a zero row stays zero (no division by 0)."""
    rng = np.random.default_rng(21)
    q = rng.standard_normal((2, 5, 3, 7)) * rng.uniform(0.1, 9.0, (2, 5, 3, 1))
    k = rng.standard_normal((2, 5, 3, 7)) * rng.uniform(0.1, 9.0, (2, 5, 3, 1))
    k[0, 1, 2] = 0.0
    g, b = rng.standard_normal((2, 5, 6)), rng.standard_normal((2, 5, 6))
    qn, kn, g2, b2 = O.prologue(q, k, g, b, O.PROLOGUE_NORM_Q | O.PROLOGUE_NORM_K)
    assert np.array_equal(g2, g) and np.array_equal(b2, b)
    assert np.allclose(np.linalg.norm(qn, axis=-1), 1.0, atol=1e-14)
    nk = np.linalg.norm(kn, axis=-1)
    assert np.all(kn[0, 1, 2] == 0.0)
    nk[0, 1, 2] = 1.0
    assert np.allclose(nk, 1.0, atol=1e-14)
    # parallel to the raw rows: <x_hat, x> = |x|
    assert np.allclose(np.sum(qn * q, -1), np.linalg.norm(q, axis=-1), rtol=1e-13)
    qn2, kn2, _, _ = O.prologue(q, k, g, b, O.PROLOGUE_NORM_K)
    assert np.array_equal(qn2, q) and np.array_equal(kn2, kn)
    qn3, kn3, _, _ = O.prologue(q, k, g, b, O.PROLOGUE_NORM_Q)
    assert np.array_equal(kn3, k) and np.array_equal(qn3, qn)


def pin_prologue_gates(lib=None):
    """beta = sigmoid(b): 1/2 at 0 and beta(b) + beta(-b) = 1; alpha = exp(g) =
    sigmoid(a): alpha / (1 - alpha) = e^a; the saturated ends stay finite
    (g -> 0 for a >> 0, g -> a for a << 0)."""
    a = np.array([-60.0, -3.0, -0.5, 0.0, 0.7, 4.0, 60.0])
    b = np.array([0.0, 1.0, -1.0, 2.5, -2.5, 30.0, -30.0])
    _, _, g, beta = O.prologue(np.zeros(2), np.zeros(2), a, b, O.PROLOGUE_GATE_LOGITS)
    assert beta[0] == 0.5
    assert abs(beta[1] + beta[2] - 1.0) < 1e-15 and abs(beta[3] + beta[4] - 1.0) < 1e-15
    assert np.all((beta > 0) & (beta < 1)) and beta[5] > 1 - 1e-12 and beta[6] < 1e-12
    alpha = np.exp(g)
    mid = slice(1, 6)
    assert np.allclose(np.log(alpha[mid] / (1.0 - alpha[mid])), a[mid], atol=1e-12)
    assert np.all(g <= 0.0) and np.all(np.isfinite(g))
    assert abs(g[-1]) < 1e-25 and abs(g[0] - a[0]) < 1e-20
    assert g[3] == -math.log(2.0)


def pin_prologue_then_rule_is_scale_free(lib=None):
    """With both norms on, scaling a token's raw q or k by any positive factor
    leaves the outputs and state unchanged; with them off, a scaled key changes
    the result (so the flag really feeds the rule)."""
    rng = np.random.default_rng(22)
    q, k, v, _, _ = _rand_problem(rng, 9, 1, 2, 5, 4, unit=False)
    a = rng.normal(2.0, 1.0, (1, 9, 2))
    b = rng.standard_normal((1, 9, 2))
    flags = O.PROLOGUE_NORM_Q | O.PROLOGUE_NORM_K | O.PROLOGUE_GATE_LOGITS
    s_q = rng.uniform(0.2, 5.0, (1, 9, 1, 1))
    s_k = rng.uniform(0.2, 5.0, (1, 9, 1, 1))
    o1, h1 = O.prefill(*O.prologue(q, k, a, b, flags)[:2], v, *O.prologue(q, k, a, b, flags)[2:],
                       lib=lib)
    qq, kk, gg, bb = O.prologue(q * s_q, k * s_k, a, b, flags)
    o2, h2 = O.prefill(qq, kk, v, gg, bb, lib=lib)
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(h1, h2, atol=1e-12)
    q3, k3, g3, b3 = O.prologue(q, k * s_k, a, b, O.PROLOGUE_NORM_Q | O.PROLOGUE_GATE_LOGITS)
    o3, _ = O.prefill(q3, k3, v, g3, b3, lib=lib)
    assert not np.allclose(o1, o3, atol=1e-6)


# ----------------------------------------------------------------------------
# One decay per value row (the teaching code's per-channel forget gate)
# ----------------------------------------------------------------------------
def pin_row_decay_worked_examples(lib=None):
    """The pages' scalar examples, one per row of a 2 x 1 state: row 0 without
    decay goes 6 -> 8 -> 9, row 1 with decay 0.5 goes 6 -> 3 -> 6.5, then (no
    decay) 6.5 -> 8.25, with the same key, target 10 and write strength 0.5."""
    S0 = np.array([[[[6.0], [6.0]]]])                      # [N=1][HV=1][dv=2][dk=1]
    one = np.ones((1, 1, 1))
    v = np.full((1, 1, 2), 10.0)
    beta = np.full((1, 1), 0.5)
    g1 = np.log(np.array([[[1.0, 0.5]]]))
    _, S1 = O.step_row_decay(one, one, v, g1, beta, S0)
    assert np.array_equal(S1[0, 0, :, 0], [8.0, 6.5])
    _, S2 = O.step_row_decay(one, one, v, np.zeros((1, 1, 2)), beta, S1)
    assert np.array_equal(S2[0, 0, :, 0], [9.0, 8.25])


def pin_row_decay_equal_rows_is_the_scalar_rule(lib=None):
    """All rows of a head sharing one decay reproduce the scalar-decay oracle
    (the independent C implementation)."""
    rng = np.random.default_rng(23)
    N, HK, HV, dk, dv = 3, 2, 4, 5, 6
    q, k, v, g, beta = _rand_problem(rng, N, HK, HV, dk, dv)
    q, k, v, g, beta = q[0], k[0], v[0], g[0], beta[0]     # N tokens -> N sequences
    S0 = rng.standard_normal((N, HV, dv, dk))
    o1, S1 = O.step(q, k, v, g, beta, S0, scale=0.7, lib=lib)
    o2, S2 = O.step_row_decay(q, k, v, np.repeat(g[:, :, None], dv, axis=2), beta, S0,
                              scale=0.7)
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(S1, S2, atol=1e-12)


def pin_row_decay_rows_are_independent(lib=None):
    """Permuting the value rows (state rows, values and decays together)
    permutes the outputs and the new state the same way; changing one row's
    decay changes only that row."""
    rng = np.random.default_rng(24)
    q, k = rng.standard_normal((2, 1, 4)), rng.standard_normal((2, 1, 4))
    v = rng.standard_normal((2, 2, 5))
    g = rng.uniform(np.log(0.5), 0.0, (2, 2, 5))
    beta = rng.uniform(0.1, 0.9, (2, 2))
    S0 = rng.standard_normal((2, 2, 5, 4))
    perm = np.array([3, 0, 4, 1, 2])
    o, S = O.step_row_decay(q, k, v, g, beta, S0)
    op, Sp = O.step_row_decay(q, k, v[:, :, perm], g[:, :, perm], beta, S0[:, :, perm])
    assert np.allclose(op, o[:, :, perm], atol=1e-13) and np.allclose(Sp, S[:, :, perm], atol=1e-13)
    g2 = g.copy()
    g2[1, 0, 2] -= 0.3
    o2, S2 = O.step_row_decay(q, k, v, g2, beta, S0)
    changed = ~np.isclose(S2, S, atol=1e-14).all(axis=-1)
    assert changed[1, 0, 2] and changed.sum() == 1


def pin_prefill_row_decay(lib=None):
    """The sequential prefill with per-row decay equals the scalar C oracle when
    every row shares its head's decay (packed sequences, nonzero h0), and equals
    a run of ``step_row_decay`` calls with different decays per row."""
    rng = np.random.default_rng(26)
    q, k, v, g, beta = _rand_problem(rng, 9, 2, 4, 5, 3)
    cu = np.array([0, 4, 9], dtype=np.int32)
    h0 = rng.standard_normal((2, 4, 3, 5))
    o1, h1 = O.prefill(q, k, v, g, beta, h0=h0, cu_seqlens=cu, scale=0.8, lib=lib)
    o2, h2 = O.prefill_row_decay(q, k, v, np.repeat(g[..., None], 3, axis=-1), beta, h0=h0,
                                 cu_seqlens=cu, scale=0.8)
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(h1, h2, atol=1e-12)
    gr = rng.uniform(np.log(0.5), 0.0, (1, 9, 4, 3))
    o3, h3 = O.prefill_row_decay(q[:, :4], k[:, :4], v[:, :4], gr[:, :4], beta[:, :4],
                                 h0=h0[:1], scale=0.8)
    S = h0[:1]
    for t in range(4):
        ot, S = O.step_row_decay(q[:, t], k[:, t], v[:, t], gr[:, t], beta[:, t], S, scale=0.8)
        assert np.allclose(o3[t], ot[0], atol=1e-13)
    assert np.allclose(h3, S, atol=1e-13)


def pin_verify_row_decay_equals_steps(lib=None):
    rng = np.random.default_rng(25)
    N, K, HK, HV, dk, dv = 2, 3, 1, 2, 4, 3
    q, k = rng.standard_normal((N, K, HK, dk)), rng.standard_normal((N, K, HK, dk))
    v = rng.standard_normal((N, K, HV, dv))
    g = rng.uniform(np.log(0.6), 0.0, (N, K, HV, dv))
    beta = rng.uniform(0.1, 0.9, (N, K, HV))
    S0 = rng.standard_normal((N, HV, dv, dk))
    o, states = O.verify_row_decay(q, k, v, g, beta, S0, scale=0.5)
    S = S0
    for t in range(K):
        ot, S = O.step_row_decay(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], S, scale=0.5)
        assert np.array_equal(o[:, t], ot) and np.array_equal(states[:, t], S)



# ----------------------------------------------------------------------------
# The short convolution on the values and the output gate around the rule
# ("Qwen3-Next 80B-A3B -- The Evolving Transformer", llamasearch.dev, section 01
# GatedDeltaNet; widths and forms are readings, see the oracle's section header)
# ----------------------------------------------------------------------------
def pin_short_conv_is_a_library_convolution(lib=None):
    """Per channel the causal convolution equals numpy's full convolution of the
    input (with the carried state in front) with the reversed kernel, cut to the
    sequence's tokens; with no state the missing history is zero."""
    rng = np.random.default_rng(31)
    B, T, C, W = 2, 11, 5, 4
    x = rng.standard_normal((B, T, C))
    w = rng.standard_normal((C, W))
    st = rng.standard_normal((B, W - 1, C))
    y0, _ = O.short_conv(x, w)
    y1, _ = O.short_conv(x, w, conv_state=st)
    for b in range(B):
        for c in range(C):
            ref0 = np.convolve(x[b, :, c], w[c, ::-1])[:T]
            full = np.concatenate([st[b, :, c], x[b, :, c]])
            ref1 = np.convolve(full, w[c, ::-1])[W - 1:W - 1 + T]
            assert np.allclose(y0[b * T:(b + 1) * T, c], ref0, atol=1e-13)
            assert np.allclose(y1[b * T:(b + 1) * T, c], ref1, atol=1e-13)


def pin_short_conv_impulse_response(lib=None):
    """A unit impulse at token t0 of channel c comes out as the kernel read
    backwards: y_{t0+d} = w[c, W-1-d] for d < W, zero before t0 and after
    t0+W-1 and on every other channel; the bias adds a constant; SiLU maps 0 to
    0 and 1 to 1/(1+e^-1)."""
    C, W, T, t0, c = 3, 4, 10, 3, 1
    w = np.arange(1.0, C * W + 1).reshape(C, W)
    x = np.zeros((1, T, C))
    x[0, t0, c] = 1.0
    y, st = O.short_conv(x, w)
    expect = np.zeros((T, C))
    for d in range(W):
        expect[t0 + d, c] = w[c, W - 1 - d]
    assert np.array_equal(y, expect)
    assert np.array_equal(st[0], x[0, T - (W - 1):])
    bias = np.array([0.5, -1.0, 2.0])
    yb, _ = O.short_conv(x, w, bias=bias)
    assert np.array_equal(yb, expect + bias)
    ys, _ = O.short_conv(x, w, activation="silu")
    assert ys[0, 0] == 0.0
    one = np.zeros((1, 1, 1))
    one[0, 0, 0] = 1.0
    y1, _ = O.short_conv(one, np.ones((1, 1)), activation="silu")
    assert abs(y1[0, 0] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15


def pin_short_conv_state_carry(lib=None):
    """Cutting a sequence anywhere (also before W-1 tokens) and carrying the
    state gives the same outputs and final state as one call; packed sequences
    with cu_seqlens equal separate calls, an empty sequence passes its state
    through unchanged."""
    rng = np.random.default_rng(32)
    T, C, W = 9, 3, 4
    x = rng.standard_normal((1, T, C))
    w = rng.standard_normal((C, W))
    b = rng.standard_normal(C)
    st = rng.standard_normal((1, W - 1, C))
    y, s_end = O.short_conv(x, w, b, st, activation="silu")
    for a in range(T + 1):
        ya, sa = O.short_conv(x[:, :a], w, b, st, activation="silu")
        yb, sb = O.short_conv(x[:, a:], w, b, sa, activation="silu")
        assert np.allclose(np.concatenate([ya, yb]), y, atol=1e-14)
        assert np.allclose(sb, s_end, atol=0.0)
    lens = [4, 0, 1, 7]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    xp = rng.standard_normal((1, int(cu[-1]), C))
    stp = rng.standard_normal((len(lens), W - 1, C))
    yp, sp = O.short_conv(xp, w, b, stp, cu_seqlens=cu)
    for n, L in enumerate(lens):
        yn, sn = O.short_conv(xp[:, cu[n]:cu[n + 1]], w, b, stp[n:n + 1])
        assert np.array_equal(yp[cu[n]:cu[n + 1]], yn) and np.array_equal(sp[n], sn[0])
    assert np.array_equal(sp[1], stp[1])
    # one token: the state shifts by one and takes the token last
    assert np.array_equal(sp[2], np.concatenate([stp[2, 1:], xp[0, 4:5]]))


def pin_output_gate(lib=None):
    """sigmoid(0) = 1/2 halves the read-out; a large positive logit passes it,
    a large negative one closes it; gate(o, z) + gate(o, -z) = o."""
    rng = np.random.default_rng(33)
    o = rng.standard_normal((4, 3, 5))
    z = rng.standard_normal((4, 3, 5)) * 3.0
    assert np.array_equal(O.output_gate(o, np.zeros_like(o)), o / 2)
    assert np.allclose(O.output_gate(o, np.full_like(o, 40.0)), o, rtol=1e-15, atol=0)
    assert np.all(np.abs(O.output_gate(o, np.full_like(o, -40.0))) < 1e-17 * np.abs(o) + 1e-300)
    assert np.allclose(O.output_gate(o, z) + O.output_gate(o, -z), o, atol=1e-15)
    assert np.all(np.abs(O.output_gate(o, z)) <= np.abs(o))


def pin_layer_prefill_equals_layer_steps(lib=None):
    """The layer over a sequence (convolution, rule, gate) equals one decode
    step per token with both states carried; a pass-through kernel (last tap 1,
    others 0) with no gate is the plain rule."""
    rng = np.random.default_rng(34)
    N, T, HK, HV, dk, dv, W = 2, 6, 1, 2, 4, 3, 4
    q, k, v, g, beta = _rand_problem(rng, T, HK, HV, dk, dv)
    q, k, v, g, beta = (np.repeat(a, N, axis=0) * (1.0 + 0.1 * np.arange(N)).reshape(
        (N,) + (1,) * (a.ndim - 1)) if a is v else np.repeat(a, N, axis=0) for a in (q, k, v, g, beta))
    w = rng.standard_normal((HV * dv, W))
    cb = rng.standard_normal(HV * dv)
    cs = rng.standard_normal((N, W - 1, HV * dv))
    z = rng.standard_normal((N, T, HV, dv))
    h0 = rng.standard_normal((N, HV, dv, dk)) * 0.3
    o, hT, cs_end = O.layer_prefill(q, k, v, g, beta, w, cb, cs, z, h0=h0, scale=0.9,
                                    activation="silu")
    S, c = h0, cs
    for t in range(T):
        ot, S, c = O.layer_step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], S, w, cb, c,
                                z[:, t], scale=0.9, activation="silu")
        assert np.allclose(o.reshape(N, T, HV, dv)[:, t], ot, atol=1e-12)
    assert np.allclose(hT, S, atol=1e-12) and np.allclose(cs_end, c, atol=0.0)
    wid = np.zeros((HV * dv, W))
    wid[:, W - 1] = 1.0
    o1, h1, _ = O.layer_prefill(q, k, v, g, beta, wid, None, cs, None, h0=h0, scale=0.9)
    o2, h2 = O.prefill(q, k, v, g, beta, h0=h0, scale=0.9, lib=lib)
    assert np.allclose(o1, o2, atol=1e-12) and np.allclose(h1, h2, atol=1e-12)

ALL_PINS = [v for k_, v in sorted(globals().items()) if k_.startswith("pin_")]
