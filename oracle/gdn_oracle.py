"""Float64 CPU oracle for the gated delta rule (Python side).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module.  The
product path (the CUDA library and its binding) never imports it and shares no
code with it.

The arithmetic lives in ``gdn_oracle.c`` (plain C, float64, one thread per
(sequence, value head) unit); this module only builds that file with gcc,
converts inputs to contiguous float64 numpy arrays and calls it.  See the C
file's header for the rule it follows and the pages it cites:

* the delta rule with decay applied first ("Qwen3-Next", sghael.github.io,
  section "Correcting a memory instead of adding to it"),
* 32 value heads reading 16 query/key heads at head dim 128 (model card
  "Qwen3-Next-80B-A3B-Instruct", section "Model Overview"),
* read-out after the update, state rows indexed by the value dimension
  ("The Evolving Transformer / Qwen3-Next", section 01 GatedDeltaNet),
* the prologue that turns a layer's raw projections into the rule's inputs
  (``prologue``, plain numpy: L2-normalised keys and sigmoid gates, same
  section of the same page).

Every function here has its result pinned by ``tests/test_oracle_pins.py``
against values the pages print, closed forms, invariants and the agreement of
the two independent forms (sequential definition vs. chunkwise WY form).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "libgdn_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no fast-math) into ``libgdn_oracle.so``."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-std=c11", "-fPIC",
             "-shared", "-pthread", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(lib):
    lib.gdn_oracle_prefill.restype = ctypes.c_int
    lib.gdn_oracle_prefill.argtypes = [
        _dp, _dp, _dp, _dp, _dp, _dp, _i64p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_int, ctypes.c_double, _dp, _dp, ctypes.c_int]
    lib.gdn_oracle_prefill_chunked.restype = ctypes.c_int
    lib.gdn_oracle_prefill_chunked.argtypes = [
        _dp, _dp, _dp, _dp, _dp, _dp, _i64p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, _dp, _dp, ctypes.c_int]
    lib.gdn_oracle_step.restype = ctypes.c_int
    lib.gdn_oracle_step.argtypes = [
        _dp, _dp, _dp, _dp, _dp, _dp, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_int, ctypes.c_double, _dp]
    return lib


def _load(path=None):
    """The oracle library; ``path`` selects another build of the same C source
    (the mutation tests load deliberately broken copies this way)."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: exact upcast (bf16/fp32 -> fp64 is exact)
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def _flatten_tokens(q, k, v, g, beta, cu_seqlens):
    """Accept [B,T,H,d] (+ no cu_seqlens) or packed [1,Ttot,H,d] / [Ttot,H,d] + cu_seqlens."""
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    if q.ndim == 4:
        B, T = q.shape[0], q.shape[1]
        q = q.reshape(B * T, *q.shape[2:])
        k = k.reshape(B * T, *k.shape[2:])
        v = v.reshape(B * T, *v.shape[2:])
        g = g.reshape(B * T, -1)
        beta = beta.reshape(B * T, -1)
    else:
        B, T = 1, q.shape[0]
    if cu_seqlens is None:
        cu = np.arange(0, B * T + 1, T, dtype=np.int64) if T > 0 else np.zeros(B + 1, np.int64)
    else:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    return q, k, v, g, beta, cu


def prefill(q, k, v, g, beta, h0=None, cu_seqlens=None, scale=1.0, nthreads=0,
            chunked=False, chunk=64, lib=None):
    """Run the oracle over a batch.

    Shapes: q,k [B,T,HK,dk]; v [B,T,HV,dv]; g,beta [B,T,HV]; or packed
    [1,Ttot,...] with ``cu_seqlens`` (N+1 offsets).  h0 [N,HV,dv,dk] or None.
    Returns (o [Ttot or B*T, HV, dv] float64, hT [N,HV,dv,dk] float64).
    ``chunked=True`` runs the chunkwise WY form instead of the definition.
    """
    q, k, v, g, beta, cu = _flatten_tokens(q, k, v, g, beta, cu_seqlens)
    Ttot, HK, dk = q.shape
    HV, dv = v.shape[1], v.shape[2]
    N = cu.shape[0] - 1
    h0 = _f64(h0)
    if h0 is not None:
        h0 = h0.reshape(N, HV, dv, dk)
    o = np.zeros((Ttot, HV, dv), dtype=np.float64)
    hT = np.zeros((N, HV, dv, dk), dtype=np.float64)
    lib = lib or _load()
    if chunked:
        rc = lib.gdn_oracle_prefill_chunked(
            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
            cu.ctypes.data_as(_i64p), N, HK, HV, dk, dv, int(chunk), float(scale),
            _ptr(o), _ptr(hT), int(nthreads))
    else:
        rc = lib.gdn_oracle_prefill(
            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
            cu.ctypes.data_as(_i64p), N, HK, HV, dk, dv, float(scale),
            _ptr(o), _ptr(hT), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (rc={rc})")
    return o, hT


def step(q, k, v, g, beta, state, scale=1.0, lib=None):
    """One decode token per sequence.  q,k [N,HK,dk]; v [N,HV,dv]; g,beta [N,HV];
    state [N,HV,dv,dk].  Returns (o [N,HV,dv], new_state) as float64 arrays."""
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    S = _f64(state).copy()
    N, HK, dk = q.shape
    HV, dv = v.shape[1], v.shape[2]
    o = np.zeros((N, HV, dv), dtype=np.float64)
    rc = (lib or _load()).gdn_oracle_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S),
                                 N, HK, HV, dk, dv, float(scale), _ptr(o))
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (rc={rc})")
    return o, S


def verify(q, k, v, g, beta, state, scale=1.0, lib=None):
    """K draft tokens per sequence, checked at once (speculative decoding, where
    drafted tokens are verified together and only an accepted prefix is kept --
    "Qwen3-Next", sghael.github.io, section "Speed depends on the serving
    software").  The rule is applied token after token from ``state``; the
    outputs of every token and the state after every token are returned, so a
    caller can roll back to the state after the last accepted token.

    q,k [N,K,HK,dk]; v [N,K,HV,dv]; g,beta [N,K,HV]; state [N,HV,dv,dk].
    Returns (o [N,K,HV,dv], states [N,K,HV,dv,dk]) float64; ``state`` is not
    modified.
    """
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    S = _f64(state).copy()
    N, K = q.shape[0], q.shape[1]
    HV, dv, dk = S.shape[1], S.shape[2], S.shape[3]
    o = np.zeros((N, K, HV, dv), dtype=np.float64)
    states = np.zeros((N, K, HV, dv, dk), dtype=np.float64)
    for j in range(K):
        o[:, j], S = step(q[:, j], k[:, j], v[:, j], g[:, j], beta[:, j], S, scale=scale, lib=lib)
        states[:, j] = S
    return o, states


def commit(states, accepted, state):
    """Roll back to the accepted prefix: for each sequence n, the state after its
    accepted[n] draft tokens (states[n, accepted[n] - 1]), or ``state[n]``
    unchanged when none was accepted.  Returns the new [N,HV,dv,dk] array."""
    states, S = _f64(states), _f64(state).copy()
    for n, a in enumerate(np.asarray(accepted).tolist()):
        if a > 0:
            S[n] = states[n, a - 1]
    return S


# flags of the input prologue (same values as the C header's GDN_PROLOGUE_*)
PROLOGUE_NORM_Q = 1
PROLOGUE_NORM_K = 2
PROLOGUE_GATE_LOGITS = 4
NORM_EPS = 1e-12


def prologue(q, k, g, beta, flags):
    """The steps just before the recurrence, in float64 ("The Evolving
    Transformer / Qwen3-Next", section 01 GatedDeltaNet: keys are L2-normalised
    along the head dimension; the write strength is a sigmoid of its logit and
    the forget gate a sigmoid of its own logit).  Reading: one forget logit per
    token and value head (the hot path's scalar decay per head), and q is
    normalised like k when asked (the model's "L2-normalised q/k").

    flags & PROLOGUE_NORM_Q: q <- q / max(|q|, 1e-12) over the last axis
    flags & PROLOGUE_NORM_K: k <- k / max(|k|, 1e-12)
    flags & PROLOGUE_GATE_LOGITS: ``g`` holds the forget logits a and ``beta``
        the write logits b; returns g = log sigmoid(a) (so alpha = exp(g) =
        sigmoid(a)) and beta = sigmoid(b).
    Returns float64 (q, k, g, beta); inputs of other shapes pass through.
    """
    q, k, g, beta = (_f64(x) for x in (q, k, g, beta))
    if flags & PROLOGUE_NORM_Q:
        q = q / np.maximum(np.sqrt(np.sum(q * q, axis=-1, keepdims=True)), NORM_EPS)
    if flags & PROLOGUE_NORM_K:
        k = k / np.maximum(np.sqrt(np.sum(k * k, axis=-1, keepdims=True)), NORM_EPS)
    if flags & PROLOGUE_GATE_LOGITS:
        # log sigmoid(x) = -log(1 + e^-x), evaluated without overflow
        g = -np.logaddexp(0.0, -g)
        beta = np.exp(-np.logaddexp(0.0, -beta))
    return q, k, g, beta


def step_row_decay(q, k, v, g_rows, beta, state, scale=1.0):
    """One decode token with one decay per value row: the forget gate of the
    teaching code ("The Evolving Transformer / Qwen3-Next", section 01
    GatedDeltaNet) has one entry per channel of the value dimension and scales
    the rows of the state.  Row i of every (sequence, value head) state:
        S_i <- alpha_i S_i                  (decay first, as in the scalar rule)
        S_i <- S_i + beta (v_i - S_i . k) k^T
        o_i  = scale * S_i . q
    q,k [N,HK,dk]; v [N,HV,dv]; g_rows [N,HV,dv] (alpha = exp(g)); beta [N,HV];
    state [N,HV,dv,dk].  Plain float64 loops; returns (o [N,HV,dv], new_state)."""
    q, k, v, g_rows, beta = (_f64(x) for x in (q, k, v, g_rows, beta))
    S = _f64(state).copy()
    N, HK, dk = q.shape
    HV, dv = v.shape[1], v.shape[2]
    o = np.zeros((N, HV, dv))
    for n in range(N):
        for h in range(HV):
            c = h // (HV // HK)
            kt, qt = k[n, c], q[n, c]
            for i in range(dv):
                row = S[n, h, i] * np.exp(g_rows[n, h, i])
                row = row + beta[n, h] * (v[n, h, i] - row @ kt) * kt
                S[n, h, i] = row
                o[n, h, i] = scale * (row @ qt)
    return o, S


def verify_row_decay(q, k, v, g_rows, beta, state, scale=1.0):
    """``verify`` with one decay per value row: K calls of ``step_row_decay``.
    q,k [N,K,HK,dk]; v, g_rows [N,K,HV,dv]; beta [N,K,HV]; state [N,HV,dv,dk]."""
    q, k, v, g_rows, beta = (_f64(x) for x in (q, k, v, g_rows, beta))
    S = _f64(state).copy()
    N, K = q.shape[:2]
    HV, dv, dk = S.shape[1], S.shape[2], S.shape[3]
    o = np.zeros((N, K, HV, dv))
    states = np.zeros((N, K, HV, dv, dk))
    for t in range(K):
        o[:, t], S = step_row_decay(q[:, t], k[:, t], v[:, t], g_rows[:, t], beta[:, t], S, scale)
        states[:, t] = S
    return o, states


def prefill_row_decay(q, k, v, g_rows, beta, h0=None, cu_seqlens=None, scale=1.0):
    """Token-by-token prefill with one decay per value row (see ``step_row_decay``),
    float64, for small problems: q,k [B,T,HK,dk]; v, g_rows [B,T,HV,dv];
    beta [B,T,HV]; h0 [N,HV,dv,dk] or None; cu_seqlens as in ``prefill``.
    Returns (o [B*T,HV,dv], hT [N,HV,dv,dk])."""
    q, k, v, g_rows, beta = (_f64(x) for x in (q, k, v, g_rows, beta))
    B, T, HK, dk = q.shape
    HV, dv = v.shape[2], v.shape[3]
    if cu_seqlens is None:
        bounds = [(b * T, (b + 1) * T) for b in range(B)]
    else:
        cu = np.asarray(_f64(cu_seqlens)).astype(np.int64)
        bounds = [(int(cu[i]), int(cu[i + 1])) for i in range(len(cu) - 1)]
    flat = lambda x: x.reshape((B * T,) + x.shape[2:])
    q, k, v, g_rows, beta = (flat(x) for x in (q, k, v, g_rows, beta))
    N = len(bounds)
    S = np.zeros((N, HV, dv, dk)) if h0 is None else _f64(h0).copy()
    o = np.zeros((B * T, HV, dv))
    r = HV // HK
    for n, (s0, s1) in enumerate(bounds):
        for t in range(s0, s1):
            for h in range(HV):
                c = h // r
                St = S[n, h] * np.exp(g_rows[t, h])[:, None]        # decay each row
                u = beta[t, h] * (v[t, h] - St @ k[t, c])
                St = St + np.outer(u, k[t, c])
                S[n, h] = St
                o[t, h] = scale * (St @ q[t, c])
    return o, S


# ----------------------------------------------------------------------------
# The layer steps around the rule: a short convolution on the values before it
# and an output gate after it ("Qwen3-Next 80B-A3B -- The Evolving Transformer",
# llamasearch.dev, section 01 GatedDeltaNet, names both: a one-dimensional
# convolution gives the values local context, and a gate sets how much of what
# the recurrence returns reaches the output).
# The pages give neither the convolution's width nor the gate's form.  Reading:
#   * a causal depthwise convolution along time, one kernel of width W per
#     value channel (channel = h * dv + i), tap j multiplying the input W-1-j
#     tokens back, an optional bias and an optional SiLU after it; inputs
#     before a sequence's first token come from a carried convolution state
#     (the last W-1 inputs of the previous call) or are zero;
#   * an elementwise sigmoid gate on the read-out, o <- o * sigmoid(z), with
#     one gate logit per output element (the same page's attention layers use
#     a sigmoid gate).
# ----------------------------------------------------------------------------
def silu(x):
    """x * sigmoid(x) in float64, without overflow for large |x|."""
    x = _f64(x)
    return x * np.exp(-np.logaddexp(0.0, -x))


def short_conv(x, weight, bias=None, conv_state=None, cu_seqlens=None, activation="none"):
    """Causal depthwise convolution of each sequence along time.

    x [B,T,C] (B sequences of T tokens) or packed [1,Ttot,C] / [Ttot,C] with
    ``cu_seqlens`` (N+1 offsets); weight [C,W]; bias [C] or None; conv_state
    [N,W-1,C] (row m = the input W-1-m tokens before the sequence's first
    token) or None (zeros).  For token t of a sequence, with x_s = the input at
    token s (s < 0 read from the state):
        y_t = bias + sum_{j=0}^{W-1} weight[:, j] * x_{t-(W-1)+j}
    then SiLU when ``activation == "silu"``.
    Returns (y [Ttot,C], new_state [N,W-1,C]): the last W-1 inputs of each
    sequence, taken from the old state where the sequence is shorter than W-1.
    """
    x, w = _f64(x), _f64(weight)
    C, W = w.shape
    if cu_seqlens is None and x.ndim == 3:
        B, T = x.shape[0], x.shape[1]
        bounds = [(b * T, (b + 1) * T) for b in range(B)]
    else:
        cu = np.asarray(_f64(cu_seqlens)).astype(np.int64)
        bounds = [(int(cu[i]), int(cu[i + 1])) for i in range(len(cu) - 1)]
    x = x.reshape(-1, C)
    N = len(bounds)
    hist = np.zeros((N, W - 1, C)) if conv_state is None else _f64(conv_state).reshape(N, W - 1, C)
    b = np.zeros(C) if bias is None else _f64(bias)
    y = np.zeros_like(x)
    new_state = np.zeros((N, W - 1, C))
    for n, (s0, s1) in enumerate(bounds):
        L = s1 - s0
        xs = np.concatenate([hist[n], x[s0:s1]], axis=0)     # tokens s0-(W-1) .. s1-1
        acc = np.tile(b, (L, 1))
        for j in range(W):
            acc = acc + w[:, j] * xs[j:j + L]
        y[s0:s1] = silu(acc) if activation == "silu" else acc
        new_state[n] = xs[L:L + W - 1]
    return y, new_state


def output_gate(o, z):
    """o * sigmoid(z), elementwise, float64 (shapes must match)."""
    o, z = _f64(o), _f64(z)
    return o * np.exp(-np.logaddexp(0.0, -z))


def layer_prefill(q, k, v, g, beta, conv_weight=None, conv_bias=None, conv_state=None, z=None,
                  h0=None, cu_seqlens=None, scale=1.0, activation="none", flags=0):
    """The rule with the steps around it, over whole sequences: the prologue
    (``flags``), the short convolution on v (when ``conv_weight`` is given),
    the prefill, and the output gate (when ``z`` is given).  Shapes as in
    ``prefill``; conv_weight [HV*dv, W]; conv_state [N, W-1, HV*dv]; z like v.
    Returns (o [Ttot,HV,dv], hT, new_conv_state or None)."""
    q, k, g, beta = prologue(q, k, g, beta, flags)
    v = _f64(v)
    new_cs = None
    if conv_weight is not None:
        vs = v.shape
        C = vs[-2] * vs[-1]
        if cu_seqlens is None and v.ndim == 4:
            xv = v.reshape(vs[0], vs[1], C)
        else:
            xv = v.reshape(-1, C)
        vc, new_cs = short_conv(xv, conv_weight, conv_bias, conv_state, cu_seqlens, activation)
        v = vc.reshape(vs)
    o, hT = prefill(q, k, v, g, beta, h0=h0, cu_seqlens=cu_seqlens, scale=scale)
    if z is not None:
        o = output_gate(o, _f64(z).reshape(o.shape))
    return o, hT, new_cs


def layer_step(q, k, v, g, beta, state, conv_weight=None, conv_bias=None, conv_state=None,
               z=None, scale=1.0, activation="none", flags=0):
    """One decode token per sequence with the steps around the rule (see
    ``layer_prefill``).  q,k [N,HK,dk]; v, z [N,HV,dv]; g, beta [N,HV];
    state [N,HV,dv,dk]; conv_state [N,W-1,HV*dv].
    Returns (o [N,HV,dv], new_state, new_conv_state or None)."""
    q, k, g, beta = prologue(q, k, g, beta, flags)
    v = _f64(v)
    new_cs = None
    if conv_weight is not None:
        N, HV, dv = v.shape
        vc, new_cs = short_conv(v.reshape(N, 1, HV * dv), conv_weight, conv_bias, conv_state,
                                activation=activation)
        v = vc.reshape(N, HV, dv)
    o, S = step(q, k, v, g, beta, state, scale=scale)
    if z is not None:
        o = output_gate(o, z)
    return o, S, new_cs
