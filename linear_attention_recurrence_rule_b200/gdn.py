"""Thin Python binding of the C ABI in ``include/gdn.h`` (argument marshalling only).

Every step of the computation runs in the CUDA library ``libgdn_b200.so``; this
module turns torch tensors into device pointers, passes the current CUDA stream
and raises on a non-OK status.  PyTorch is used for device memory and streams
only.  If the library is missing, every call raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import _build

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_ALIGNMENT, GDN_ERR_CUDA, \
    GDN_ERR_TIMEOUT, GDN_ERR_WORKSPACE = range(7)
GDN_F32, GDN_BF16 = 0, 1
# input prologue flags (GDN_PROLOGUE_* in gdn.h)
PROLOGUE_NORM_Q, PROLOGUE_NORM_K, PROLOGUE_GATE_LOGITS = 1, 2, 4
PROLOGUE_ALL = 7
ROW_DECAY = 8   # one decay per value row: g [..., HV, dv] (GDN_ROW_DECAY)
CONV_SILU = 16  # SiLU after the short convolution (GDN_CONV_SILU)
CONV_MAX_WIDTH = 8

_lock = threading.Lock()
_handle = None


class GDNError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


def lib_path() -> str:
    return _build.LIB


def load_library() -> ctypes.CDLL:
    """Load ``libgdn_b200.so`` (raises if it has not been built)."""
    global _handle
    with _lock:
        if _handle is None:
            if not os.path.exists(_build.LIB):
                raise RuntimeError(
                    f"CUDA library {_build.LIB} is not built; run "
                    "`python -c 'import __graft_entry__ as g; g.build()'` first")
            lib = ctypes.CDLL(_build.LIB)
            vp, sz, i64, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64, ctypes.c_int
            lib.gdn_status_string.restype = ctypes.c_char_p
            lib.gdn_status_string.argtypes = [i32]
            lib.gdn_version.restype = i32
            lib.gdn_version.argtypes = []
            lib.gdn_chunk_prefill_workspace_size.restype = sz
            lib.gdn_chunk_prefill_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32, i32,
                                                             i32, i32]
            lib.gdn_chunk_prefill.restype = i32
            lib.gdn_chunk_prefill.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32,
                                              i32, i32, ctypes.c_float, i32, vp, vp, vp, sz, vp]
            lib.gdn_chunk_prefill_ex.restype = i32
            lib.gdn_chunk_prefill_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32,
                                                 i32, i32, i32, ctypes.c_float, i32, vp, vp, vp,
                                                 sz, ctypes.c_uint, vp]
            lib.gdn_recurrent_step_ex.restype = i32
            lib.gdn_recurrent_step_ex.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                                  i32, ctypes.c_float, i32, vp, ctypes.c_uint, vp]
            lib.gdn_recurrent_step.restype = i32
            lib.gdn_recurrent_step.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                               ctypes.c_float, i32, vp, vp]
            lib.gdn_recurrent_verify.restype = i32
            lib.gdn_recurrent_verify.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                                 i32, ctypes.c_float, i32, vp, vp, vp,
                                                 ctypes.c_uint, vp, sz, vp]
            lib.gdn_recurrent_verify_workspace_size.restype = sz
            lib.gdn_recurrent_verify_workspace_size.argtypes = [i32, i32, i32, i32]
            lib.gdn_recurrent_commit_verify.restype = i32
            lib.gdn_recurrent_commit_verify.argtypes = [vp, vp, vp, vp, i32, vp, vp, vp, vp, vp,
                                                        vp, i32, i32, i32, i32, i32, i32,
                                                        ctypes.c_float, i32, vp, vp,
                                                        ctypes.c_uint, vp, sz, vp]
            lib.gdn_recurrent_commit_verify_workspace_size.restype = sz
            lib.gdn_recurrent_commit_verify_workspace_size.argtypes = [i32, i32, i32, i32, i32]
            lib.gdn_state_commit.restype = i32
            lib.gdn_state_commit.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, vp]
            lib.gdn_state_commit_deltas.restype = i32
            lib.gdn_state_commit_deltas.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                                    i32, i32, ctypes.c_uint, vp]
            lib.gdn_chunk_prefill_path.restype = i32
            lib.gdn_chunk_prefill_path.argtypes = [i32, i32, i32, i32]
            lib.gdn_read_status.restype = i32
            lib.gdn_read_status.argtypes = [vp, sz, vp]
            lib.gdn_validate_cu_seqlens.restype = i32
            lib.gdn_validate_cu_seqlens.argtypes = [vp, i32, i64, vp, vp]
            lib.gdn_chunk_prefill_host_workspace_size.restype = sz
            lib.gdn_chunk_prefill_host_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32,
                                                                  i32, i32, i64]
            lib.gdn_chunk_prefill_host.restype = i32
            lib.gdn_chunk_prefill_host.argtypes = [vp, vp, vp, vp, vp, vp, i32, i64, i32, i32,
                                                   i32, i32, i32, ctypes.c_float, i32, vp, vp,
                                                   vp, sz, i64, vp, vp, vp]
            lib.gdn_short_conv.restype = i32
            lib.gdn_short_conv.argtypes = [vp, vp, vp, vp, vp, i32, i64, i32, i32, ctypes.c_uint,
                                           i32, vp, vp]
            lib.gdn_output_gate.restype = i32
            lib.gdn_output_gate.argtypes = [vp, vp, i64, i32, i32, vp]
            lib.gdn_recurrent_step_layer.restype = i32
            lib.gdn_recurrent_step_layer.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp,
                                                     i32, i32, i32, i32, i32, ctypes.c_float, i32,
                                                     vp, ctypes.c_uint, vp]
            lib.gdn_chunk_prefill_layer_workspace_size.restype = sz
            lib.gdn_chunk_prefill_layer_workspace_size.argtypes = [i32, i64, i32, i32, i32, i32,
                                                                   i32, i32, i32, i32, i32]
            lib.gdn_chunk_prefill_layer.restype = i32
            lib.gdn_chunk_prefill_layer.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i64, i32,
                                                    i32, i32, i32, i32, ctypes.c_float, i32, vp,
                                                    vp, vp, vp, vp, i32, vp, ctypes.c_uint, vp,
                                                    sz, vp]
            _handle = lib
    return _handle


def status_string(status: int) -> str:
    return load_library().gdn_status_string(int(status)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream, device):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def gdn_chunk_prefill_workspace_size(N, T, HK, HV, dk, dv, chunk, dtype, varlen) -> int:
    code = dtype if isinstance(dtype, int) else _dtype_code(torch.empty(0, dtype=dtype))
    return int(load_library().gdn_chunk_prefill_workspace_size(
        int(N), int(T), int(HK), int(HV), int(dk), int(dv), int(chunk), code, int(bool(varlen))))


def gdn_chunk_prefill(q, k, v, g, beta, h0=None, cu_seqlens=None, chunk: int = 64,
                      scale: float = 1.0, o=None, hT=None, workspace=None, stream=None,
                      output_final_state: bool = True, prologue: int = 0):
    """Chunkwise prefill through ``gdn_chunk_prefill``.

    q, k [B,T,HK,dk]; v [B,T,HV,dv] (bf16 or fp32); g, beta [B,T,HV] fp32;
    h0 [N,HV,dv,dk] fp32 or None; cu_seqlens int32 [N+1] (then B == 1) or None.
    ``prologue``: PROLOGUE_* flags fused into the kernels (L2-normalised q / k,
    g and beta given as logits).  Returns (o [B,T,HV,dv], hT [N,HV,dv,dk] or None).
    """
    lib = load_library()
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:2] != q.shape[:2]:
        raise ValueError("expected q,k [B,T,HK,dk] and v [B,T,HV,dv]")
    B, T, HK, dk = q.shape
    HV, dv = v.shape[2], v.shape[3]
    g_shape = (B, T, HV, dv) if prologue & ROW_DECAY else (B, T, HV)
    if g.shape != g_shape or beta.shape != (B, T, HV):
        raise ValueError(f"expected g {g_shape} and beta [B,T,HV]")
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
        if B != 1:
            raise ValueError("with cu_seqlens the batch dimension must be 1 (packed)")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    if h0 is not None:
        _need(h0, "h0", torch.float32, dev)
        if h0.shape != (N, HV, dv, dk):
            raise ValueError(f"h0 must be [N,HV,dv,dk] = {(N, HV, dv, dk)}")
    if o is None:
        o = torch.empty_like(v)
    else:
        _need(o, "o", v.dtype, dev)
    if hT is None and output_final_state:
        hT = torch.empty((N, HV, dv, dk), dtype=torch.float32, device=dev)
    elif hT is not None:
        _need(hT, "hT", torch.float32, dev)
    code = _dtype_code(q)
    need = lib.gdn_chunk_prefill_workspace_size(N, T, HK, HV, dk, dv, chunk, code,
                                                int(cu_seqlens is not None))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.gdn_chunk_prefill_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                                  _ptr(cu_seqlens), N, T, HK, HV, dk, dv, int(chunk),
                                  float(scale), code, _ptr(o), _ptr(hT), _ptr(workspace),
                                  ws_bytes, int(prologue), _stream_ptr(stream, dev))
    if st != GDN_OK:
        raise GDNError(st, "gdn_chunk_prefill")
    return o, hT


def gdn_recurrent_step(q, k, v, g, beta, state, scale: float = 1.0, o=None, stream=None,
                       prologue: int = 0):
    """One fused decode token through ``gdn_recurrent_step``; ``state`` is updated in place.

    q, k [N,HK,dk]; v [N,HV,dv] (bf16 or fp32); g, beta [N,HV] fp32;
    state [N,HV,dv,dk] fp32.  ``prologue``: PROLOGUE_* flags.  Returns o [N,HV,dv].
    """
    lib = load_library()
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(state, "state", torch.float32, dev)
    if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[0] != q.shape[0]:
        raise ValueError("expected q,k [N,HK,dk] and v [N,HV,dv]")
    N, HK, dk = q.shape
    HV, dv = v.shape[1], v.shape[2]
    g_shape = (N, HV, dv) if prologue & ROW_DECAY else (N, HV)
    if g.shape != g_shape or beta.shape != (N, HV) or state.shape != (N, HV, dv, dk):
        raise ValueError(f"expected g {g_shape}, beta [N,HV] and state [N,HV,dv,dk]")
    if o is None:
        o = torch.empty_like(v)
    else:
        _need(o, "o", v.dtype, dev)
    st = lib.gdn_recurrent_step_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state),
                                   N, HK, HV, dk, dv, float(scale), _dtype_code(q), _ptr(o),
                                   int(prologue), _stream_ptr(stream, dev))
    if st != GDN_OK:
        raise GDNError(st, "gdn_recurrent_step")
    return o


def gdn_recurrent_verify(q, k, v, g, beta, state, scale: float = 1.0, o=None, states_out=None,
                         u_out=None, rollback="states", stream=None, prologue: int = 0,
                         workspace=None):
    """K draft tokens per sequence through ``gdn_recurrent_verify``; ``state`` is only read.

    q, k [N,K,HK,dk]; v [N,K,HV,dv] (bf16 or fp32); g, beta [N,K,HV] fp32;
    state [N,HV,dv,dk] fp32.  ``rollback`` picks what is written for the
    commit: "states" (states_out [N,K,HV,dv,dk], the state after each draft),
    "deltas" (u_out [N,K,HV,dv], each draft's update vector), "both" or "none".
    Without per-draft states the call needs a device ``workspace`` of
    ``gdn_recurrent_verify_workspace_size`` bytes (allocated here if not given).
    Returns (o [N,K,HV,dv], states_out or None, u_out or None).
    """
    if rollback not in ("states", "deltas", "both", "none"):
        raise ValueError("rollback must be 'states', 'deltas', 'both' or 'none'")
    lib = load_library()
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(state, "state", torch.float32, dev)
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:2] != q.shape[:2]:
        raise ValueError("expected q,k [N,K,HK,dk] and v [N,K,HV,dv]")
    N, K, HK, dk = q.shape
    HV, dv = v.shape[2], v.shape[3]
    g_shape = (N, K, HV, dv) if prologue & ROW_DECAY else (N, K, HV)
    if g.shape != g_shape or beta.shape != (N, K, HV) or state.shape != (N, HV, dv, dk):
        raise ValueError(f"expected g {g_shape}, beta [N,K,HV] and state [N,HV,dv,dk]")
    if o is None:
        o = torch.empty_like(v)
    else:
        _need(o, "o", v.dtype, dev)
        if o.shape != v.shape:
            raise ValueError("o must have the shape of v")
    if rollback in ("states", "both"):
        if states_out is None:
            states_out = torch.empty((N, K, HV, dv, dk), dtype=torch.float32, device=dev)
        _need(states_out, "states_out", torch.float32, dev)
        if states_out.shape != (N, K, HV, dv, dk):
            raise ValueError("expected states_out [N,K,HV,dv,dk]")
    else:
        states_out = None
    if rollback in ("deltas", "both"):
        if u_out is None:
            u_out = torch.empty((N, K, HV, dv), dtype=torch.float32, device=dev)
        _need(u_out, "u_out", torch.float32, dev)
        if u_out.shape != (N, K, HV, dv):
            raise ValueError("expected u_out [N,K,HV,dv]")
    else:
        u_out = None
    ws_bytes = 0
    if states_out is None and N > 0:
        need = int(lib.gdn_recurrent_verify_workspace_size(N, K, HV, dk))
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
        _need(workspace, "workspace", None, dev)
        ws_bytes = workspace.numel() * workspace.element_size()
    st = lib.gdn_recurrent_verify(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state),
                                  N, K, HK, HV, dk, dv, float(scale), _dtype_code(q), _ptr(o),
                                  _ptr(states_out), _ptr(u_out), int(prologue),
                                  _ptr(workspace) if states_out is None else None, ws_bytes,
                                  _stream_ptr(stream, dev))
    if st != GDN_OK:
        raise GDNError(st, "gdn_recurrent_verify")
    return o, states_out, u_out


def gdn_recurrent_commit_verify(prev_k, prev_g, prev_u, accepted, q, k, v, g, beta, state,
                                scale: float = 1.0, o=None, u_out=None, workspace=None,
                                stream=None, prologue: int = 0):
    """Keep the previous round's accepted drafts, then verify this round's
    (``gdn_recurrent_commit_verify``): ``state`` is updated in place to the
    committed state; returns (o [N,K,HV,dv], u_out [N,K,HV,dv]) of this round.

    prev_k [N,Kp,HK,dk]; prev_g [N,Kp,HV] ([N,Kp,HV,dv] with ROW_DECAY, like g);
    prev_u [N,Kp,HV,dv] (the previous verify's u_out); accepted [N] int32 on the
    device; the rest as ``gdn_recurrent_verify``.
    """
    lib = load_library()
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v), ("prev_k", prev_k)):
        _need(t, name, q.dtype, dev)
    for name, t in (("g", g), ("beta", beta), ("state", state), ("prev_g", prev_g),
                    ("prev_u", prev_u)):
        _need(t, name, torch.float32, dev)
    _need(accepted, "accepted", torch.int32, dev)
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:2] != q.shape[:2]:
        raise ValueError("expected q,k [N,K,HK,dk] and v [N,K,HV,dv]")
    N, K, HK, dk = q.shape
    HV, dv = v.shape[2], v.shape[3]
    Kp = prev_k.shape[1] if prev_k.dim() == 4 else -1
    rd = (dv,) if prologue & ROW_DECAY else ()
    if (g.shape != (N, K, HV) + rd or beta.shape != (N, K, HV) or state.shape != (N, HV, dv, dk)
            or prev_k.shape != (N, Kp, HK, dk) or prev_g.shape != (N, Kp, HV) + rd
            or prev_u.shape != (N, Kp, HV, dv) or accepted.shape != (N,)):
        raise ValueError("shapes: prev_k [N,Kp,HK,dk], prev_g [N,Kp,HV(,dv)], prev_u [N,Kp,HV,dv], "
                         "accepted [N], q,k [N,K,HK,dk], v [N,K,HV,dv], g [N,K,HV(,dv)], "
                         "beta [N,K,HV], state [N,HV,dv,dk]")
    if o is None:
        o = torch.empty_like(v)
    if u_out is None:
        u_out = torch.empty((N, K, HV, dv), dtype=torch.float32, device=dev)
    _need(o, "o", v.dtype, dev)
    _need(u_out, "u_out", torch.float32, dev)
    if workspace is None and N > 0:
        need = int(lib.gdn_recurrent_commit_verify_workspace_size(N, Kp, K, HV, dk))
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.gdn_recurrent_commit_verify(_ptr(prev_k), _ptr(prev_g), _ptr(prev_u), _ptr(accepted),
                                         Kp, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                         _ptr(state), N, K, HK, HV, dk, dv, float(scale),
                                         _dtype_code(q), _ptr(o), _ptr(u_out), int(prologue),
                                         _ptr(workspace), ws_bytes, _stream_ptr(stream, dev))
    if st != GDN_OK:
        raise GDNError(st, "gdn_recurrent_commit_verify")
    return o, u_out


def gdn_recurrent_commit_verify_workspace_size(N, prev_K, K, HV, dk) -> int:
    """Bytes of workspace ``gdn_recurrent_commit_verify`` needs."""
    return int(load_library().gdn_recurrent_commit_verify_workspace_size(
        int(N), int(prev_K), int(K), int(HV), int(dk)))


def gdn_recurrent_verify_workspace_size(N, K, HV, dk) -> int:
    """Bytes of workspace ``gdn_recurrent_verify`` needs without per-draft states."""
    return int(load_library().gdn_recurrent_verify_workspace_size(int(N), int(K), int(HV),
                                                                  int(dk)))


def gdn_state_commit(states, accepted, state, stream=None):
    """state[n] <- states[n, accepted[n]-1] for 1 <= accepted[n] <= K (``gdn_state_commit``).

    states [N,K,HV,dv,dk] fp32; accepted [N] int32 on the device; state
    [N,HV,dv,dk] fp32, updated in place.  Returns state.
    """
    lib = load_library()
    dev = state.device
    _need(states, "states", torch.float32, dev)
    _need(accepted, "accepted", torch.int32, dev)
    _need(state, "state", torch.float32, dev)
    if states.dim() != 5 or state.shape != (states.shape[0],) + tuple(states.shape[2:]) \
            or accepted.shape != (states.shape[0],):
        raise ValueError("expected states [N,K,HV,dv,dk], accepted [N], state [N,HV,dv,dk]")
    N, K, HV, dv, dk = states.shape
    st = lib.gdn_state_commit(_ptr(states), _ptr(accepted), _ptr(state), N, K, HV, dk, dv,
                              _stream_ptr(stream, dev))
    if st != GDN_OK:
        raise GDNError(st, "gdn_state_commit")
    return state


def gdn_state_commit_deltas(k, g, u, accepted, state, stream=None, prologue: int = 0):
    """In-place roll-back from a verify pass's update vectors (``gdn_state_commit_deltas``).

    k [N,K,HK,dk] (the verify input, bf16 or fp32); g [N,K,HV] fp32; u
    [N,K,HV,dv] fp32 (verify's u_out); accepted [N] int32 on the device; state
    [N,HV,dv,dk] fp32 (verify's input state), updated in place.  Returns state.
    """
    lib = load_library()
    dev = state.device
    _need(k, "k", k.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(u, "u", torch.float32, dev)
    _need(accepted, "accepted", torch.int32, dev)
    _need(state, "state", torch.float32, dev)
    if k.dim() != 4 or u.dim() != 4 or state.dim() != 4:
        raise ValueError("expected k [N,K,HK,dk], u [N,K,HV,dv], state [N,HV,dv,dk]")
    N, K, HK, dk = k.shape
    HV, dv = u.shape[2], u.shape[3]
    g_shape = (N, K, HV, dv) if prologue & ROW_DECAY else (N, K, HV)
    if u.shape[:2] != (N, K) or g.shape != g_shape or accepted.shape != (N,) \
            or state.shape != (N, HV, dv, dk):
        raise ValueError("expected k [N,K,HK,dk], g [N,K,HV], u [N,K,HV,dv], accepted [N], "
                         "state [N,HV,dv,dk]")
    st = lib.gdn_state_commit_deltas(_ptr(k), _ptr(g), _ptr(u), _ptr(accepted), _ptr(state), N, K,
                                     HK, HV, dk, dv, _dtype_code(k), int(prologue),
                                     _stream_ptr(stream, dev))
    if st != GDN_OK:
        raise GDNError(st, "gdn_state_commit_deltas")
    return state


def gdn_chunk_prefill_path(dk, dv, chunk, dtype) -> int:
    """1 = tcgen05 tensor-core path, 0 = CUDA-core path, -1 = unsupported."""
    code = dtype if isinstance(dtype, int) else _dtype_code(torch.empty(0, dtype=dtype))
    return int(load_library().gdn_chunk_prefill_path(int(dk), int(dv), int(chunk), code))


def gdn_read_status(workspace, stream=None) -> int:
    """Status word of the last prefill on ``workspace`` (synchronises the stream).
    ``None``: the word in the library array the workspace-free prefill uses on the
    current device."""
    if workspace is None:
        import torch
        dev = torch.device("cuda", torch.cuda.current_device())
        return int(load_library().gdn_read_status(None, 0, _stream_ptr(stream, dev)))
    return int(load_library().gdn_read_status(
        _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream_ptr(stream, workspace.device)))


_copy_streams = {}


def _host_need(t, name, dtype=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cpu":
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def gdn_chunk_prefill_host_workspace_size(N, T, HK, HV, dk, dv, chunk, dtype, segment=0) -> int:
    code = dtype if isinstance(dtype, int) else _dtype_code(torch.empty(0, dtype=dtype))
    return int(load_library().gdn_chunk_prefill_host_workspace_size(
        int(N), int(T), int(HK), int(HV), int(dk), int(dv), int(chunk), code, int(segment)))


def gdn_chunk_prefill_host(q, k, v, g, beta, h0=None, chunk: int = 64, scale: float = 1.0,
                           o=None, hT=None, workspace=None, segment: int = 0, device=None,
                           stream=None, copy_streams=None, output_final_state: bool = True):
    """Prefill of host-resident data through ``gdn_chunk_prefill_host``.

    q, k [B,T,HK,dk]; v [B,T,HV,dv]; g, beta [B,T,HV] fp32 -- CPU tensors (pinned
    memory lets the copies overlap the computation); o: CPU output [B,T,HV,dv]
    (allocated pinned if None).  h0, hT: CUDA tensors [B,HV,dv,dk] fp32 or None.
    copy_streams: (copy_in, copy_out) CUDA streams; two cached side streams of the
    device are used if None.  Returns (o, hT); the results are ready once
    ``stream`` (default: the current stream) has been synchronised.
    """
    lib = load_library()
    dev = torch.device(device) if device is not None else (
        h0.device if h0 is not None else torch.device("cuda", torch.cuda.current_device()))
    for name, t in (("q", q), ("k", k), ("v", v)):
        _host_need(t, name, q.dtype)
    _host_need(g, "g", torch.float32)
    _host_need(beta, "beta", torch.float32)
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:2] != q.shape[:2]:
        raise ValueError("expected q,k [B,T,HK,dk] and v [B,T,HV,dv]")
    B, T, HK, dk = q.shape
    HV, dv = v.shape[2], v.shape[3]
    if g.shape != (B, T, HV) or beta.shape != (B, T, HV):
        raise ValueError("expected g, beta [B,T,HV]")
    if h0 is not None:
        _need(h0, "h0", torch.float32, dev)
        if h0.shape != (B, HV, dv, dk):
            raise ValueError(f"h0 must be [B,HV,dv,dk] = {(B, HV, dv, dk)}")
    if o is None:
        o = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
    else:
        _host_need(o, "o", v.dtype)
    if hT is None and output_final_state:
        hT = torch.empty((B, HV, dv, dk), dtype=torch.float32, device=dev)
    elif hT is not None:
        _need(hT, "hT", torch.float32, dev)
    code = _dtype_code(q)
    need = lib.gdn_chunk_prefill_host_workspace_size(B, T, HK, HV, dk, dv, chunk, code,
                                                     int(segment))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    if copy_streams is None:
        key = dev.index
        if key not in _copy_streams:
            _copy_streams[key] = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
        copy_streams = _copy_streams[key]
    st = lib.gdn_chunk_prefill_host(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0), B,
                                    T, HK, HV, dk, dv, int(chunk), float(scale), code, _ptr(o),
                                    _ptr(hT), _ptr(workspace), ws_bytes, int(segment),
                                    _stream_ptr(stream, dev),
                                    ctypes.c_void_p(copy_streams[0].cuda_stream),
                                    ctypes.c_void_p(copy_streams[1].cuda_stream))
    if st != GDN_OK:
        raise GDNError(st, "gdn_chunk_prefill_host")
    return o, hT


def gdn_validate_cu_seqlens(cu_seqlens, T, stream=None) -> int:
    """Runs ``gdn_validate_cu_seqlens`` on a device int32 [N+1] tensor and waits for
    it: 0 when valid, else 1 + the first offending index."""
    lib = load_library()
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    dev = cu_seqlens.device
    res = torch.empty(1, dtype=torch.int32, device=dev)
    st = lib.gdn_validate_cu_seqlens(_ptr(cu_seqlens), cu_seqlens.numel() - 1, int(T), _ptr(res),
                                     _stream_ptr(stream, dev))
    if st != GDN_OK:
        raise GDNError(st, "gdn_validate_cu_seqlens")
    return int(res.item())



# ---- the layer steps around the rule: short convolution on v, output gate ----
def _conv_args(conv_weight, conv_bias, conv_state, C, N, dtype, dev):
    """Shape checks of the convolution's weight [C,W], bias [C] and carried state
    [N,W-1,C]; returns the width (0 without a convolution)."""
    if conv_weight is None:
        return 0
    _need(conv_weight, "conv_weight", torch.float32, dev)
    if conv_weight.dim() != 2 or conv_weight.shape[0] != C:
        raise ValueError(f"conv_weight must be [C, width] with C = {C}")
    W = conv_weight.shape[1]
    if conv_bias is not None:
        _need(conv_bias, "conv_bias", torch.float32, dev)
        if conv_bias.shape != (C,):
            raise ValueError(f"conv_bias must be [{C}]")
    if conv_state is not None:
        _need(conv_state, "conv_state", dtype, dev)
        if conv_state.shape != (N, W - 1, C):
            raise ValueError(f"conv_state must be [N, width-1, C] = {(N, W - 1, C)}")
    return W


def gdn_short_conv(x, weight, bias=None, conv_state=None, cu_seqlens=None, silu: bool = False,
                   y=None, stream=None):
    """Causal depthwise convolution of each sequence through ``gdn_short_conv``.

    x [B,T,C] (bf16 or fp32; or packed [1,Ttot,C] with cu_seqlens); weight [C,W]
    fp32; bias [C] fp32 or None; conv_state [N,W-1,C] (x's dtype) or None: read
    as the history and overwritten with each sequence's last W-1 inputs.
    Returns y like x.
    """
    lib = load_library()
    dev = x.device
    _need(x, "x", None, dev)
    if x.dim() != 3:
        raise ValueError("expected x [B,T,C]")
    B, T, C = x.shape
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
        if B != 1:
            raise ValueError("with cu_seqlens the batch dimension must be 1 (packed)")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    W = _conv_args(weight, bias, conv_state, C, N, x.dtype, dev)
    if y is None:
        y = torch.empty_like(x)
    else:
        _need(y, "y", x.dtype, dev)
    st = lib.gdn_short_conv(_ptr(x), _ptr(weight), _ptr(bias), _ptr(conv_state),
                            _ptr(cu_seqlens), N, T, C, W, CONV_SILU if silu else 0,
                            _dtype_code(x), _ptr(y), _stream_ptr(stream, dev))
    if st != GDN_OK:
        raise GDNError(st, "gdn_short_conv")
    return y


def gdn_output_gate(o, z, stream=None):
    """o <- o * sigmoid(z) in place through ``gdn_output_gate``; returns o."""
    lib = load_library()
    dev = o.device
    _need(o, "o", None, dev)
    _need(z, "z", o.dtype, dev)
    if z.shape != o.shape:
        raise ValueError("z must have o's shape")
    if o.numel() == 0:
        return o
    C = o.shape[-1] if o.dim() > 0 else 1
    rows = o.numel() // C
    st = lib.gdn_output_gate(_ptr(o), _ptr(z), rows, C, _dtype_code(o), _stream_ptr(stream, dev))
    if st != GDN_OK:
        raise GDNError(st, "gdn_output_gate")
    return o


def gdn_recurrent_step_layer(q, k, v, g, beta, state, conv_weight=None, conv_bias=None,
                             conv_state=None, z=None, scale: float = 1.0, o=None, stream=None,
                             prologue: int = 0, silu: bool = False):
    """One decode token with the layer steps fused (``gdn_recurrent_step_layer``):
    v is convolved with the carried inputs ``conv_state`` [N,W-1,HV*dv] (updated
    in place) and o gated by sigmoid(z) (z [N,HV,dv]).  Other arguments as in
    ``gdn_recurrent_step``.  Returns o [N,HV,dv]."""
    lib = load_library()
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(state, "state", torch.float32, dev)
    if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[0] != q.shape[0]:
        raise ValueError("expected q,k [N,HK,dk] and v [N,HV,dv]")
    N, HK, dk = q.shape
    HV, dv = v.shape[1], v.shape[2]
    g_shape = (N, HV, dv) if prologue & ROW_DECAY else (N, HV)
    if g.shape != g_shape or beta.shape != (N, HV) or state.shape != (N, HV, dv, dk):
        raise ValueError(f"expected g {g_shape}, beta [N,HV] and state [N,HV,dv,dk]")
    if conv_weight is not None and conv_state is None:
        raise ValueError("a convolution needs its conv_state")
    W = _conv_args(conv_weight, conv_bias, conv_state, HV * dv, N, q.dtype, dev)
    if z is not None:
        _need(z, "z", q.dtype, dev)
        if z.shape != v.shape:
            raise ValueError("z must be [N,HV,dv]")
    if o is None:
        o = torch.empty_like(v)
    else:
        _need(o, "o", v.dtype, dev)
    flags = int(prologue) | (CONV_SILU if silu else 0)
    st = lib.gdn_recurrent_step_layer(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                      _ptr(state), _ptr(conv_weight), _ptr(conv_bias),
                                      _ptr(conv_state), W, _ptr(z), N, HK, HV, dk, dv,
                                      float(scale), _dtype_code(q), _ptr(o), flags,
                                      _stream_ptr(stream, dev))
    if st != GDN_OK:
        raise GDNError(st, "gdn_recurrent_step_layer")
    return o


def gdn_chunk_prefill_layer_workspace_size(N, T, HK, HV, dk, dv, chunk, dtype, varlen,
                                           has_conv, has_gate=False) -> int:
    code = dtype if isinstance(dtype, int) else _dtype_code(torch.empty(0, dtype=dtype))
    return int(load_library().gdn_chunk_prefill_layer_workspace_size(
        int(N), int(T), int(HK), int(HV), int(dk), int(dv), int(chunk), code,
        int(bool(varlen)), int(bool(has_conv)), int(bool(has_gate))))


def gdn_chunk_prefill_layer(q, k, v, g, beta, h0=None, cu_seqlens=None, conv_weight=None,
                            conv_bias=None, conv_state=None, z=None, chunk: int = 64,
                            scale: float = 1.0, o=None, hT=None, workspace=None, stream=None,
                            output_final_state: bool = True, prologue: int = 0,
                            silu: bool = False):
    """Prefill with the layer steps (``gdn_chunk_prefill_layer``): the short
    convolution of v (``conv_state`` [N,W-1,HV*dv] carried and updated when
    given), the rule, and the gate o <- o * sigmoid(z) (z like v).  Other
    arguments as in ``gdn_chunk_prefill``.  Returns (o, hT or None)."""
    lib = load_library()
    dev = q.device
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.dtype, dev)
    _need(g, "g", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:2] != q.shape[:2]:
        raise ValueError("expected q,k [B,T,HK,dk] and v [B,T,HV,dv]")
    B, T, HK, dk = q.shape
    HV, dv = v.shape[2], v.shape[3]
    g_shape = (B, T, HV, dv) if prologue & ROW_DECAY else (B, T, HV)
    if g.shape != g_shape or beta.shape != (B, T, HV):
        raise ValueError(f"expected g {g_shape} and beta [B,T,HV]")
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32, dev)
        if B != 1:
            raise ValueError("with cu_seqlens the batch dimension must be 1 (packed)")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    W = _conv_args(conv_weight, conv_bias, conv_state, HV * dv, N, q.dtype, dev)
    if z is not None:
        _need(z, "z", q.dtype, dev)
        if z.shape != v.shape:
            raise ValueError("z must have v's shape")
    if h0 is not None:
        _need(h0, "h0", torch.float32, dev)
        if h0.shape != (N, HV, dv, dk):
            raise ValueError(f"h0 must be [N,HV,dv,dk] = {(N, HV, dv, dk)}")
    if o is None:
        o = torch.empty_like(v)
    else:
        _need(o, "o", v.dtype, dev)
    if hT is None and output_final_state:
        hT = torch.empty((N, HV, dv, dk), dtype=torch.float32, device=dev)
    elif hT is not None:
        _need(hT, "hT", torch.float32, dev)
    code = _dtype_code(q)
    need = lib.gdn_chunk_prefill_layer_workspace_size(N, T, HK, HV, dk, dv, chunk, code,
                                                      int(cu_seqlens is not None),
                                                      int(conv_weight is not None),
                                                      int(z is not None))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    flags = int(prologue) | (CONV_SILU if silu else 0)
    st = lib.gdn_chunk_prefill_layer(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
                                     _ptr(cu_seqlens), N, T, HK, HV, dk, dv, int(chunk),
                                     float(scale), code, _ptr(o), _ptr(hT), _ptr(conv_weight),
                                     _ptr(conv_bias), _ptr(conv_state), W, _ptr(z), flags,
                                     _ptr(workspace), ws_bytes, _stream_ptr(stream, dev))
    if st != GDN_OK:
        raise GDNError(st, "gdn_chunk_prefill_layer")
    return o, hT
