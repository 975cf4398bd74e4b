"""Shared helpers for the GPU parity tests: tolerance checks and slicing of
sampled heads / sequences so the float64 oracle finishes in seconds."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances of the workloads: fp32 configs max |err| <= 1e-4;
# bf16 configs max |err| / RMS(reference) <= 2e-2, outputs and final states separately.
FP32_ATOL = 1e-4
BF16_REL = 2e-2


def to_np(t):
    return t.detach().to("cpu", torch.float64).numpy() if isinstance(t, torch.Tensor) else t


def assert_close(out, ref, dtype, what=""):
    out = np.asarray(to_np(out), dtype=np.float64).reshape(np.shape(ref))
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(out)), f"{what}: non-finite values"
    if out.size == 0:
        return 0.0
    err = float(np.abs(out - ref).max())
    if dtype == torch.float32:
        assert err <= FP32_ATOL, f"{what}: max|err| {err:.3e} > {FP32_ATOL}"
        return err
    rms = float(np.sqrt(np.mean(ref ** 2)))
    rel = err / max(rms, 1e-30)
    assert rel <= BF16_REL, f"{what}: max|err|/RMS {rel:.3e} > {BF16_REL} (max|err| {err:.3e})"
    return rel


def to_dev(x, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def head_slice(x, qk_heads, HV_per_HK):
    """Restrict a prefill problem (CPU tensors) to the given query/key heads and
    the value heads that read them; returns the smaller problem for the oracle
    and the list of value-head indices it covers."""
    vh = [c * HV_per_HK + r for c in qk_heads for r in range(HV_per_HK)]
    out = dict(q=x["q"][:, :, qk_heads], k=x["k"][:, :, qk_heads], v=x["v"][:, :, vh],
               g=x["g"][:, :, vh], beta=x["beta"][:, :, vh],
               h0=None if x["h0"] is None else x["h0"][:, vh],
               cu_seqlens=x["cu_seqlens"])
    return out, vh
