"""Shared helpers for the GPU parity tests: tolerance checks and slicing of
sampled heads / sequences so the float64 oracle finishes in seconds."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances of the workloads: fp32 configs max |err| <= 1e-4; bf16 configs
# max |err| <= 2e-2 x RMS(reference), outputs and final states separately.
# Reading for results STORED in bf16 (the outputs o of bf16 workloads): an
# exactly computed value rounded to bf16 already differs from the float64
# reference by up to u = 2^-8 of its magnitude (8-bit significand, round to
# nearest), which at max|o|/RMS(o) ~ 7 exceeds 2e-2 x RMS on its own.  The
# format's own rounding is therefore allowed on top of the bound, per element:
#     |out - ref| <= 2e-2 x RMS(ref) + 2^-8 x |ref|,
# and in addition the relative RMS error must stay within 2e-2.  Results stored
# in fp32 (final states, decode state) get no such allowance.
FP32_ATOL = 1e-4
BF16_REL = 2e-2
BF16_UNIT_ROUNDOFF = 2.0 ** -8


def to_np(t):
    return t.detach().to("cpu", torch.float64).numpy() if isinstance(t, torch.Tensor) else t


def assert_close(out, ref, dtype, what="", stored_bf16=None):
    """``stored_bf16`` overrides the detection of a bf16-stored result (for
    results rescaled on the host after being read back from bf16)."""
    if stored_bf16 is None:
        stored_bf16 = isinstance(out, torch.Tensor) and out.dtype == torch.bfloat16
    out = np.asarray(to_np(out), dtype=np.float64).reshape(np.shape(ref))
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(out)), f"{what}: non-finite values"
    if out.size == 0:
        return 0.0
    diff = np.abs(out - ref)
    err = float(diff.max())
    if dtype == torch.float32:
        assert err <= FP32_ATOL, f"{what}: max|err| {err:.3e} > {FP32_ATOL}"
        return err
    rms = max(float(np.sqrt(np.mean(ref ** 2))), 1e-30)
    allow = BF16_REL * rms + (BF16_UNIT_ROUNDOFF * np.abs(ref) if stored_bf16 else 0.0)
    worst = float((diff / allow).max()) if np.ndim(allow) else err / allow
    rel_rms = float(np.sqrt(np.mean(diff ** 2))) / rms
    assert worst <= 1.0, (f"{what}: max|err| {err:.3e} exceeds 2e-2*RMS ({BF16_REL * rms:.3e})"
                          f"{' + bf16 rounding' if stored_bf16 else ''}; worst ratio {worst:.3f}")
    assert rel_rms <= BF16_REL, f"{what}: RMS(err)/RMS(ref) {rel_rms:.3e} > {BF16_REL}"
    return err / rms


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
