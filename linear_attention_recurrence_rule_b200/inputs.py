"""Seeded synthetic inputs for the gated delta rule workloads.

This module holds workload shapes and value distributions only: none of the
rule's arithmetic.  Both the CUDA path (tests, bench) and the float64 oracle
are fed from it, so the two sides see bit-identical inputs.

Distributions follow the workload recipe for a Qwen3-Next Gated DeltaNet
layer (model card "Qwen3-Next-80B-A3B-Instruct", section "Model Overview":
32 value heads, 16 query/key heads, head dim 128):

* q, k ~ N(0, 1), then L2-normalised per head in fp32, then cast to the
  workload dtype (so bf16 keys are unit length only up to rounding; the oracle
  receives the rounded values, not re-normalised ones);
* v ~ N(0, 1);
* g = log(alpha) with alpha ~ U(0.9, 1.0) per token and value head (fp32);
* beta = sigmoid(N(0, 1)) per token and value head (fp32);
* h0 = 0, or ~N(0, 0.02) where the workload asks for a nonzero start state.

Everything is drawn on the CPU from ``torch.Generator().manual_seed(seed)``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    kind: str                    # "prefill", "decode" or "verify"
    B: int                       # batch (prefill without cu_seqlens) or sequences (decode)
    T: int                       # tokens per sequence (prefill) / decode steps / drafts (verify)
    HK: int
    HV: int
    dk: int
    dv: int
    chunk: int
    dtype: torch.dtype
    h0_std: float = 0.0          # 0 -> zero start state
    varlen: tuple = field(default=())   # (n_seqs, lo, hi) -> packed lengths ~U[lo, hi]

    @property
    def dtype_name(self) -> str:
        return {torch.float32: "f32", torch.bfloat16: "bf16"}[self.dtype]


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 0, "prefill", 1, 128, 1, 2, 32, 32, 16, torch.float32),
    "layer_prefill_4k": Workload("layer_prefill_4k", 1, "prefill", 1, 4096, 16, 32, 128, 128, 64,
                                 torch.bfloat16),
    "long_prefill_64k": Workload("long_prefill_64k", 2, "prefill", 1, 65536, 16, 32, 128, 128, 64,
                                 torch.bfloat16),
    "varlen_8": Workload("varlen_8", 3, "prefill", 1, 0, 16, 32, 128, 128, 64, torch.bfloat16,
                         h0_std=0.02, varlen=(8, 1024, 32768)),
    "decode_256x64": Workload("decode_256x64", 4, "decode", 256, 64, 16, 32, 128, 128, 1,
                              torch.bfloat16, h0_std=0.02),
    # speculative decoding: 4 draft tokens per sequence checked at once (the
    # model factory's multi-token-prediction head proposes 4), decode shapes
    "verify_256x4": Workload("verify_256x4", 5, "verify", 256, 4, 16, 32, 128, 128, 1,
                             torch.bfloat16, h0_std=0.02),
}


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    # L2 normalisation of each head vector, in fp32, before the cast
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def draw_lengths(gen: torch.Generator, n: int, lo: int, hi: int) -> list[int]:
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=gen)]


def make_prefill(HK: int, HV: int, dk: int, dv: int, lengths, dtype=torch.bfloat16,
                 seed: int = 0, h0_std: float = 0.0, packed: bool | None = None,
                 g_low: float = 0.9, g_high: float = 1.0):
    """Draw one prefill problem.

    ``lengths`` is a list of per-sequence token counts.  If every length is
    equal and ``packed`` is not True, tensors are [B,T,H,d] and ``cu_seqlens``
    is None; otherwise they are packed as [1,Ttot,H,d] with int32 ``cu_seqlens``.
    Returns a dict of CPU tensors: q,k,v (dtype), g,beta (fp32), h0 (fp32 or
    None), cu_seqlens (int32 or None).
    """
    gen = torch.Generator().manual_seed(seed)
    lengths = [int(x) for x in lengths]
    if packed is None:
        packed = len(set(lengths)) > 1
    N = len(lengths)
    Ttot = sum(lengths)
    q = _unit_rows(torch.randn(Ttot, HK, dk, generator=gen)).to(dtype)
    k = _unit_rows(torch.randn(Ttot, HK, dk, generator=gen)).to(dtype)
    v = torch.randn(Ttot, HV, dv, generator=gen).to(dtype)
    alpha = g_low + (g_high - g_low) * torch.rand(Ttot, HV, generator=gen)
    g = torch.log(alpha).float()
    beta = torch.sigmoid(torch.randn(Ttot, HV, generator=gen)).float()
    h0 = None
    if h0_std > 0:
        h0 = (h0_std * torch.randn(N, HV, dv, dk, generator=gen)).float()
    if packed:
        cu = torch.zeros(N + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
        shape = lambda x: x.reshape(1, Ttot, *x.shape[1:])
        return dict(q=shape(q), k=shape(k), v=shape(v), g=shape(g), beta=shape(beta), h0=h0,
                    cu_seqlens=cu)
    T = lengths[0] if N else 0
    shape = lambda x: x.reshape(N, T, *x.shape[1:])
    return dict(q=shape(q), k=shape(k), v=shape(v), g=shape(g), beta=shape(beta), h0=h0,
                cu_seqlens=None)


def make_decode(N: int, steps: int, HK: int, HV: int, dk: int, dv: int, dtype=torch.bfloat16,
                seed: int = 0, h0_std: float = 0.02):
    """Draw ``steps`` successive single-token inputs for N sequences plus a start state.

    Returns q,k [steps,N,HK,dk], v [steps,N,HV,dv], g,beta [steps,N,HV] and
    state [N,HV,dv,dk] fp32, all CPU tensors.
    """
    gen = torch.Generator().manual_seed(seed)
    q = _unit_rows(torch.randn(steps, N, HK, dk, generator=gen)).to(dtype)
    k = _unit_rows(torch.randn(steps, N, HK, dk, generator=gen)).to(dtype)
    v = torch.randn(steps, N, HV, dv, generator=gen).to(dtype)
    g = torch.log(0.9 + 0.1 * torch.rand(steps, N, HV, generator=gen)).float()
    beta = torch.sigmoid(torch.randn(steps, N, HV, generator=gen)).float()
    state = (h0_std * torch.randn(N, HV, dv, dk, generator=gen)).float()
    return dict(q=q, k=k, v=v, g=g, beta=beta, state=state)


def make_verify(N: int, K: int, HK: int, HV: int, dk: int, dv: int, dtype=torch.bfloat16,
                seed: int = 0, h0_std: float = 0.02):
    """K draft tokens for each of N sequences plus a start state (the draw of
    ``make_decode`` laid out sequence-major): q,k [N,K,HK,dk], v [N,K,HV,dv],
    g,beta [N,K,HV] and state [N,HV,dv,dk] fp32, all CPU tensors."""
    x = make_decode(N, K, HK, HV, dk, dv, dtype, seed, h0_std)
    out = {n: x[n].transpose(0, 1).contiguous() for n in ("q", "k", "v", "g", "beta")}
    out["state"] = x["state"]
    return out


def raw_projections(x: dict, seed: int, norm_range=(0.25, 4.0), forget_logit=(3.0, 1.0)):
    """Turn a generated problem into the raw projections a layer produces before
    its prologue: every q, k row multiplied by its own positive factor
    ~U(norm_range) (kept in the problem's dtype), and the gate arrays replaced
    by logits: ``g`` <- forget logits ~N(forget_logit) (alpha = sigmoid near
    0.95 at the default), ``beta`` <- write logits ~N(0, 1).  Only random draws
    and scalings; CPU tensors in, CPU tensors out."""
    gen = torch.Generator().manual_seed(seed)
    out = dict(x)
    for n in ("q", "k"):
        t = x[n]
        f = norm_range[0] + (norm_range[1] - norm_range[0]) * torch.rand(
            t.shape[:-1] + (1,), generator=gen)
        out[n] = (t.float() * f).to(t.dtype)
    out["g"] = (forget_logit[0] + forget_logit[1] * torch.randn(x["g"].shape, generator=gen)).float()
    out["beta"] = torch.randn(x["beta"].shape, generator=gen).float()
    return out


def row_decays(shape, seed: int, low: float = 0.8, high: float = 1.0):
    """One log decay per value row: g = log(alpha), alpha ~U(low, high), fp32,
    of the given shape ([..., HV, dv]); a random draw only."""
    gen = torch.Generator().manual_seed(seed)
    return torch.log(low + (high - low) * torch.rand(tuple(shape), generator=gen)).float()


def layer_extras(N: int, C: int, width: int, z_shape, dtype=torch.bfloat16, seed: int = 0):
    """Seeded inputs of the layer steps around the rule (random draws only):
    short-convolution weights [C, width] ~ N(0, 1/width) and bias [C] ~ N(0, 0.1^2)
    (fp32), a carried convolution state [N, width-1, C] ~ N(0, 1) and gate
    logits z of ``z_shape`` ~ N(0, 1), both in ``dtype``."""
    gen = torch.Generator().manual_seed(seed)
    w = (torch.randn((C, width), generator=gen) / width ** 0.5).float()
    b = (0.1 * torch.randn((C,), generator=gen)).float()
    cs = torch.randn((N, max(width - 1, 0), C), generator=gen).to(dtype)
    z = torch.randn(tuple(z_shape), generator=gen).to(dtype)
    return {"conv_weight": w, "conv_bias": b, "conv_state": cs, "z": z}


def workload_inputs(name: str, steps: int | None = None, seed_offset: int = 0,
                    tokens: int | None = None):
    """Inputs for one named workload (see ``WORKLOADS``).  ``seed_offset`` gives
    another draw of the same workload (one per replica); ``tokens`` truncates a
    single-sequence prefill workload to its first ``tokens`` tokens."""
    w = WORKLOADS[name]
    if seed_offset:
        from dataclasses import replace
        w = replace(w, seed=w.seed + 7919 * seed_offset)
    if w.kind == "decode":
        return make_decode(w.B, steps or w.T, w.HK, w.HV, w.dk, w.dv, w.dtype, w.seed, w.h0_std)
    if w.kind == "verify":
        return make_verify(w.B, w.T, w.HK, w.HV, w.dk, w.dv, w.dtype, w.seed, w.h0_std)
    if w.varlen:
        gen = torch.Generator().manual_seed(w.seed)
        n, lo, hi = w.varlen
        lengths = draw_lengths(gen, n, lo, hi)
        return make_prefill(w.HK, w.HV, w.dk, w.dv, lengths, w.dtype, seed=w.seed + 1000,
                            h0_std=w.h0_std, packed=True)
    T = w.T if tokens is None else min(int(tokens), w.T)
    return make_prefill(w.HK, w.HV, w.dk, w.dv, [T] * w.B, w.dtype, seed=w.seed,
                        h0_std=w.h0_std)


def varlen_lengths(name: str = "varlen_8") -> list[int]:
    w = WORKLOADS[name]
    gen = torch.Generator().manual_seed(w.seed)
    n, lo, hi = w.varlen
    return draw_lengths(gen, n, lo, hi)
