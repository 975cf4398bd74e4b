"""CUDA path (through the C ABI) against the float64 oracle, element by element.

Small cases span several chunks and a ragged tail; the full-size workloads run
in the launch configuration the benchmark times and are compared on sampled
heads / sequences the oracle computes in seconds.
"""
import math

import numpy as np
import pytest
import torch

from linear_attention_recurrence_rule_b200 import gdn_chunk_prefill, gdn_recurrent_step
from linear_attention_recurrence_rule_b200.inputs import (WORKLOADS, make_decode, make_prefill,
                                                          workload_inputs)
from oracle import gdn_oracle as O
from parity_util import assert_close, head_slice, to_dev

pytestmark = pytest.mark.gpu


def run_both(x, chunk, scale=1.0):
    d = to_dev(x)
    o, hT = gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"],
                              cu_seqlens=d["cu_seqlens"], chunk=chunk, scale=scale)
    torch.cuda.synchronize()
    o_ref, h_ref = O.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], h0=x["h0"],
                             cu_seqlens=x["cu_seqlens"], scale=scale)
    return o, hT, o_ref, h_ref


# ---------------------------------------------------------------------------
# workload configs
# ---------------------------------------------------------------------------
def test_tiny_fp32_workload():
    w = WORKLOADS["tiny_fp32"]
    x = workload_inputs("tiny_fp32")
    o, hT, o_ref, h_ref = run_both(x, w.chunk)
    assert_close(o, o_ref, torch.float32, "o")
    assert_close(hT, h_ref, torch.float32, "hT")


def test_layer_prefill_4k_workload():
    w = WORKLOADS["layer_prefill_4k"]
    x = workload_inputs("layer_prefill_4k")
    o, hT, o_ref, h_ref = run_both(x, w.chunk)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(hT, h_ref, torch.bfloat16, "hT")


def test_long_prefill_64k_sampled_heads():
    """Full T = 65536, all 32 value heads on the GPU (the benchmarked launch);
    the oracle recomputes two query/key groups (four value heads)."""
    w = WORKLOADS["long_prefill_64k"]
    x = workload_inputs("long_prefill_64k")
    d = to_dev(x)
    o, hT = gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], chunk=w.chunk)
    torch.cuda.synchronize()
    sub, vh = head_slice(x, [0, 11], w.HV // w.HK)
    o_ref, h_ref = O.prefill(sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"])
    assert_close(o[0][:, vh], o_ref, torch.bfloat16, "o")
    assert_close(hT[:, vh], h_ref, torch.bfloat16, "hT")


def test_varlen_8_sampled_heads():
    w = WORKLOADS["varlen_8"]
    x = workload_inputs("varlen_8")
    d = to_dev(x)
    o, hT = gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"],
                              cu_seqlens=d["cu_seqlens"], chunk=w.chunk)
    torch.cuda.synchronize()
    sub, vh = head_slice(x, [3], w.HV // w.HK)
    o_ref, h_ref = O.prefill(sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"], h0=sub["h0"],
                             cu_seqlens=sub["cu_seqlens"])
    assert_close(o[0][:, vh], o_ref, torch.bfloat16, "o")
    assert_close(hT[:, vh], h_ref, torch.bfloat16, "hT")


def test_decode_256x64_sampled_sequences():
    """All 256 sequences x 64 steps on the GPU; the oracle follows 6 of them."""
    w = WORKLOADS["decode_256x64"]
    x = workload_inputs("decode_256x64")
    d = to_dev(x)
    state = d["state"].clone()
    outs = []
    for t in range(w.T):
        outs.append(gdn_recurrent_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t],
                                       d["beta"][t], state))
    torch.cuda.synchronize()
    seqs = [0, 1, 77, 128, 200, 255]
    S = x["state"][seqs]
    for t in range(w.T):
        o_ref, S = O.step(x["q"][t][seqs], x["k"][t][seqs], x["v"][t][seqs], x["g"][t][seqs],
                          x["beta"][t][seqs], S)
        assert_close(outs[t][seqs], o_ref, torch.bfloat16, f"o step {t}")
    assert_close(state[seqs], S, torch.bfloat16, "state")


# ---------------------------------------------------------------------------
# edge cases: ragged tails, tiny and empty sequences, chunk sizes, head dims
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("T", [1, 15, 16, 17, 63, 64, 65, 130])
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_fp32_ragged_lengths(T, chunk):
    x = make_prefill(1, 2, 32, 32, [T], torch.float32, seed=100 + T, h0_std=0.5)
    o, hT, o_ref, h_ref = run_both(x, chunk)
    assert_close(o, o_ref, torch.float32, "o")
    assert_close(hT, h_ref, torch.float32, "hT")


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (32, 128), (128, 64)])
def test_fp32_head_dims(dk, dv):
    x = make_prefill(2, 4, dk, dv, [150, 150], torch.float32, seed=7, h0_std=0.1)
    o, hT, o_ref, h_ref = run_both(x, 64)
    assert_close(o, o_ref, torch.float32, "o")
    assert_close(hT, h_ref, torch.float32, "hT")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_varlen_with_empty_and_short_sequences(dtype):
    d = 32 if dtype == torch.float32 else 128
    lengths = [0, 5, 64, 1, 130, 0, 65, 200]
    x = make_prefill(2, 4, d, d, lengths, dtype, seed=11, h0_std=0.3, packed=True)
    o, hT, o_ref, h_ref = run_both(x, 64)
    assert_close(o, o_ref, dtype, "o")
    assert_close(hT, h_ref, dtype, "hT")
    # an empty sequence hands its start state through unchanged
    assert torch.equal(hT[0].cpu(), x["h0"][0]) and torch.equal(hT[5].cpu(), x["h0"][5])


@pytest.mark.parametrize("nseq,maxlen", [(300, 100), (1100, 9)])
def test_varlen_many_sequences(nseq, maxlen):
    # many packed sequences with repeated and zero lengths on the tensor-core path:
    # up to 1024 sequences run longest first (a permutation of the grid rows, ties
    # by index), more in launch order
    gen = torch.Generator().manual_seed(12)
    lengths = torch.randint(0, maxlen + 1, (nseq,), generator=gen).tolist()
    x = make_prefill(1, 2, 128, 128, lengths, torch.bfloat16, seed=13, h0_std=0.2, packed=True)
    o, hT, o_ref, h_ref = run_both(x, 64)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(hT, h_ref, torch.bfloat16, "hT")
    empty = [i for i, n in enumerate(lengths) if n == 0]
    assert empty and all(torch.equal(hT[i].cpu(), x["h0"][i]) for i in empty)


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 1000])
def test_bf16_d128_ragged_lengths(T):
    x = make_prefill(2, 4, 128, 128, [T, T], torch.bfloat16, seed=300 + T, h0_std=0.05)
    o, hT, o_ref, h_ref = run_both(x, 64)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(hT, h_ref, torch.bfloat16, "hT")


def test_strong_decay_tokens():
    """g = -30 on some tokens: factored forms must not overflow."""
    for dtype, d in ((torch.float32, 32), (torch.bfloat16, 128)):
        x = make_prefill(1, 2, d, d, [300], dtype, seed=5, h0_std=0.2)
        x["g"][0, ::13, :] = -30.0
        x["g"][0, 70, 1] = -80.0
        o, hT, o_ref, h_ref = run_both(x, 64)
        assert_close(o, o_ref, dtype, "o")
        assert_close(hT, h_ref, dtype, "hT")


def test_scale_and_state_alias():
    x = make_prefill(1, 2, 64, 64, [100], torch.float32, seed=9, h0_std=0.3)
    d = to_dev(x)
    h = d["h0"].clone()
    o, hT = gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=h, hT=h, chunk=32,
                              scale=0.125)
    torch.cuda.synchronize()
    o_ref, h_ref = O.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], h0=x["h0"], scale=0.125)
    assert hT.data_ptr() == h.data_ptr()
    assert_close(o, o_ref, torch.float32, "o")
    assert_close(h, h_ref, torch.float32, "hT (aliased h0)")


# ---------------------------------------------------------------------------
# structure on the GPU: decode == prefill, split/resume == whole
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_steps_equal_prefill(dtype):
    d = 32 if dtype == torch.float32 else 128
    T = 40
    x = make_prefill(2, 4, d, d, [T, T, T], dtype, seed=21, h0_std=0.1)
    g = to_dev(x)
    o_pre, h_pre = gdn_chunk_prefill(g["q"], g["k"], g["v"], g["g"], g["beta"], h0=g["h0"],
                                     chunk=16 if dtype == torch.float32 else 64)
    state = g["h0"].clone()
    outs = [gdn_recurrent_step(g["q"][:, t].contiguous(), g["k"][:, t].contiguous(),
                               g["v"][:, t].contiguous(), g["g"][:, t].contiguous(),
                               g["beta"][:, t].contiguous(), state) for t in range(T)]
    torch.cuda.synchronize()
    o_dec = torch.stack(outs, 1)
    o_ref, h_ref = O.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], h0=x["h0"])
    assert_close(o_dec.reshape(-1, 4, d), o_ref, dtype, "decode o")
    assert_close(state, h_ref, dtype, "decode state")
    assert_close(o_pre.reshape(-1, 4, d), o_ref, dtype, "prefill o")


def test_decode_fp32_tight():
    x = make_decode(5, 3, 2, 4, 64, 48, torch.float32, seed=3, h0_std=0.5)
    d = to_dev(x)
    S = d["state"].clone()
    Sref = x["state"]
    for t in range(3):
        o = gdn_recurrent_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], S,
                               scale=0.5)
        o_ref, Sref = O.step(x["q"][t], x["k"][t], x["v"][t], x["g"][t], x["beta"][t], Sref,
                             scale=0.5)
        assert_close(o, o_ref, torch.float32, "o")
    assert_close(S, Sref, torch.float32, "state")


@pytest.mark.parametrize("N,HK,HV,dk,dv,dtype", [
    (40, 2, 4, 64, 48, torch.float32),     # 160 states: the persistent streaming kernel
    (37, 1, 4, 32, 200, torch.bfloat16),   # 148 states, rows not a multiple of a pass
    (300, 2, 4, 128, 128, torch.bfloat16), # several states per SM
    (9, 1, 2, 128, 256, torch.float32),    # 128 KB states: the register kernel
])
def test_decode_streaming_shapes(N, HK, HV, dk, dv, dtype):
    x = make_decode(N, 2, HK, HV, dk, dv, dtype, seed=11, h0_std=0.3)
    d = to_dev(x)
    S = d["state"].clone()
    Sref = x["state"]
    for t in range(2):
        o = gdn_recurrent_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], S)
        o_ref, Sref = O.step(x["q"][t], x["k"][t], x["v"][t], x["g"][t], x["beta"][t], Sref)
        assert_close(o, o_ref, dtype, f"o step {t}")
    assert_close(S, Sref, dtype, "state")


def test_split_resume_equals_whole():
    x = make_prefill(2, 4, 128, 128, [700], torch.bfloat16, seed=31, h0_std=0.05)
    d = to_dev(x)
    o, hT = gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"], chunk=64)
    cut = 300
    part = lambda t, a, b: t[:, a:b].contiguous()
    o1, h1 = gdn_chunk_prefill(*(part(d[n], 0, cut) for n in ("q", "k", "v", "g", "beta")),
                               h0=d["h0"], chunk=64)
    o2, h2 = gdn_chunk_prefill(*(part(d[n], cut, 700) for n in ("q", "k", "v", "g", "beta")),
                               h0=h1, chunk=64)
    torch.cuda.synchronize()
    o_ref, h_ref = O.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], h0=x["h0"])
    assert_close(torch.cat([o1, o2], 1), o_ref, torch.bfloat16, "split o")
    assert_close(h2, h_ref, torch.bfloat16, "split hT")
    assert_close(o, o_ref, torch.bfloat16, "whole o")


def test_validate_cu_seqlens():
    from linear_attention_recurrence_rule_b200 import gdn_validate_cu_seqlens
    cu = lambda xs: torch.tensor(xs, dtype=torch.int32, device="cuda")
    assert gdn_validate_cu_seqlens(cu([0, 5, 5, 12]), 12) == 0
    assert gdn_validate_cu_seqlens(cu([0]), 0) == 0
    assert gdn_validate_cu_seqlens(cu([1, 5, 12]), 12) == 1           # does not start at 0
    assert gdn_validate_cu_seqlens(cu([0, 7, 5, 12]), 12) == 3        # decreases at index 2
    assert gdn_validate_cu_seqlens(cu([0, 5, 11]), 12) == 3           # does not end at T
    big = torch.arange(0, 3001 * 4, 4, dtype=torch.int32, device="cuda")
    assert gdn_validate_cu_seqlens(big, 12000) == 0
    big[1777] = 0
    assert gdn_validate_cu_seqlens(big, 12000) == 1778
