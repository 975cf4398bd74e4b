"""The fused input prologue (L2-normalised q / k, sigmoid gates from logits) on
every path, through the C ABI, against the float64 oracle's ``prologue``
followed by the rule."""
import numpy as np
import pytest
import torch

from linear_attention_recurrence_rule_b200 import (PROLOGUE_ALL, PROLOGUE_GATE_LOGITS,
                                                   PROLOGUE_NORM_K, PROLOGUE_NORM_Q,
                                                   gdn_chunk_prefill, gdn_recurrent_step,
                                                   gdn_recurrent_verify, gdn_state_commit_deltas)
from linear_attention_recurrence_rule_b200.inputs import (make_decode, make_prefill, make_verify,
                                                          raw_projections)
from oracle import gdn_oracle as O
from parity_util import assert_close, to_dev

pytestmark = pytest.mark.gpu


def oracle_prefill(x, flags, scale=1.0):
    q, k, g, b = O.prologue(x["q"], x["k"], x["g"], x["beta"], flags)
    return O.prefill(q, k, x["v"], g, b, h0=x["h0"], cu_seqlens=x["cu_seqlens"], scale=scale)


def raw_for(base, flags, seed):
    """Raw projections for the tensors the flags prepare; the others keep the
    problem's prepared values (unit keys: with raw keys of norm up to 4 and no
    normalisation, beta |k|^2 reaches 16 and the rule itself diverges)."""
    x = raw_projections(base, seed=seed)
    if not flags & PROLOGUE_NORM_Q:
        x["q"] = base["q"]
    if not flags & PROLOGUE_NORM_K:
        x["k"] = base["k"]
    if not flags & PROLOGUE_GATE_LOGITS:
        x["g"], x["beta"] = base["g"], base["beta"]
    return x


def run_prefill(x, chunk, flags, scale=1.0):
    d = to_dev(x)
    o, hT = gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"],
                              cu_seqlens=d["cu_seqlens"], chunk=chunk, scale=scale,
                              prologue=flags)
    torch.cuda.synchronize()
    return o, hT


@pytest.mark.parametrize("flags", [PROLOGUE_ALL, PROLOGUE_NORM_K | PROLOGUE_GATE_LOGITS,
                                   PROLOGUE_NORM_Q])
def test_prefill_tensor_core_path(flags):
    base = make_prefill(2, 4, 128, 128, [300, 300], torch.bfloat16, seed=61, h0_std=0.05)
    x = raw_for(base, flags, seed=62)
    o, hT = run_prefill(x, 64, flags, scale=0.5)
    o_ref, h_ref = oracle_prefill(x, flags, scale=0.5)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(hT, h_ref, torch.bfloat16, "hT")


def test_prefill_tensor_core_path_packed():
    # packed sequences: a chunk's tile reaches into the next sequence's rows
    base = make_prefill(2, 4, 128, 128, [70, 200, 5, 130], torch.bfloat16, seed=63,
                        h0_std=0.05, packed=True)
    x = raw_projections(base, seed=64)
    o, hT = run_prefill(x, 64, PROLOGUE_ALL)
    o_ref, h_ref = oracle_prefill(x, PROLOGUE_ALL)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(hT, h_ref, torch.bfloat16, "hT")


@pytest.mark.parametrize("flags", [PROLOGUE_ALL, PROLOGUE_NORM_Q, PROLOGUE_NORM_K,
                                   PROLOGUE_GATE_LOGITS])
def test_prefill_cuda_core_path_fp32(flags):
    base = make_prefill(1, 2, 32, 32, [150], torch.float32, seed=65, h0_std=0.1)
    x = raw_for(base, flags, seed=66)
    o, hT = run_prefill(x, 16, flags)
    o_ref, h_ref = oracle_prefill(x, flags)
    assert_close(o, o_ref, torch.float32, "o")
    assert_close(hT, h_ref, torch.float32, "hT")


def test_prefill_prologue_is_scale_free_on_gpu():
    base = make_prefill(2, 4, 128, 128, [256], torch.bfloat16, seed=67)
    x = raw_projections(base, seed=68)
    y = dict(x)
    y["k"] = (x["k"].float() * 2.0).to(torch.bfloat16)   # exact: a power of two
    y["q"] = (x["q"].float() * 0.5).to(torch.bfloat16)
    o1, h1 = run_prefill(x, 64, PROLOGUE_ALL)
    o2, h2 = run_prefill(y, 64, PROLOGUE_ALL)
    assert torch.allclose(o1.float(), o2.float(), atol=1e-2, rtol=1e-2)
    assert torch.allclose(h1, h2, atol=1e-3, rtol=1e-3)


@pytest.mark.parametrize("N,HK,HV,dk,dv,dtype", [
    (16, 2, 4, 128, 128, torch.bfloat16),
    (5, 1, 2, 64, 48, torch.float32),
    (3, 1, 1, 32, 200, torch.float32),
])
def test_decode_step(N, HK, HV, dk, dv, dtype):
    base = make_decode(N, 3, HK, HV, dk, dv, dtype, seed=71, h0_std=0.3)
    x = raw_projections(base, seed=72)
    d = to_dev(x)
    S = d["state"].clone()
    Sref = x["state"]
    for t in range(3):
        o = gdn_recurrent_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], S,
                               scale=0.8, prologue=PROLOGUE_ALL)
        q, k, g, b = O.prologue(x["q"][t], x["k"][t], x["g"][t], x["beta"][t], PROLOGUE_ALL)
        o_ref, Sref = O.step(q, k, x["v"][t], g, b, Sref, scale=0.8)
        assert_close(o, o_ref, dtype, f"o step {t}")
    torch.cuda.synchronize()
    assert_close(S, Sref, dtype, "state")


@pytest.mark.parametrize("rollback", ["both", "deltas"])
@pytest.mark.parametrize("N,K,HK,HV,dk,dv,dtype", [
    (9, 4, 2, 4, 128, 128, torch.bfloat16),
    (4, 7, 1, 2, 64, 96, torch.float32),
])
def test_verify_and_commit(N, K, HK, HV, dk, dv, dtype, rollback):
    base = make_verify(N, K, HK, HV, dk, dv, dtype, seed=73, h0_std=0.3)
    x = raw_projections(base, seed=74)
    d = to_dev(x)
    o, states, u = gdn_recurrent_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"],
                                        rollback=rollback, prologue=PROLOGUE_ALL)
    accepted = torch.arange(N, dtype=torch.int32) % (K + 1)
    S = d["state"].clone()
    gdn_state_commit_deltas(d["k"], d["g"], u, accepted.cuda(), S, prologue=PROLOGUE_ALL)
    torch.cuda.synchronize()
    q, k, g, b = O.prologue(x["q"], x["k"], x["g"], x["beta"], PROLOGUE_ALL)
    o_ref, states_ref = O.verify(q, k, x["v"], g, b, x["state"])
    assert_close(o, o_ref, dtype, "o")
    if states is not None:
        for t in range(K):
            assert_close(states[:, t], states_ref[:, t], dtype, f"state after draft {t}")
    assert_close(S, O.commit(states_ref, accepted.numpy(), x["state"]), dtype, "committed")


def test_gate_logits_saturate_without_nan():
    # extreme logits: alpha, beta at 0 and 1 exactly; no inf or NaN anywhere
    base = make_prefill(1, 2, 32, 32, [64], torch.float32, seed=75, h0_std=0.1)
    x = dict(base)
    T = x["g"].shape[1]
    x["g"] = torch.tensor([[-200.0, 200.0]] * (T // 2)).reshape(1, T, 1).expand(1, T, 2).contiguous()
    x["beta"] = torch.tensor([[200.0, -200.0]] * (T // 2)).reshape(1, T, 1).expand(1, T, 2).contiguous()
    o, hT = run_prefill(x, 16, PROLOGUE_GATE_LOGITS)
    assert bool(torch.isfinite(o).all()) and bool(torch.isfinite(hT).all())
    o_ref, h_ref = oracle_prefill(x, PROLOGUE_GATE_LOGITS)
    assert_close(o, o_ref, torch.float32, "o")
    assert_close(hT, h_ref, torch.float32, "hT")
    assert np.all(np.isfinite(h_ref))


def test_long_prefill_64k_raw_projections_sampled_heads():
    """The bench's prologue leg: all 32 value heads of the 64K prefill from raw
    projections on the GPU; the oracle recomputes one query/key group."""
    from linear_attention_recurrence_rule_b200.inputs import WORKLOADS, workload_inputs
    from parity_util import head_slice
    w = WORKLOADS["long_prefill_64k"]
    x = raw_projections(workload_inputs("long_prefill_64k"), seed=900)
    d = to_dev(x)
    o, hT = gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], chunk=w.chunk,
                              prologue=PROLOGUE_ALL)
    torch.cuda.synchronize()
    sub, vh = head_slice(x, [5], w.HV // w.HK)
    q, k, g, b = O.prologue(sub["q"], sub["k"], sub["g"], sub["beta"], PROLOGUE_ALL)
    o_ref, h_ref = O.prefill(q, k, sub["v"], g, b)
    assert_close(o[0][:, vh], o_ref, torch.bfloat16, "o")
    assert_close(hT[:, vh], h_ref, torch.bfloat16, "hT")


def test_decode_256_raw_projections_sampled_sequences():
    """One decode step over the decode workload's 256 sequences from raw projections."""
    from linear_attention_recurrence_rule_b200.inputs import workload_inputs
    x = raw_projections(workload_inputs("decode_256x64", steps=2), seed=901)
    d = to_dev(x)
    S = d["state"].clone()
    outs = [gdn_recurrent_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], S,
                               prologue=PROLOGUE_ALL) for t in range(2)]
    torch.cuda.synchronize()
    seqs = [0, 64, 255]
    Sref = x["state"][seqs]
    for t in range(2):
        q, k, g, b = O.prologue(x["q"][t][seqs], x["k"][t][seqs], x["g"][t][seqs],
                                x["beta"][t][seqs], PROLOGUE_ALL)
        o_ref, Sref = O.step(q, k, x["v"][t][seqs], g, b, Sref)
        assert_close(outs[t][seqs], o_ref, torch.bfloat16, f"o step {t}")
    assert_close(S[seqs], Sref, torch.bfloat16, "state")
