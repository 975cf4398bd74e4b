"""One decay per value row (GDN_ROW_DECAY: the teaching code's per-channel
forget gate) in the decode step, the per-draft-state verify and both commits,
through the C ABI, against the float64 oracle's ``step_row_decay`` and
``verify_row_decay``."""
import numpy as np
import pytest
import torch

from linear_attention_recurrence_rule_b200 import (PROLOGUE_ALL, PROLOGUE_GATE_LOGITS, ROW_DECAY,
                                                   gdn_chunk_prefill, gdn_recurrent_commit_verify,
                                                   gdn_recurrent_step, gdn_recurrent_verify,
                                                   gdn_state_commit, gdn_state_commit_deltas)
from linear_attention_recurrence_rule_b200.inputs import (make_decode, make_prefill, make_verify,
                                                          raw_projections, row_decays,
                                                          workload_inputs)
from oracle import gdn_oracle as O
from parity_util import assert_close, head_slice, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("extra", [0, PROLOGUE_ALL])
@pytest.mark.parametrize("N,HK,HV,dk,dv,dtype", [
    (16, 2, 4, 128, 128, torch.bfloat16),
    (5, 1, 2, 64, 48, torch.float32),
    (3, 1, 1, 32, 200, torch.float32),
])
def test_decode_row_decay(N, HK, HV, dk, dv, dtype, extra):
    base = make_decode(N, 3, HK, HV, dk, dv, dtype, seed=81, h0_std=0.3)
    x = raw_projections(base, seed=82) if extra else base
    g_rows = row_decays((3, N, HV, dv), seed=83)
    if extra & PROLOGUE_GATE_LOGITS:   # logits of the same decays: alpha = sigmoid(a)
        a = torch.exp(g_rows)
        g_rows = torch.log(a / (1 - a)).float()
    d = to_dev(x)
    gd = g_rows.cuda()
    S = d["state"].clone()
    Sref = x["state"]
    flags = ROW_DECAY | extra
    for t in range(3):
        o = gdn_recurrent_step(d["q"][t], d["k"][t], d["v"][t], gd[t].contiguous(), d["beta"][t],
                               S, scale=0.8, prologue=flags)
        q, k, g, b = O.prologue(x["q"][t], x["k"][t], g_rows[t], x["beta"][t], extra)
        o_ref, Sref = O.step_row_decay(q, k, x["v"][t], g, b, Sref, scale=0.8)
        assert_close(o, o_ref, dtype, f"o step {t}")
    torch.cuda.synchronize()
    assert_close(S, Sref, dtype, "state")


@pytest.mark.parametrize("N,K,HK,HV,dk,dv,dtype", [
    (9, 4, 2, 4, 128, 128, torch.bfloat16),
    (4, 7, 1, 2, 64, 96, torch.float32),
])
def test_verify_and_commits_row_decay(N, K, HK, HV, dk, dv, dtype):
    x = make_verify(N, K, HK, HV, dk, dv, dtype, seed=84, h0_std=0.3)
    g_rows = row_decays((N, K, HV, dv), seed=85)
    d = to_dev(x)
    gd = g_rows.cuda()
    o, states, u = gdn_recurrent_verify(d["q"], d["k"], d["v"], gd, d["beta"], d["state"],
                                        scale=0.6, rollback="both", prologue=ROW_DECAY)
    accepted = torch.arange(N, dtype=torch.int32) % (K + 1)
    S1 = d["state"].clone()
    gdn_state_commit(states, accepted.cuda(), S1)
    S2 = d["state"].clone()
    gdn_state_commit_deltas(d["k"], gd, u, accepted.cuda(), S2, prologue=ROW_DECAY)
    torch.cuda.synchronize()
    o_ref, states_ref = O.verify_row_decay(x["q"], x["k"], x["v"], g_rows, x["beta"], x["state"],
                                           scale=0.6)
    assert_close(o, o_ref, dtype, "o")
    for t in range(K):
        assert_close(states[:, t], states_ref[:, t], dtype, f"state after draft {t}")
    kept = O.commit(states_ref, accepted.numpy(), x["state"])
    assert_close(S1, kept, dtype, "committed (copy)")
    assert_close(S2, kept, dtype, "committed (deltas)")


@pytest.mark.parametrize("extra", [0, PROLOGUE_ALL])
@pytest.mark.parametrize("HK,HV,dk,dv,lengths,chunk,dtype", [
    (1, 2, 32, 32, [150], 16, torch.float32),
    (2, 2, 64, 64, [40, 100, 7], 32, torch.float32),         # packed, ragged
    (2, 4, 128, 128, [130, 130], 64, torch.bfloat16),        # the tensor-core shape
    (1, 2, 128, 64, [0, 65, 33, 1], 64, torch.bfloat16),     # an empty sequence, dk != dv
    (1, 4, 64, 128, [97], 16, torch.float32),               # dk != dv the other way
])
def test_prefill_row_decay(HK, HV, dk, dv, lengths, chunk, dtype, extra):
    """The prefill with one decay per value row runs on the row-recurrent CUDA-core
    kernel (each state row carried token by token): blocks of 32 tokens with
    ragged tails, empty sequences, every head-dim pair it takes."""
    base = make_prefill(HK, HV, dk, dv, lengths, dtype, seed=86, h0_std=0.2)
    x = raw_projections(base, seed=87) if extra else base
    B, T = x["q"].shape[0], x["q"].shape[1]
    g_rows = row_decays((B, T, HV, dv), seed=88)
    if extra & PROLOGUE_GATE_LOGITS:
        a = torch.exp(g_rows)
        g_rows = torch.log(a / (1 - a)).float()
    d = to_dev(x)
    o, hT = gdn_chunk_prefill(d["q"], d["k"], d["v"], g_rows.cuda(), d["beta"], h0=d["h0"],
                              cu_seqlens=d["cu_seqlens"], chunk=chunk, scale=0.7,
                              prologue=ROW_DECAY | extra)
    torch.cuda.synchronize()
    q, k, g, b = O.prologue(x["q"], x["k"], g_rows, x["beta"], extra)
    o_ref, h_ref = O.prefill_row_decay(q, k, x["v"], g, b, h0=x["h0"], cu_seqlens=x["cu_seqlens"],
                                       scale=0.7)
    assert_close(o, o_ref, dtype, "o")
    assert_close(hT, h_ref, dtype, "hT")


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_row_decay_update_vector_forms(dtype, d):
    """The update-vector verify and the fused commit-then-verify with one decay
    per value row (they run the per-draft kernel without writing states, the fused
    round after a commit from the previous round's update vectors)."""
    N, K, HK, HV = 6, 4, 2, 4
    x = make_verify(N, K, HK, HV, d, d, dtype, seed=91, h0_std=0.3)
    g_rows = row_decays((N, K, HV, d), seed=92)
    dx = to_dev(x)
    gd = g_rows.cuda()
    o, _, u = gdn_recurrent_verify(dx["q"], dx["k"], dx["v"], gd, dx["beta"], dx["state"],
                                   scale=0.6, rollback="deltas", prologue=ROW_DECAY)
    accepted = torch.tensor([0, 1, 2, 3, 4, 2], dtype=torch.int32)
    S2 = dx["state"].clone()
    gdn_state_commit_deltas(dx["k"], gd, u, accepted.cuda(), S2, prologue=ROW_DECAY)
    torch.cuda.synchronize()
    o_ref, states_ref = O.verify_row_decay(x["q"], x["k"], x["v"], g_rows, x["beta"], x["state"],
                                           scale=0.6)
    assert_close(o, o_ref, dtype, "o")
    kept = torch.as_tensor(O.commit(states_ref, accepted.numpy(), x["state"])).float()
    assert_close(S2, kept, dtype, "committed from the update vectors")
    # next round: this round's commit fused with the verify of new drafts
    y = make_verify(N, K, HK, HV, d, d, dtype, seed=93, h0_std=0.3)
    g2 = row_decays((N, K, HV, d), seed=94)
    dy = to_dev(y)
    S3 = dx["state"].clone()
    o2, u2 = gdn_recurrent_commit_verify(dx["k"], gd, u, accepted.cuda(), dy["q"], dy["k"], dy["v"],
                                         g2.cuda(), dy["beta"], S3, scale=0.6, prologue=ROW_DECAY)
    torch.cuda.synchronize()
    assert_close(S3, kept, dtype, "committed state (fused round)")
    o2_ref, states2_ref = O.verify_row_decay(y["q"], y["k"], y["v"], g2, y["beta"], kept, scale=0.6)
    assert_close(o2, o2_ref, dtype, "o (fused round)")
    S4 = S3.clone()
    gdn_state_commit_deltas(dy["k"], g2.cuda(), u2, torch.full((N,), K, dtype=torch.int32).cuda(), S4,
                            prologue=ROW_DECAY)
    torch.cuda.synchronize()
    assert_close(S4, states2_ref[:, K - 1], dtype, "state after the fused round's drafts")


def test_prefill_row_decay_bench_size_sampled_heads():
    """The workload the bench times for one decay per value row: the 4K-token
    layer (16 query/key heads, 32 value heads, d = 128, bf16) with row decays
    alpha ~U(0.8, 1), all heads in one call; the oracle checks two query/key
    heads and their value heads."""
    x = workload_inputs("layer_prefill_4k")
    g_rows = row_decays(tuple(x["v"].shape), seed=903)
    d = to_dev(x)
    o, hT = gdn_chunk_prefill(d["q"], d["k"], d["v"], g_rows.cuda(), d["beta"], chunk=64,
                              prologue=ROW_DECAY)
    torch.cuda.synchronize()
    HV = x["v"].shape[2]
    for qk in ([0], [15]):
        sub, vh = head_slice(x, qk, HV // x["q"].shape[2])
        o_ref, h_ref = O.prefill_row_decay(sub["q"], sub["k"], sub["v"], g_rows[:, :, vh],
                                           sub["beta"])
        assert_close(o[0][:, vh], o_ref, torch.bfloat16, f"o heads {vh}")
        assert_close(hT[:, vh], h_ref, torch.bfloat16, f"hT heads {vh}")
