"""Multi-token verify (speculative drafts) and the roll-back commit, through the
C ABI, against the float64 oracle's ``verify`` and ``commit``."""
import numpy as np
import pytest
import torch

from linear_attention_recurrence_rule_b200 import (GDNError, gdn_read_status, gdn_recurrent_step,
                                                   gdn_recurrent_verify,
                                                   gdn_recurrent_verify_workspace_size,
                                                   gdn_state_commit, gdn_state_commit_deltas)
from linear_attention_recurrence_rule_b200.inputs import make_verify
from oracle import gdn_oracle as O
from parity_util import assert_close, to_dev

pytestmark = pytest.mark.gpu


# "both" runs the kernel that carries the state through the drafts (and writes
# it after each); "deltas" the one that keeps S_0 and unrolls the drafts.
@pytest.mark.parametrize("rollback", ["both", "deltas"])
@pytest.mark.parametrize("N,K,HK,HV,dk,dv,dtype", [
    (5, 1, 2, 4, 64, 48, torch.float32),      # one draft: the decode step
    (7, 2, 1, 2, 32, 200, torch.bfloat16),    # dv not a multiple of a band
    (33, 4, 2, 4, 128, 128, torch.bfloat16),  # the model's head shape
    (9, 1, 1, 2, 128, 128, torch.bfloat16),   # tensor-core form, one draft
    (80, 8, 1, 2, 128, 128, torch.bfloat16),  # its largest count, 160 heads: two per CTA
    (6, 5, 1, 2, 128, 128, torch.float32),    # first count past the 4-draft bound
    (3, 8, 1, 2, 128, 256, torch.float32),    # two bands per state
    (4, 11, 2, 2, 32, 72, torch.bfloat16),    # a count between the 8 and 16 bounds
    (4, 16, 2, 4, 64, 64, torch.float32),     # the largest draft count
])
def test_verify_matches_oracle(N, K, HK, HV, dk, dv, dtype, rollback):
    x = make_verify(N, K, HK, HV, dk, dv, dtype, seed=41 + K, h0_std=0.3)
    d = to_dev(x)
    state0 = d["state"].clone()
    o, states, u = gdn_recurrent_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"],
                                        scale=0.7, rollback=rollback)
    torch.cuda.synchronize()
    o_ref, states_ref = O.verify(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state"], scale=0.7)
    assert torch.equal(d["state"], state0), "verify must not modify the input state"
    assert_close(o, o_ref, dtype, "o")
    if rollback == "both":
        for t in range(K):
            assert_close(states[:, t], states_ref[:, t], dtype, f"state after draft {t}")
    else:
        assert states is None
    # u_t is the rank-1 update of draft t: S_t - alpha_t S_{t-1} (oracle states)
    prev = np.concatenate([x["state"].double().numpy()[:, None], states_ref[:, :-1]], 1)
    alpha = np.exp(x["g"].double().numpy())[..., None, None]
    k_rep = x["k"].double().numpy().repeat(HV // HK, axis=2)       # [N,K,HV,dk]
    delta = states_ref - alpha * prev                                 # = u_t k_t^T
    u_ref = np.einsum("nthvd,nthd->nthv", delta, k_rep) / np.einsum("nthd,nthd->nth", k_rep,
                                                                     k_rep)[..., None]
    assert_close(u, u_ref, dtype, "u")


def test_verify_one_draft_equals_decode_step():
    x = make_verify(9, 1, 2, 4, 128, 128, torch.bfloat16, seed=5, h0_std=0.2)
    d = to_dev(x)
    o, states, _ = gdn_recurrent_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"])
    S = d["state"].clone()
    o1 = gdn_recurrent_step(d["q"][:, 0].contiguous(), d["k"][:, 0].contiguous(),
                            d["v"][:, 0].contiguous(), d["g"][:, 0].contiguous(),
                            d["beta"][:, 0].contiguous(), S)
    torch.cuda.synchronize()
    # the same recurrence with the dot products summed in another order: the
    # states agree to fp32 rounding, the bf16 outputs to one rounding step
    assert float((states[:, 0] - S).abs().max()) <= 1e-5
    diff = (o[:, 0].float() - o1.float()).abs()
    assert bool((diff <= 2.0 ** -7 * o1.float().abs() + 1e-6).all())


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_commit_keeps_accepted_prefix(dtype):
    N, K = 11, 6
    x = make_verify(N, K, 1, 2, 64, 96, dtype, seed=8, h0_std=0.3)
    d = to_dev(x)
    o, states, u = gdn_recurrent_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"],
                                        rollback="both")
    gen = torch.Generator().manual_seed(3)
    accepted = torch.randint(0, K + 1, (N,), generator=gen, dtype=torch.int32)
    accepted[0], accepted[1], accepted[2] = 0, K, 1       # none, all, one
    accepted[3] = K + 2                                   # out of range: treated as none
    S = d["state"].clone()
    gdn_state_commit(states, accepted.cuda(), S)
    torch.cuda.synchronize()
    # the commit is a copy: bit-exact against the verify output it selects
    expect = O.commit(states.cpu().double().numpy(),
                      np.where(accepted.numpy() <= K, accepted.numpy(), 0), d["state"].cpu())
    assert np.array_equal(S.cpu().double().numpy(), expect)
    # and the kept state is the oracle's state after the accepted drafts
    _, states_ref = O.verify(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state"])
    acc = np.where(accepted.numpy() <= K, accepted.numpy(), 0)
    assert_close(S, O.commit(states_ref, acc, x["state"]), dtype, "committed state")
    # the deltas form reaches the same state from u, k and g in place
    S2 = d["state"].clone()
    gdn_state_commit_deltas(d["k"], d["g"], u, accepted.cuda(), S2)
    torch.cuda.synchronize()
    assert_close(S2, O.commit(states_ref, acc, x["state"]), dtype, "committed state (deltas)")
    untouched = np.flatnonzero(acc == 0)
    assert torch.equal(S2[untouched], d["state"][untouched])


@pytest.mark.parametrize("N,K,HK,HV,dk,dv,dtype", [
    (8, 4, 2, 4, 128, 128, torch.bfloat16),
    (5, 16, 1, 2, 32, 200, torch.float32),    # the largest draft count, ragged band
    (3, 3, 1, 1, 64, 256, torch.float32),
])
def test_commit_deltas_matches_oracle(N, K, HK, HV, dk, dv, dtype):
    x = make_verify(N, K, HK, HV, dk, dv, dtype, seed=17 + K, h0_std=0.5)
    d = to_dev(x)
    ws = torch.empty(gdn_recurrent_verify_workspace_size(N, K, HV, dk), dtype=torch.uint8,
                     device="cuda")
    _, states_none, u = gdn_recurrent_verify(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                             d["state"], rollback="deltas", workspace=ws)
    assert states_none is None
    assert gdn_read_status(ws) == 0   # every bounded wait of the streaming kernel completed
    accepted = (torch.arange(N, dtype=torch.int32) % (K + 1))
    S = d["state"].clone()
    gdn_state_commit_deltas(d["k"], d["g"], u, accepted.cuda(), S)
    torch.cuda.synchronize()
    _, states_ref = O.verify(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state"])
    assert_close(S, O.commit(states_ref, accepted.numpy(), x["state"]), dtype, "state")


def test_verify_then_commit_all_equals_decode_steps():
    N, K = 6, 4
    x = make_verify(N, K, 2, 4, 128, 128, torch.float32, seed=13, h0_std=0.2)
    d = to_dev(x)
    o, states, u = gdn_recurrent_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"],
                                        rollback="both")
    S = d["state"].clone()
    gdn_state_commit(states, torch.full((N,), K, dtype=torch.int32, device="cuda"), S)
    S2 = d["state"].clone()
    outs = [gdn_recurrent_step(*(d[n][:, t].contiguous() for n in ("q", "k", "v", "g", "beta")),
                               S2) for t in range(K)]
    torch.cuda.synchronize()
    assert_close(o, torch.stack(outs, 1).cpu().double().numpy(), torch.float32, "o")
    assert_close(S, S2.cpu().double().numpy(), torch.float32, "state")
    S3 = d["state"].clone()
    gdn_state_commit_deltas(d["k"], d["g"], u, torch.full((N,), K, dtype=torch.int32,
                                                          device="cuda"), S3)
    torch.cuda.synchronize()
    assert_close(S3, S2.cpu().double().numpy(), torch.float32, "state (deltas)")


def test_verify_empty_and_errors():
    x = make_verify(2, 3, 1, 2, 32, 32, torch.float32, seed=1)
    d = to_dev(x)
    e = {n: d[n][:0] for n in ("q", "k", "v", "g", "beta", "state")}
    o, states, u = gdn_recurrent_verify(e["q"], e["k"], e["v"], e["g"], e["beta"], e["state"],
                                        rollback="both")
    assert o.numel() == 0 and states.numel() == 0 and u.numel() == 0
    gdn_state_commit_deltas(e["k"], e["g"], u, torch.zeros(0, dtype=torch.int32, device="cuda"),
                            e["state"])
    with pytest.raises(ValueError):
        gdn_recurrent_verify(d["q"], d["k"], d["v"], d["g"][:, :2].contiguous(), d["beta"],
                             d["state"])
    with pytest.raises(GDNError):   # update-vector form with a too small workspace
        gdn_recurrent_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"],
                             rollback="deltas",
                             workspace=torch.empty(64, dtype=torch.uint8, device="cuda"))
    big = make_verify(1, 17, 1, 2, 32, 32, torch.float32, seed=2)
    b = to_dev(big)
    with pytest.raises(GDNError):
        gdn_recurrent_verify(b["q"], b["k"], b["v"], b["g"], b["beta"], b["state"])


@pytest.mark.parametrize("rollback", ["deltas", "states"])
def test_verify_256x4_sampled_sequences(rollback):
    """The benchmarked round: all 256 sequences x 4 drafts x 32 value heads on the
    GPU, verify then commit of ~U{0..4} accepted drafts; the oracle follows 5
    sequences."""
    from linear_attention_recurrence_rule_b200.inputs import WORKLOADS, workload_inputs
    w = WORKLOADS["verify_256x4"]
    x = workload_inputs("verify_256x4")
    d = to_dev(x)
    gen = torch.Generator().manual_seed(w.seed + 77)
    accepted = torch.randint(0, w.T + 1, (w.B,), generator=gen, dtype=torch.int32)
    o, states, u = gdn_recurrent_verify(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"],
                                        rollback=rollback)
    S = d["state"].clone()
    if rollback == "deltas":
        gdn_state_commit_deltas(d["k"], d["g"], u, accepted.cuda(), S)
    else:
        gdn_state_commit(states, accepted.cuda(), S)
    torch.cuda.synchronize()
    seqs = [0, 3, 100, 201, 255]
    sub = {n: x[n][seqs] for n in ("q", "k", "v", "g", "beta", "state")}
    o_ref, states_ref = O.verify(sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"], sub["state"])
    assert_close(o[seqs], o_ref, torch.bfloat16, "o")
    assert_close(S[seqs], O.commit(states_ref, accepted[seqs].numpy(), sub["state"]),
                 torch.bfloat16, "committed state")


@pytest.mark.parametrize("prologue", [0, 7])
@pytest.mark.parametrize("N,K1,K2,HK,HV,dk,dv,dtype", [
    (33, 4, 4, 2, 4, 128, 128, torch.bfloat16),   # the benchmarked shapes
    (5, 3, 6, 1, 2, 64, 48, torch.float32),       # next round's bound (8) above the kept one
    (4, 16, 2, 2, 2, 32, 200, torch.float32),     # the largest kept round, ragged band
])
def test_commit_verify_equals_commit_then_verify(N, K1, K2, HK, HV, dk, dv, dtype, prologue):
    from linear_attention_recurrence_rule_b200 import (gdn_recurrent_commit_verify,
                                                       gdn_recurrent_commit_verify_workspace_size)
    from linear_attention_recurrence_rule_b200.inputs import raw_projections
    x1 = make_verify(N, K1, HK, HV, dk, dv, dtype, seed=90 + K1, h0_std=0.3)
    x2 = make_verify(N, K2, HK, HV, dk, dv, dtype, seed=91 + K2, h0_std=0.3)
    if prologue:
        x1, x2 = raw_projections(x1, seed=92), raw_projections(x2, seed=93)
    d1, d2 = to_dev(x1), to_dev(x2)
    _, _, u1 = gdn_recurrent_verify(d1["q"], d1["k"], d1["v"], d1["g"], d1["beta"], d1["state"],
                                    rollback="deltas", prologue=prologue)
    accepted = (torch.arange(N, dtype=torch.int32) * 7) % (K1 + 2)   # includes 0 and K1 + 1
    S = d1["state"].clone()
    ws = torch.empty(gdn_recurrent_commit_verify_workspace_size(N, K1, K2, HV, dk),
                     dtype=torch.uint8, device="cuda")
    o2, u2 = gdn_recurrent_commit_verify(d1["k"], d1["g"], u1, accepted.cuda(), d2["q"], d2["k"],
                                         d2["v"], d2["g"], d2["beta"], S, scale=0.9,
                                         workspace=ws, prologue=prologue)
    # the same round as two calls on the GPU
    Sb = d1["state"].clone()
    gdn_state_commit_deltas(d1["k"], d1["g"], u1, accepted.cuda(), Sb, prologue=prologue)
    o2b, _, u2b = gdn_recurrent_verify(d2["q"], d2["k"], d2["v"], d2["g"], d2["beta"], Sb,
                                       scale=0.9, rollback="deltas", prologue=prologue)
    torch.cuda.synchronize()
    assert gdn_read_status(ws) == 0
    # against the oracle: commit of the first drafts, then verify of the second
    q1, k1, g1, b1 = O.prologue(x1["q"], x1["k"], x1["g"], x1["beta"], prologue)
    _, st1 = O.verify(q1, k1, x1["v"], g1, b1, x1["state"])
    acc = np.where(accepted.numpy() <= K1, accepted.numpy(), 0)
    Sc = O.commit(st1, acc, x1["state"])
    q2, k2, g2, b2 = O.prologue(x2["q"], x2["k"], x2["g"], x2["beta"], prologue)
    o2_ref, _ = O.verify(q2, k2, x2["v"], g2, b2, Sc, scale=0.9)
    assert_close(S, Sc, dtype, "committed state")
    assert_close(o2, o2_ref, dtype, "o")
    assert_close(o2, o2b.double().cpu().numpy(), dtype, "o vs two calls")
    assert_close(u2, u2b.double().cpu().numpy(), dtype, "u vs two calls")
    untouched = np.flatnonzero(acc == 0)
    assert torch.equal(S[untouched], d1["state"][untouched])


def test_commit_verify_256x4_sampled_sequences():
    """The benchmarked fused round at full size: 256 sequences x 4 drafts x 32 value
    heads keep the previous round's ~U{0..4} accepted drafts and verify the next 4;
    the oracle follows 4 sequences."""
    from linear_attention_recurrence_rule_b200 import gdn_recurrent_commit_verify
    from linear_attention_recurrence_rule_b200.inputs import WORKLOADS, workload_inputs
    w = WORKLOADS["verify_256x4"]
    x1 = workload_inputs("verify_256x4")
    x2 = workload_inputs("verify_256x4", seed_offset=1)
    d1, d2 = to_dev(x1), to_dev(x2)
    gen = torch.Generator().manual_seed(w.seed + 77)
    accepted = torch.randint(0, w.T + 1, (w.B,), generator=gen, dtype=torch.int32)
    _, _, u1 = gdn_recurrent_verify(d1["q"], d1["k"], d1["v"], d1["g"], d1["beta"], d1["state"],
                                    rollback="deltas")
    S = d1["state"].clone()
    o2, _ = gdn_recurrent_commit_verify(d1["k"], d1["g"], u1, accepted.cuda(), d2["q"], d2["k"],
                                        d2["v"], d2["g"], d2["beta"], S)
    torch.cuda.synchronize()
    seqs = [0, 17, 128, 255]
    s1 = {n: x1[n][seqs] for n in ("q", "k", "v", "g", "beta", "state")}
    s2 = {n: x2[n][seqs] for n in ("q", "k", "v", "g", "beta")}
    _, st1 = O.verify(s1["q"], s1["k"], s1["v"], s1["g"], s1["beta"], s1["state"])
    Sc = O.commit(st1, accepted[seqs].numpy(), s1["state"])
    o2_ref, _ = O.verify(s2["q"], s2["k"], s2["v"], s2["g"], s2["beta"], Sc)
    assert_close(S[seqs], Sc, torch.bfloat16, "committed state")
    assert_close(o2[seqs], o2_ref, torch.bfloat16, "o")
