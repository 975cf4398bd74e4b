#!/usr/bin/env python
"""Benchmark of the gated delta rule hot path on B200.

Metric: "GDN prefill tokens/s (T=64K, 32 V heads); decode state HBM GB/s vs peak".

One step = one chunkwise prefill (``gdn_chunk_prefill``) of a Qwen3-Next
Gated DeltaNet layer over one synthetic sequence: B=1, T=65536, 16 query/key
heads shared by 32 value heads, head dim 128, chunk 64, bf16 q/k/v, fp32
g/beta/state.  The same run also measures the fused decode step
(``gdn_recurrent_step``) on 256 sequences x 64 tokens and reports its state
HBM bandwidth in the ``decode`` object, the speculative-decoding round
(``gdn_recurrent_verify`` of 4 drafts per sequence + the commit of the accepted
prefix) in the ``verify`` object, the fused input prologue and one decay per
value row in the ``prologue`` object, and the layer steps around the rule (the
short convolution on the values and the output gate, in the prefill and in
the decode step) in the ``layer`` object.  ``--no-decode``, ``--no-verify``,
``--no-prologue``, ``--no-layer``, ``--no-configs``, ``--no-e2e`` and ``--no-cpu-baseline`` skip
the respective legs.

Launch: ``python bench.py [--gpus N --steps K --warmup W]``; for N > 1 under
``torch.distributed.run``, one replica per GPU (each rank runs its own
sequence; no data-path collective; ``scaling: weak``).  ``--impl reference``
times the float64 CPU oracle on the host cores instead (the reference arm).
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN prefill tokens/s (T=64K, 32 V heads); decode state HBM GB/s vs peak"
WORKLOAD = "long_prefill_64k"
DECODE_WORKLOAD = "decode_256x64"
VERIFY_WORKLOAD = "verify_256x4"

# Fallback peaks (only if the measured-peaks file is absent).
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
N_SM = 148
FP32_FMA_PER_SM_PER_CLK = 128


def prefill_flops_per_token(HK, HV, d, C):
    """Algorithmic FLOPs of the chunkwise form per token: per query/key head the
    stacked [Q;K] K^T products (4 C d); per value head W, U~ and P U (6 C d) plus
    the three state products W S^T, Q S^T and U^T K (6 d^2)."""
    return HK * 4 * C * d + HV * (6 * C * d + 6 * d * d)


def prefill_min_bytes_per_token(HK, HV, d, elt=2):
    """Mandatory HBM bytes per token: read q, k, v, g, beta, write o."""
    return 2 * HK * d * elt + 2 * HV * d * elt + 2 * HV * 4


def decode_bytes_per_step(N, HK, HV, dk, dv, elt=2):
    """State read + write (fp32) plus q, k, v, o, g, beta."""
    return 2 * N * HV * dv * dk * 4 + 2 * N * HK * dk * elt + 2 * N * HV * dv * elt + 2 * N * HV * 4


def verify_bytes(N, K, HK, HV, dk, dv, accepted, rollback, elt=2):
    """Algorithmic HBM bytes of one verify + commit round (state fp32).

    verify: the state read once, q, k, v, o, g, beta of K drafts, plus either
    every draft's state ("states") or every draft's update vector u ("deltas").
    commit: the state of each sequence that kept >= 1 draft read and written
    once; the deltas form also reads k, g and u of the kept drafts, the states
    form the selected state instead of the current one."""
    state = HV * dv * dk * 4                      # one sequence
    io = N * K * (2 * HK * dk * elt + 2 * HV * dv * elt + 2 * HV * 4)
    kept = sum(1 for a in accepted if 1 <= a <= K)
    drafts_kept = sum(a for a in accepted if 1 <= a <= K)
    if rollback == "fused":   # commit of the previous round's drafts, then verify, one pass
        ver = (N * state + kept * state + io + N * K * HV * dv * 4 +
               drafts_kept * (HK * dk * elt + HV * 4 + HV * dv * 4) + N * 4)
        com = 0
    elif rollback == "states":
        ver = N * state * (1 + K) + io
        com = kept * 2 * state + N * 4
    else:
        ver = N * state + io + N * K * HV * dv * 4
        com = kept * 2 * state + drafts_kept * (HK * dk * elt + HV * 4 + HV * dv * 4) + N * 4
    return ver, com


def measure_verify(gdn, torch, dev, stream, peaks, peak_src, rank, world, max_over_ranks,
                   barrier, args):
    """Speculative-decoding round on the verify_256x4 workload: K=4 drafts per
    sequence checked in one pass (``gdn_recurrent_verify``), then the accepted
    prefix kept (``gdn_state_commit_deltas`` / ``gdn_state_commit``).  The
    acceptance counts are synthetic, ~U{0..K} per sequence from the seed."""
    from linear_attention_recurrence_rule_b200.inputs import WORKLOADS, workload_inputs
    name = VERIFY_WORKLOAD
    wv = WORKLOADS[name]
    y = workload_inputs(name, seed_offset=replica_seed_offset(rank))
    dy = {k: v.to(dev) for k, v in y.items()}
    N, K = wv.B, wv.T
    gen = torch.Generator().manual_seed(wv.seed + 77 + rank)
    acc_host = torch.randint(0, K + 1, (N,), generator=gen, dtype=torch.int32)
    accepted = acc_host.to(dev)
    S = dy["state"].clone()
    o = torch.empty_like(dy["v"])
    u = torch.empty((N, K, wv.HV, wv.dv), dtype=torch.float32, device=dev)
    states = torch.empty((N, K, wv.HV, wv.dv, wv.dk), dtype=torch.float32, device=dev)
    hbm_peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    out = {"workload": name, "drafts": K, "sequences": N,
           "accepted_mean": float(acc_host.float().mean()),
           "acceptance": "synthetic ~U{0..K} per sequence"}
    rounds = max(1, args.verify_rounds)
    # fused rounds: each call keeps the previous round's accepted drafts, then
    # verifies this round's (the same draft inputs every round, u alternating)
    u_alt = torch.empty_like(u)
    fws = torch.empty(gdn.gdn_recurrent_commit_verify_workspace_size(N, K, K, wv.HV, wv.dk),
                      dtype=torch.uint8, device=dev)

    def fused_round(prev_u, new_u):
        gdn.gdn_recurrent_commit_verify(dy["k"], dy["g"], prev_u, accepted, dy["q"], dy["k"],
                                        dy["v"], dy["g"], dy["beta"], S, o=o, u_out=new_u,
                                        workspace=fws, stream=stream)

    S.copy_(dy["state"])
    gdn.gdn_recurrent_verify(dy["q"], dy["k"], dy["v"], dy["g"], dy["beta"], S, o=o, u_out=u,
                             rollback="deltas", stream=stream)
    bufs = [u, u_alt]
    for w_ in range(max(3, args.warmup)):
        fused_round(bufs[w_ & 1], bufs[(w_ + 1) & 1])
    torch.cuda.synchronize()
    barrier()
    fsampler = ClockSampler(int(dev.index or 0))
    fsampler.start()
    fev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(rounds)]
    for r_, (a_, b_) in enumerate(fev):
        a_.record(stream)
        fused_round(bufs[r_ & 1], bufs[(r_ + 1) & 1])
        b_.record(stream)
    torch.cuda.synchronize()
    barrier()
    fclocks = fsampler.stop()
    f_ms = statistics.mean(a_.elapsed_time(b_) for a_, b_ in fev)
    ftotal = max_over_ranks(fev[0][0].elapsed_time(fev[-1][1]))
    fb, _ = verify_bytes(N, K, wv.HK, wv.HV, wv.dk, wv.dv, acc_host.tolist(), "fused")
    f_gbs = fb / (f_ms / 1e3) / 1e9
    out["fused"] = {
        "value": world * N * K * rounds / (ftotal / 1e3), "unit": "draft tokens/s",
        "ms_per_round": ftotal / rounds, "bytes_per_round": fb,
        "roofline": {"bound": "hbm", "achieved": f_gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": f_gbs / hbm_peak, "traffic": kernel_traffic("verify_fused"),
                     "peak_source": peak_src, "kernel": "verify_wy (commit fused)"},
        "gpu_launches": 2 * rounds, "clocks": fclocks,
        "call": "gdn_recurrent_commit_verify: previous round's commit + this round's verify"}
    for form in ("deltas", "states"):
        def verify():
            if form == "deltas":
                gdn.gdn_recurrent_verify(dy["q"], dy["k"], dy["v"], dy["g"], dy["beta"], S, o=o,
                                         u_out=u, rollback="deltas", stream=stream)
            else:
                gdn.gdn_recurrent_verify(dy["q"], dy["k"], dy["v"], dy["g"], dy["beta"], S, o=o,
                                         states_out=states, rollback="states", stream=stream)

        def commit():
            if form == "deltas":
                gdn.gdn_state_commit_deltas(dy["k"], dy["g"], u, accepted, S, stream=stream)
            else:
                gdn.gdn_state_commit(states, accepted, S, stream=stream)

        S.copy_(dy["state"])
        for _ in range(max(3, args.warmup)):
            verify()
            commit()
        S.copy_(dy["state"])
        torch.cuda.synchronize()
        barrier()
        sampler = ClockSampler(int(dev.index or 0))
        sampler.start()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(rounds)]
        for r in range(rounds):
            ev[r][0].record(stream)
            verify()
            ev[r][1].record(stream)
            commit()
            ev[r][2].record(stream)
        torch.cuda.synchronize()
        barrier()
        clocks = sampler.stop()
        v_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
        c_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
        total_ms = max_over_ranks(ev[0][0].elapsed_time(ev[-1][2]))
        vb, cb = verify_bytes(N, K, wv.HK, wv.HV, wv.dk, wv.dv, acc_host.tolist(), form)
        v_gbs = vb / (v_ms / 1e3) / 1e9
        c_gbs = cb / (c_ms / 1e3) / 1e9
        out[form] = {
            "value": world * N * K * rounds / (total_ms / 1e3), "unit": "draft tokens/s",
            "ms_per_round": total_ms / rounds, "verify_ms": v_ms, "commit_ms": c_ms,
            "bytes_per_round": vb + cb, "gb_per_s": (vb + cb) / (total_ms / rounds / 1e3) / 1e9,
            "roofline": {"bound": "hbm", "achieved": v_gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": v_gbs / hbm_peak, "traffic": kernel_traffic("verify_" + form),
                         "peak_source": peak_src,
                         "kernel": "verify_tc" if form == "deltas" else "verify"},
            "commit_roofline": {"bound": "hbm", "achieved": c_gbs, "peak": hbm_peak,
                                "unit": "GB/s", "frac": c_gbs / hbm_peak},
            "gpu_launches": 2 * rounds, "clocks": clocks}
    return out


def measure_prologue(gdn, torch, dev, stream, x, w, ws, o, hT, rank, barrier, max_over_ranks,
                     plain_s, args):
    """Prefill (the bench workload) and one decode step (decode_256x64 shapes)
    with every prologue flag on raw projections: q, k rows of norm ~U(0.25, 4)
    and gate logits.  Reported beside the plain kernels' times."""
    from linear_attention_recurrence_rule_b200.inputs import (WORKLOADS, raw_projections,
                                                              workload_inputs)
    flags = gdn.PROLOGUE_ALL
    r = raw_projections(x, seed=900 + rank)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in r.items()}
    tokens = d["q"].shape[0] * d["q"].shape[1]

    def step():
        gdn.gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], chunk=w.chunk, o=o,
                              hT=hT, workspace=ws, stream=stream, prologue=flags)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    barrier()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for a_, b_ in ev:
        a_.record(stream)
        step()
        b_.record(stream)
    torch.cuda.synchronize()
    pf_s = statistics.mean(a_.elapsed_time(b_) for a_, b_ in ev) / 1e3
    total_ms = max_over_ranks(ev[0][0].elapsed_time(ev[-1][1]))
    del d
    # decode: one step over the decode workload's 256 sequences, raw inputs
    wd = WORKLOADS[DECODE_WORKLOAD]
    y = raw_projections(workload_inputs(DECODE_WORKLOAD, steps=8,
                                        seed_offset=replica_seed_offset(rank)), seed=901 + rank)
    dy = {k: v.to(dev) for k, v in y.items()}
    S = dy["state"].clone()
    od = torch.empty_like(dy["v"][0])
    res = {}
    # one decay per value row (the per-channel forget gate), logits from the same draw
    from linear_attention_recurrence_rule_b200.inputs import row_decays
    g_rows = row_decays((8,) + tuple(dy["v"].shape[1:]), seed=902 + rank).to(dev)
    for tag, fl in (("plain", 0), ("prologue", flags), ("row_decay", gdn.ROW_DECAY)):
        gsel = g_rows if fl & gdn.ROW_DECAY else dy["g"]
        for t in range(3):
            gdn.gdn_recurrent_step(dy["q"][t], dy["k"][t], dy["v"][t], gsel[t], dy["beta"][t],
                                   S, o=od, stream=stream, prologue=fl)
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(8)]
        for t, (a_, b_) in enumerate(evs):
            a_.record(stream)
            gdn.gdn_recurrent_step(dy["q"][t], dy["k"][t], dy["v"][t], gsel[t], dy["beta"][t],
                                   S, o=od, stream=stream, prologue=fl)
            b_.record(stream)
        torch.cuda.synchronize()
        res[tag] = statistics.mean(a_.elapsed_time(b_) for a_, b_ in evs)
    # the chunked prefill with one decay per value row (CUDA-core path) on the 4K layer
    from linear_attention_recurrence_rule_b200.inputs import workload_inputs as _wi
    wl = WORKLOADS["layer_prefill_4k"]
    z = {k_: (v_.to(dev) if isinstance(v_, torch.Tensor) else v_)
         for k_, v_ in _wi("layer_prefill_4k", seed_offset=replica_seed_offset(rank)).items()}
    gz = row_decays(tuple(z["v"].shape), seed=903 + rank).to(dev)
    oz = torch.empty_like(z["v"])

    def rd_prefill():
        gdn.gdn_chunk_prefill(z["q"], z["k"], z["v"], gz, z["beta"], chunk=wl.chunk, o=oz,
                              stream=stream, prologue=gdn.ROW_DECAY)

    rd_prefill()
    torch.cuda.synchronize()
    rev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(3)]
    for a_, b_ in rev:
        a_.record(stream)
        rd_prefill()
        b_.record(stream)
    torch.cuda.synchronize()
    rd_ms = statistics.mean(a_.elapsed_time(b_) for a_, b_ in rev)
    ztok = z["q"].shape[0] * z["q"].shape[1]
    return {"flags": "norm_q|norm_k|gate_logits",
            "prefill_row_decay": {"workload": "layer_prefill_4k", "path": "cuda-core",
                                  "ms_per_step": rd_ms, "value": ztok / (rd_ms / 1e3),
                                  "unit": "tokens/s", "gpu_launches": 4,
                                  "decays": "one per value row, alpha ~U(0.8, 1)"},
            "prefill": {"workload": WORKLOAD, "value": tokens * args.steps / (total_ms / 1e3),
                        "unit": "tokens/s", "ms_per_step": pf_s * 1e3,
                        "plain_ms_per_step": plain_s * 1e3,
                        "overhead": pf_s / plain_s - 1.0, "gpu_launches": args.steps},
            "decode": {"workload": DECODE_WORKLOAD, "ms_per_step": res["prologue"],
                       "plain_ms_per_step": res["plain"],
                       "overhead": res["prologue"] / res["plain"] - 1.0, "gpu_launches": 11},
            "decode_row_decay": {"workload": DECODE_WORKLOAD, "ms_per_step": res["row_decay"],
                                 "overhead": res["row_decay"] / res["plain"] - 1.0,
                                 "gpu_launches": 11,
                                 "decays": "one per value row, alpha ~U(0.8, 1)"},
            "inputs": "raw projections: q, k rows of norm ~U(0.25, 4), forget logits ~N(3, 1), "
                      "write logits ~N(0, 1)"}


def _time_events(torch, stream, fn, reps, warm=3):
    """Mean CUDA-event time (ms) of ``fn`` on ``stream`` over ``reps`` launches."""
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    for a_, b_ in ev:
        a_.record(stream)
        fn()
        b_.record(stream)
    torch.cuda.synchronize()
    return statistics.mean(a_.elapsed_time(b_) for a_, b_ in ev)


def measure_layer(gdn, torch, dev, stream, x, w, o, hT, rank, peaks, peak_src, plain_s, args):
    """The layer steps around the rule: the bench prefill with the short
    convolution on v (width 4, bias, no activation, carried state) and the output gate (fused
    into the prefill's read-out), one call; the convolution and the standalone
    gate kernels alone with their HBM rooflines; and the decode step of
    decode_256x64 with both fused into it."""
    from linear_attention_recurrence_rule_b200.inputs import (WORKLOADS, layer_extras,
                                                              workload_inputs)
    W = 4
    B, T, HV, dv = x["v"].shape
    C = HV * dv
    ex = layer_extras(B, C, W, tuple(x["v"].shape), torch.bfloat16, seed=950 + rank)
    e = {k: v.to(dev) for k, v in ex.items()}
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    tokens = B * T
    ws = torch.empty(gdn.gdn_chunk_prefill_layer_workspace_size(
        B, T, w.HK, w.HV, w.dk, w.dv, w.chunk, w.dtype, 0, 1, 1), dtype=torch.uint8, device=dev)
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])

    def layer_prefill():
        gdn.gdn_chunk_prefill_layer(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                    conv_weight=e["conv_weight"], conv_bias=e["conv_bias"],
                                    conv_state=e["conv_state"], z=e["z"], chunk=w.chunk, o=o,
                                    hT=hT, workspace=ws, stream=stream)

    lp_ms = _time_events(torch, stream, layer_prefill, max(args.steps, 3))
    y = torch.empty_like(d["v"])
    vin = d["v"].reshape(B, T, C)

    def conv(silu):
        gdn.gdn_short_conv(vin, e["conv_weight"], e["conv_bias"], e["conv_state"], silu=silu,
                           y=y.reshape(B, T, C), stream=stream)

    # the layer's configuration (no activation), then with SiLU
    cv_ms = _time_events(torch, stream, lambda: conv(False), 10)
    cvs_ms = _time_events(torch, stream, lambda: conv(True), 10)
    elt = 2
    cv_bytes = 2 * tokens * C * elt + 2 * B * (W - 1) * C * elt + C * (W + 1) * 4

    def gate():
        gdn.gdn_output_gate(o, e["z"], stream=stream)

    gt_ms = _time_events(torch, stream, gate, 10)
    gt_bytes = 3 * tokens * C * elt
    del d, y, ws
    # decode with both steps fused, 256 sequences (decode_256x64 shapes)
    wd = WORKLOADS[DECODE_WORKLOAD]
    yd = workload_inputs(DECODE_WORKLOAD, steps=8, seed_offset=replica_seed_offset(rank))
    dy = {k: v.to(dev) for k, v in yd.items()}
    exd = layer_extras(wd.B, wd.HV * wd.dv, W, (8, wd.B, wd.HV, wd.dv), torch.bfloat16,
                       seed=960 + rank)
    ed = {k: v.to(dev) for k, v in exd.items()}
    S = dy["state"].clone()
    od = torch.empty_like(dy["v"][0])
    it = [0]

    def dstep(layer):
        t = it[0] % 8
        it[0] += 1
        if layer:
            gdn.gdn_recurrent_step_layer(dy["q"][t], dy["k"][t], dy["v"][t], dy["g"][t],
                                         dy["beta"][t], S, conv_weight=ed["conv_weight"],
                                         conv_bias=ed["conv_bias"], conv_state=ed["conv_state"],
                                         z=ed["z"][t], o=od, stream=stream, silu=True)
        else:
            gdn.gdn_recurrent_step(dy["q"][t], dy["k"][t], dy["v"][t], dy["g"][t], dy["beta"][t],
                                   S, o=od, stream=stream)

    plain_d = _time_events(torch, stream, lambda: dstep(False), 8)
    layer_d = _time_events(torch, stream, lambda: dstep(True), 8)
    dbytes = (decode_bytes_per_step(wd.B, wd.HK, wd.HV, wd.dk, wd.dv)
              + 2 * wd.B * (W - 1) * wd.HV * wd.dv * elt + wd.B * wd.HV * wd.dv * elt)
    dach = dbytes / (layer_d / 1e3) / 1e9
    return {"conv": "causal depthwise, width 4, bias, no activation, carried state "
                    "(the standalone kernel also timed with SiLU)",
            "gate": "o * sigmoid(z)",
            "prefill": {"workload": WORKLOAD, "ms_per_step": lp_ms,
                        "value": tokens / (lp_ms / 1e3), "unit": "tokens/s",
                        "plain_ms_per_step": plain_s * 1e3, "overhead": lp_ms / (plain_s * 1e3) - 1.0,
                        "gpu_launches": 3,
                        "launches": "convolution with the gate factors in the same pass, carried "
                                    "state, prefill (gate applied in its read-out)"},
            "conv_kernel": {"ms": cv_ms, "bytes": cv_bytes, "gpu_launches": 2,
                            "roofline": {"bound": "hbm", "achieved": cv_bytes / (cv_ms / 1e3) / 1e9,
                                         "peak": hbm, "unit": "GB/s",
                                         "frac": cv_bytes / (cv_ms / 1e3) / 1e9 / hbm,
                                         "traffic": kernel_traffic("short_conv"),
                                         "peak_source": peak_src, "kernel": "conv"}},
            "conv_kernel_silu": {"ms": cvs_ms, "bytes": cv_bytes, "gpu_launches": 2,
                                 "roofline": {"bound": "hbm",
                                              "achieved": cv_bytes / (cvs_ms / 1e3) / 1e9,
                                              "peak": hbm, "unit": "GB/s",
                                              "frac": cv_bytes / (cvs_ms / 1e3) / 1e9 / hbm,
                                              "peak_source": peak_src, "kernel": "conv with SiLU"}},
            "gate_kernel": {"ms": gt_ms, "bytes": gt_bytes, "gpu_launches": 1,
                            "roofline": {"bound": "hbm", "achieved": gt_bytes / (gt_ms / 1e3) / 1e9,
                                         "peak": hbm, "unit": "GB/s",
                                         "frac": gt_bytes / (gt_ms / 1e3) / 1e9 / hbm,
                                         "traffic": kernel_traffic("output_gate"),
                                         "peak_source": peak_src, "kernel": "gate"}},
            "decode": {"workload": DECODE_WORKLOAD, "ms_per_step": layer_d,
                       "plain_ms_per_step": plain_d, "overhead": layer_d / plain_d - 1.0,
                       "bytes_per_step": dbytes, "gpu_launches": 8,
                       "roofline": {"bound": "hbm", "achieved": dach, "peak": hbm, "unit": "GB/s",
                                    "frac": dach / hbm, "traffic": kernel_traffic("decode_layer"),
                                    "peak_source": peak_src, "kernel": "decode (layer instance)"}}}


def dist_max(x, device=None):
    """Max of a host float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(world, units_per_rank, steps, max_ms):
    """Whole-job throughput: units every rank processed over the slowest rank's time."""
    return world * units_per_rank * steps / (max_ms / 1000.0)


def replica_seed_offset(rank):
    """Each replica draws its own sequence of the same workload."""
    return rank


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# DRAM traffic per launch of the dominant kernels, from the ncu captures
# summarised under profiles/ (dram__bytes_read.sum + dram__bytes_write.sum).
# Each entry carries the sha256 of the kernel source it was taken on; a changed
# source reports null.
NCU_TRAFFIC = {
    # full decode_256x64 step: 541,171,712 read + 476,291,072 written
    "decode": {"bytes": 1017462784, "source": "gdn_decode.cu",
               "sha256": "342c1ce55a1419f66a4d3b79e1f521987b47cfa44938be1fd8bc6c150858c6b6"},
    # the same step with the short convolution and the output gate fused (layer
    # instance): 549,628,160 read + 482,972,928 written
    "decode_layer": {"bytes": 1032601088, "source": "gdn_decode.cu",
                     "sha256": "342c1ce55a1419f66a4d3b79e1f521987b47cfa44938be1fd8bc6c150858c6b6"},
    # full long_prefill_64k launch of the ring prefill: 1,102,597,376 read + 514,424,064
    # written (algorithmic 1,627,389,952)
    "prefill_ring": {"bytes": 1617021440, "source": "gdn_prefill_ring.cu",
                     "sha256": "60d3e2431e39242ff1549de34f0749eda08d3036e9c679e38c9be45722cf180b"},
    # the same workload on the cluster kernel (no-allocation entry point): 1,091,336,960
    # read + 509,906,688 written
    "prefill_cluster": {"bytes": 1601243648, "source": "gdn_prefill_cluster.cu",
                        "sha256": "4ef0fef23fee2a3208626b5a458640654ce023f7ea5ab71922fbe7ecd21b2990"},
    # short convolution of the 64K bench values (width 4): 540,828,672 read + 483,701,248
    # written (its carried-state launch adds 55,296)
    "short_conv": {"bytes": 1024529920, "source": "gdn_layer.cu",
                   "sha256": "03e2d96c3e8a4dbc194fc0970d48afd7b79fc033f0bb351a248b95dfc9e837bd"},
    # standalone output gate over the 64K bench outputs: 1,073,846,528 read + 492,012,288 written
    "output_gate": {"bytes": 1565858816, "source": "gdn_layer.cu",
                    "sha256": "03e2d96c3e8a4dbc194fc0970d48afd7b79fc033f0bb351a248b95dfc9e837bd"},
    # verify_256x4, update-vector form, the tensor-core kernel: 579,903,488 read +
    # 24,379,904 written (its setup kernel adds 8,682,752)
    "verify_deltas": {"bytes": 604283392, "source": "gdn_verify.cu",
                      "sha256": "19b8174a5cb7f9ff183a9cf3f22d26aca35eac177b8e8b360788a170159747f9"},
    # verify_256x4, per-draft states: 554,959,104 read + 2,092,982,784 written
    "verify_states": {"bytes": 2647941888, "source": "gdn_verify.cu",
                      "sha256": "19b8174a5cb7f9ff183a9cf3f22d26aca35eac177b8e8b360788a170159747f9"},
    # verify_256x4 fused round (previous commit + verify), the streaming kernel:
    # 613,593,856 read + 382,361,600 written
    "verify_fused": {"bytes": 995955456, "source": "gdn_verify.cu",
                     "sha256": "19b8174a5cb7f9ff183a9cf3f22d26aca35eac177b8e8b360788a170159747f9"},
}


def kernel_traffic(key, units_scale=1.0):
    e = NCU_TRAFFIC.get(key)
    if not e:
        return None
    src = os.path.join(ROOT, "linear_attention_recurrence_rule_b200", "csrc", e["source"])
    try:
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except OSError:
        return None
    if h != e["sha256"]:
        return None
    return e["bytes"] * units_scale


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.lines = []
        self.device_index = device_index

    def start(self):
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.device_index).uuid)
            sel = ["-i", "GPU-" + uuid if not uuid.startswith("GPU-") else uuid]
        except Exception:
            sel = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline leg and reference arm)
# ---------------------------------------------------------------------------
def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def time_oracle_prefill(tokens, seed_offset=0):
    """Seconds the float64 oracle takes on the first ``tokens`` tokens of the
    benchmark workload (all 32 value heads), on every host core."""
    from linear_attention_recurrence_rule_b200.inputs import workload_inputs
    from oracle import gdn_oracle as O
    x = workload_inputs(WORKLOAD, tokens=tokens, seed_offset=seed_offset)
    t0 = time.perf_counter()
    O.prefill(x["q"], x["k"], x["v"], x["g"], x["beta"], nthreads=host_cores())
    return time.perf_counter() - t0


def cpu_sample_tokens(target_s):
    """Tokens of the workload the oracle processes in about ``target_s`` seconds."""
    probe = 512
    dt = max(time_oracle_prefill(probe), 1e-3)
    tok = int(probe * target_s / dt)
    return max(512, min(65536, (tok // 256) * 256))


def cpu_baseline(target_s=12.0):
    tok = cpu_sample_tokens(target_s)
    dt = time_oracle_prefill(tok)
    return {"value": tok / dt, "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
            "sample": f"first {tok} of 65536 tokens of the benchmark workload, all 32 value "
                      f"heads, float64 token-by-token recurrence, {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    tok = cpu_sample_tokens(args.ref_step_seconds)
    for i in range(args.warmup):
        time_oracle_prefill(tok)
    times = [time_oracle_prefill(tok) for _ in range(args.steps)]
    total = sum(times)
    value = tok * args.steps / total
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD, "B": 1, "T": 65536, "HK": 16, "HV": 32, "d": 128,
                   "chunk": 64, "parallelism": "replicas" if world > 1 else "single",
                   "sample_tokens_per_step": tok},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": host_cores(),
                         "kind": "oracle",
                         "sample": f"first {tok} of 65536 tokens per step, all 32 value heads"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def measure_s0_pair_cost(gdn, torch, d, w, o, hT, stream, ring_ms):
    """What carrying S0 as a bf16 hi + lo pair in the read-out costs: the same 64K
    prefill through the no-allocation entry point, whose tensor-core kernel (the
    cluster design with a DSMEM hand-over) reads out with a single-bf16 S0.  The
    two kernels also differ in their hand-over (DSMEM against the L2 ring), so
    the difference bounds the pair's cost from above."""
    import ctypes
    from linear_attention_recurrence_rule_b200 import gdn as core
    P = ctypes.c_void_p
    lib = core.load_library()
    f = lib.gdn_chunk_prefill_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [P, P, P, P, P, P, P, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_int, P, P, P]
    B, T = d["q"].shape[0], d["q"].shape[1]
    sp = P(stream.cuda_stream)

    def call():
        rc = f(P(d["q"].data_ptr()), P(d["k"].data_ptr()), P(d["v"].data_ptr()), P(d["g"].data_ptr()),
               P(d["beta"].data_ptr()), None, None, B, T, w.HK, w.HV, w.dk, w.dv, w.chunk, 1.0,
               core.GDN_BF16, P(o.data_ptr()), P(hT.data_ptr()), sp)
        if rc != core.GDN_OK:
            raise RuntimeError(core.status_string(rc))

    ms = _time_events(torch, stream, call, 5)
    return {"single_bf16_s0_ms": ms, "pair_s0_ms": ring_ms, "difference_ms": ring_ms - ms,
            "kernels": "prefill_cluster_kernel (no-allocation entry point) against prefill_ring_kernel",
            "gpu_launches": 1}


def measure_configs(gdn, torch, dev, stream, peaks, peak_src, rank, args):
    """The other prefill workloads of the suite, each timed on its own (one call per
    step, CUDA events on the launching stream, 3 warm-up calls): tokens/s and the
    fraction of the roofline that bounds its path -- the bf16 tensor peak for the
    tensor-core path, the fp32 FMA peak (148 SMs x 128 FMA x 2 x max clock) for the
    CUDA-core path.  A step is one launch of ours plus the status-word reset."""
    from linear_attention_recurrence_rule_b200.inputs import WORKLOADS, workload_inputs
    out = {}
    for name in ("layer_prefill_4k", "varlen_8", "tiny_fp32"):
        w = WORKLOADS[name]
        x = workload_inputs(name, seed_offset=replica_seed_offset(rank))
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
        cu = d["cu_seqlens"]
        B, T = d["q"].shape[0], d["q"].shape[1]
        N = (cu.numel() - 1) if cu is not None else B
        tokens = B * T
        ws_b = gdn.gdn_chunk_prefill_workspace_size(N, T if cu is not None else T, w.HK, w.HV, w.dk,
                                                    w.dv, w.chunk, w.dtype, cu is not None)
        ws = torch.empty(max(ws_b, 1), dtype=torch.uint8, device=dev) if ws_b else None
        o = torch.empty_like(d["v"])
        hT = torch.empty((N, w.HV, w.dv, w.dk), dtype=torch.float32, device=dev)

        def call():
            gdn.gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"],
                                  cu_seqlens=cu, chunk=w.chunk, o=o, hT=hT, workspace=ws,
                                  stream=stream)

        reps = 10
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        for a_, b_ in evs:
            a_.record(stream)
            call()
            b_.record(stream)
        torch.cuda.synchronize()
        ms = statistics.median(a_.elapsed_time(b_) for a_, b_ in evs)
        flops = prefill_flops_per_token(w.HK, w.HV, w.dk, w.chunk) * tokens
        tc = gdn.gdn_chunk_prefill_path(w.dk, w.dv, w.chunk, w.dtype) == 1
        if tc:
            peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
            bound = "tensor"
        else:
            mhz = peaks.get("sm_max_mhz", FALLBACK_PEAKS["sm_max_mhz"])
            peak = N_SM * FP32_FMA_PER_SM_PER_CLK * 2 * mhz * 1e6 / 1e12
            bound = "alu"
        achieved = flops / (ms / 1e3) / 1e12
        out[name] = {"value": tokens / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
                     "tokens": tokens, "sequences": N, "path": "tcgen05" if tc else "cuda-core",
                     "dtype": "bf16" if w.dtype == torch.bfloat16 else "fp32",
                     "roofline": {"bound": bound, "achieved": achieved, "peak": peak,
                                  "unit": "TFLOP/s", "frac": achieved / peak,
                                  "peak_source": peak_src if tc else "derived (unit counts x max clock)"},
                     "gpu_launches_per_step": 1,
                     "h0": "nonzero" if x["h0"] is not None else "zero"}
    return out


def run_b200(args):
    import torch
    import torch.distributed as dist

    import linear_attention_recurrence_rule_b200 as gdn
    from linear_attention_recurrence_rule_b200.inputs import WORKLOADS, workload_inputs

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: WORLD_SIZE={world} but --gpus {args.gpus}", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return dist_max(x, dev)

    peaks, peak_src = load_peaks()
    w = WORKLOADS[WORKLOAD]
    x = workload_inputs(WORKLOAD, seed_offset=replica_seed_offset(rank), tokens=args.tokens)
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    B, T = d["q"].shape[0], d["q"].shape[1]
    tokens = B * T
    path = gdn.gdn_chunk_prefill_path(w.dk, w.dv, w.chunk, w.dtype)
    ws_bytes = gdn.gdn_chunk_prefill_workspace_size(B, T, w.HK, w.HV, w.dk, w.dv, w.chunk,
                                                    w.dtype, False)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev) if ws_bytes else None
    o = torch.empty_like(d["v"])
    hT = torch.empty((B, w.HV, w.dv, w.dk), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    launches_per_step = 1  # one kernel per call on either path (the status memset is not a kernel of ours)

    def step():
        gdn.gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], chunk=w.chunk, o=o,
                              hT=hT, workspace=ws, stream=stream)

    n_steps = 0 if args.no_prefill else args.steps
    for _ in range(0 if args.no_prefill else args.warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(max(n_steps, 1))]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(n_steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    elapsed_ms = t0.elapsed_time(t1)
    launch_ms = [a.elapsed_time(b) for a, b in ev[:n_steps]] or [float("nan")]
    elapsed_ms = max_over_ranks(elapsed_ms)
    value = aggregate_throughput(world, tokens, n_steps, elapsed_ms) if n_steps else None
    mean_launch_s = statistics.mean(launch_ms) / 1000.0

    flops = prefill_flops_per_token(w.HK, w.HV, w.dk, w.chunk) * tokens
    if path == 1:
        peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        roof = {"bound": "tensor", "achieved": flops / mean_launch_s / 1e12, "peak": peak,
                "unit": "TFLOP/s"}
        kernel_key = "prefill_ring"
    else:
        mhz = peaks.get("sm_max_mhz", FALLBACK_PEAKS["sm_max_mhz"])
        peak = N_SM * FP32_FMA_PER_SM_PER_CLK * 2 * mhz * 1e6 / 1e12
        roof = {"bound": "alu", "achieved": flops / mean_launch_s / 1e12, "peak": peak,
                "unit": "TFLOP/s"}
        kernel_key = "prefill_simt"
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = kernel_traffic(kernel_key)
    roof["peak_source"] = peak_src
    roof["kernel"] = kernel_key
    if not n_steps:
        roof = None

    # ---- end to end through the public call, host buffers, copies timed ----
    e2e = None
    if not args.no_e2e and n_steps:
        names = ("q", "k", "v", "g", "beta")
        host_in = {n: x[n].pin_memory() for n in names}
        host_o = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        host_h = torch.empty(hT.shape, dtype=hT.dtype, pin_memory=True)
        h2d = sum(host_in[n].numel() * host_in[n].element_size() for n in names)
        d2h = host_o.numel() * host_o.element_size() + host_h.numel() * host_h.element_size()
        e_steps = max(1, min(args.steps, args.e2e_steps))

        # the host-memory entry point streams segments: the copies of one segment
        # overlap the computation of the next on the public call's three streams
        h_ws = torch.empty(gdn.gdn_chunk_prefill_host_workspace_size(
            B, T, w.HK, w.HV, w.dk, w.dv, w.chunk, w.dtype, 0), dtype=torch.uint8, device=dev)

        def e2e_step():
            gdn.gdn_chunk_prefill_host(host_in["q"], host_in["k"], host_in["v"], host_in["g"],
                                       host_in["beta"], chunk=w.chunk, o=host_o, hT=hT,
                                       workspace=h_ws, device=dev, stream=stream)
            host_h.copy_(hT, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        e_ms = max_over_ranks(a.elapsed_time(b))
        # what the copies alone cost on this machine: the step's inputs host -> device and
        # its outputs device -> host as plain pinned copies on one stream
        dbuf = {n: torch.empty(host_in[n].shape, dtype=host_in[n].dtype, device=dev) for n in names}
        dout = torch.empty(o.shape, dtype=o.dtype, device=dev)

        def timed(fn, reps=3):
            fn()
            torch.cuda.synchronize()
            a_ = torch.cuda.Event(enable_timing=True)
            b_ = torch.cuda.Event(enable_timing=True)
            a_.record(stream)
            for _ in range(reps):
                fn()
            b_.record(stream)
            torch.cuda.synchronize()
            return a_.elapsed_time(b_) / reps

        h2d_ms = timed(lambda: [dbuf[n].copy_(host_in[n], non_blocking=True) for n in names])
        d2h_ms = timed(lambda: (host_o.copy_(dout, non_blocking=True),
                                host_h.copy_(hT, non_blocking=True)))
        kern_ms = mean_launch_s * 1e3
        serial_ms = h2d_ms + kern_ms + d2h_ms
        # with the two copy directions and the kernels all overlapped the step could
        # take as little as the slowest of the three
        bound_ms = max(h2d_ms, d2h_ms, kern_ms)
        step_ms = e_ms / e_steps
        e2e = {"value": world * tokens * e_steps / (e_ms / 1000.0), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e_steps,
               "ms_per_step": step_ms, "segments": -(-T // 4096), "segment_tokens": 4096,
               "h2d_gbs": h2d / (h2d_ms / 1e3) / 1e9, "d2h_gbs": d2h / (d2h_ms / 1e3) / 1e9,
               "h2d_alone_ms": h2d_ms, "d2h_alone_ms": d2h_ms, "kernel_alone_ms": kern_ms,
               "serial_ms": serial_ms, "bound_ms": bound_ms,
               "overlap": (serial_ms - step_ms) / (serial_ms - bound_ms),
               "note": "overlap = (serial - step) / (serial - bound): 0 when the copies and "
                       "kernels run one after another, 1 when the step takes only its slowest "
                       "part (here the host-to-device copy of the inputs)"}

    # ---- decode: 256 sequences x 64 single-token steps ----
    dec = None
    if not args.no_decode:
        wd = WORKLOADS[DECODE_WORKLOAD]
        y = workload_inputs(DECODE_WORKLOAD, seed_offset=replica_seed_offset(rank))
        dy = {k: v.to(dev) for k, v in y.items()}
        S = dy["state"].clone()
        od = torch.empty_like(dy["v"][0])

        def dstep(t):
            gdn.gdn_recurrent_step(dy["q"][t], dy["k"][t], dy["v"][t], dy["g"][t], dy["beta"][t],
                                   S, o=od, stream=stream)

        for t in range(max(3, args.warmup)):
            dstep(t % wd.T)
        S.copy_(dy["state"])
        torch.cuda.synchronize()
        barrier()
        dsampler = ClockSampler(local)
        dsampler.start()
        dev_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(wd.T)]
        for t in range(wd.T):
            dev_ev[t][0].record(stream)
            dstep(t)
            dev_ev[t][1].record(stream)
        torch.cuda.synchronize()
        barrier()
        dclocks = dsampler.stop()
        step_ms = [a_.elapsed_time(b_) for a_, b_ in dev_ev]
        total_ms = max_over_ranks(dev_ev[0][0].elapsed_time(dev_ev[-1][1]))
        bytes_step = decode_bytes_per_step(wd.B, wd.HK, wd.HV, wd.dk, wd.dv)
        mean_s = statistics.mean(step_ms) / 1000.0
        hbm_peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        achieved = bytes_step / mean_s / 1e9
        dec = {"workload": DECODE_WORKLOAD, "value": world * bytes_step * wd.T / (total_ms / 1e3) / 1e9,
               "unit": "GB/s", "tokens_per_s": world * wd.B * wd.T / (total_ms / 1e3),
               "ms_per_step": total_ms / wd.T, "steps": wd.T,
               "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak,
                            "unit": "GB/s", "frac": achieved / hbm_peak,
                            "traffic": kernel_traffic("decode"), "peak_source": peak_src,
                            "kernel": "decode"},
               "bytes_per_step": bytes_step, "gpu_launches": wd.T, "clocks": dclocks,
               "l2": "state 537 MB per step, larger than L2"}

    # ---- the fused input prologue: the same prefill and decode on raw projections ----
    pro = None
    if not args.no_prologue and n_steps:
        pro = measure_prologue(gdn, torch, dev, stream, x, w, ws, o, hT, rank, barrier,
                               max_over_ranks, mean_launch_s, args)

    lay = None
    if not args.no_layer and n_steps:
        lay = measure_layer(gdn, torch, dev, stream, x, w, o, hT, rank, peaks, peak_src,
                            mean_launch_s, args)

    cfgs = None
    if not args.no_configs:
        cfgs = measure_configs(gdn, torch, dev, stream, peaks, peak_src, rank, args)
        if path == 1 and n_steps:
            cfgs["s0_pair_cost"] = measure_s0_pair_cost(gdn, torch, d, w, o, hT, stream,
                                                        mean_launch_s * 1e3)

    ver = None
    if not args.no_verify:
        ver = measure_verify(gdn, torch, dev, stream, peaks, peak_src, rank, world,
                             max_over_ranks, barrier, args)

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": elapsed_ms / n_steps if n_steps else None, "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD if tokens == 65536 else f"{WORKLOAD} truncated to {tokens} tokens",
                       "B": 1, "T": tokens, "HK": 16, "HV": 32, "d": 128,
                       "chunk": 64, "parallelism": "replicas" if world > 1 else "single",
                       "path": "tcgen05" if path == 1 else "cuda-core",
                       "l2": "inputs larger than L2 (q,k,v 1.07 GB per step)"},
            "roofline": roof, "cpu_baseline": base, "e2e": e2e,
            "gpu_launches": launches_per_step * n_steps, "clocks": clocks, "decode": dec,
            "verify": ver, "prologue": pro, "layer": lay, "configs": cfgs,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


PROFILE_CASES = ("ring_4k", "rows_4k", "conv_16k", "gate_16k")


def run_profile_case(name):
    """One small case of one kernel for an ncu capture (no timing, no JSON line):
    a warm-up launch and two more, on inputs of a few hundred MB at most.
      ring_4k  -- the tensor-core prefill on the 4096-token layer workload
      rows_4k  -- the one-decay-per-value-row prefill on the same workload
      conv_16k -- the short convolution (width 4, SiLU, carried state) over the
                  first 16K tokens' values of the 64K workload (134 MB in, 134 MB out)
      gate_16k -- the standalone output gate o <- o sigmoid(z) on 16K x 4096 outputs
    """
    import torch
    from linear_attention_recurrence_rule_b200 import gdn
    from linear_attention_recurrence_rule_b200.inputs import layer_extras, row_decays, workload_inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if name == "conv_16k":
        x = workload_inputs("long_prefill_64k", tokens=16384)["v"].reshape(1, 16384, -1).to(dev)
        ex = layer_extras(1, x.shape[-1], 4, (1,), torch.bfloat16, seed=305)
        w, b, cs = (ex[k].to(dev) for k in ("conv_weight", "conv_bias", "conv_state"))
        y = torch.empty_like(x)
        run = lambda: gdn.gdn_short_conv(x, w, b, cs, silu=True, y=y)   # noqa: E731
    elif name == "gate_16k":
        o = workload_inputs("long_prefill_64k", tokens=16384)["v"].to(dev)
        z = layer_extras(1, o.shape[2] * o.shape[3], 4, tuple(o.shape), torch.bfloat16, seed=306)["z"].to(dev)
        run = lambda: gdn.gdn_output_gate(o, z)   # noqa: E731
    else:
        z = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v)
             for k, v in workload_inputs("layer_prefill_4k").items()}
        g = row_decays(tuple(z["v"].shape), seed=903).to(dev) if name == "rows_4k" else z["g"]
        pro = gdn.ROW_DECAY if name == "rows_4k" else 0
        o = torch.empty_like(z["v"])
        run = lambda: gdn.gdn_chunk_prefill(z["q"], z["k"], z["v"], g, z["beta"], chunk=64, o=o,   # noqa: E731
                                            prologue=pro)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    print(f"profile case {name}: 3 launches done")
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-verify", action="store_true")
    ap.add_argument("--no-prologue", action="store_true")
    ap.add_argument("--no-layer", action="store_true")
    ap.add_argument("--no-configs", action="store_true")
    ap.add_argument("--verify-rounds", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="decode measurement only")
    ap.add_argument("--tokens", type=int, default=None,
                    help="truncate the prefill workload (profiling runs; not a bench line)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-step-seconds", type=float, default=4.0)
    ap.add_argument("--profile-case", choices=PROFILE_CASES, default=None,
                    help="run one small case of one kernel for an ncu capture and exit")
    args = ap.parse_args()
    if args.profile_case:
        return run_profile_case(args.profile_case)
    if args.warmup < 3:
        print("note: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    return run_b200(args)


if __name__ == "__main__":
    sys.exit(main())
