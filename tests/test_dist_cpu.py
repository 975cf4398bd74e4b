"""Multi-rank host logic of the benchmark's replica mode, on CPU with gloo
(world size 2): ranks draw different sequences of the same workload, the
timing reduction is a max over ranks, and the aggregate throughput counts the
units of every rank over the slowest rank's time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from linear_attention_recurrence_rule_b200.inputs import workload_inputs
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            init_method=f"tcp://127.0.0.1:{port}",
                            timeout=datetime.timedelta(seconds=60))
    try:
        x = workload_inputs("long_prefill_64k", tokens=256,
                            seed_offset=bench.replica_seed_offset(rank))
        sig = torch.tensor([float(x["v"].float().sum()), float(x["g"].sum())])
        sigs = [torch.zeros(2) for _ in range(world)]
        dist.all_gather(sigs, sig)
        local_ms = 10.0 + 5.0 * rank
        mx = bench.dist_max(local_ms)
        out[rank] = (sigs[0].tolist(), sigs[1].tolist(), mx,
                     bench.aggregate_throughput(world, 256, 4, mx))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_replicas():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(150)
        assert p.exitcode == 0, f"rank exited with {p.exitcode}"
    s0, s1, mx0, thr0 = out[0]
    _, _, mx1, thr1 = out[1]
    assert s0 != s1, "replicas must draw different sequences"
    assert mx0 == mx1 == 15.0, "timing must be the max over ranks"
    assert thr0 == thr1 == pytest.approx(2 * 256 * 4 / 0.015)


def test_single_process_helpers():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.dist_max(3.5) == 3.5
    assert bench.aggregate_throughput(1, 65536, 10, 1000.0) == pytest.approx(655360.0)
    assert bench.prefill_flops_per_token(16, 32, 128, 64) == 5242880
    assert bench.decode_bytes_per_step(256, 16, 32, 128, 128) == 1080098816
    # verify_256x4 with every draft kept: hand-counted bytes of one round
    acc = [4] * 256
    assert bench.verify_bytes(256, 4, 16, 32, 128, 128, acc, "deltas") == (579076096, 1094845440)
    assert bench.verify_bytes(256, 4, 16, 32, 128, 128, acc, "states") == (2709782528, 1073742848)
    # nothing kept: the commit touches no state
    assert bench.verify_bytes(256, 4, 16, 32, 128, 128, [0] * 256, "deltas")[1] == 1024
