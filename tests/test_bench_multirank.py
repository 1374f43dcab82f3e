"""Host logic of the multi-GPU bench on CPU: two gloo ranks, each with its own
time and its own requests; the reported time is the slowest rank's and the
rate counts every rank's items (weak scaling, no collective on the data path)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    from quantized_recurrent_state_sm_b200 import workload as W
    my_ms = [7.0, 11.0][rank]
    ms = bench.max_over_ranks(my_ms, world, "cpu")
    rate = bench.whole_job_rate(world, 24576, 10, ms)
    cfg = W.with_overrides(W.CONFIGS[3], batch=2)
    x = W.step_inputs(cfg, 0 + bench.rank_step_offset(rank))
    q.put((rank, ms, rate, float(x["k"][0, 0, 0])))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, rate0, k0), (r1, ms1, rate1, k1) = res
    assert ms0 == ms1 == 11.0
    assert rate0 == rate1 == pytest.approx(2 * 24576 * 10 / 11e-3)
    assert k0 != k1  # each rank serves different requests


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.whole_job_rate(1, 100, 10, 1.0) == pytest.approx(1e6)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    """Under torchrun the reference arm (the oracle on the host cores) runs
    and prints on rank 0 alone; every other rank exits 0 without work."""
    import types

    import bench
    from quantized_recurrent_state_sm_b200 import workload as W
    monkeypatch.setenv("RANK", "1")
    called = []
    monkeypatch.setattr(bench, "cpu_oracle_rate", lambda *a, **k: called.append(a) or (1.0, {}))
    args = types.SimpleNamespace(steps=3, warmup=3, gpus=2, cpu_seconds=1.0)
    assert bench.run_reference(args, W.CONFIGS[3]) == 0
    assert not called and capsys.readouterr().out == ""
