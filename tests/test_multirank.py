"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The path shards with no exchange (every rank runs its own batch against a
replicated packed weight), so the only cross-rank steps are the barrier and
the max-over-ranks reduction of the device times; these tests run them on
two gloo processes.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench

    # per-rank step times: rank 1 is the slow one for the first value
    mine = [1.0 + rank, 5.0 - rank, 0.25 * (rank + 1)]
    got = bench.reduce_max(mine, world, torch.device("cpu"))
    dist.barrier()
    out[rank] = got + [bench.job_throughput(world, 4096, got[0])]
    dist.destroy_process_group()


def test_timing_is_the_max_over_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        assert res[r][:3] == [2.0, 5.0, 0.5]
        # whole-job throughput: 2 ranks x 4096 tokens in the slowest rank's 2 ms
        assert res[r][3] == pytest.approx(2 * 4096 / 2e-3)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.reduce_max([3.0, 1.5], 1, torch.device("cpu")) == [3.0, 1.5]
    assert bench.job_throughput(1, 4096, 0.5) == pytest.approx(4096 / 0.5e-3)


def test_reference_arm_does_no_work_off_rank_zero(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setenv("RANK", "1")

    class A:
        workload = "flux_qkv_w4a4"
        steps = 1
        warmup = 0
        gpus = 2

    bench.run_reference(A())
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_one_contract_line(monkeypatch, capsys):
    """Rank 0 of the reference arm (the oracle on the host cores) prints one
    JSON line with the keys the bench contract asks of it."""
    sys.path.insert(0, ROOT)
    import json

    import bench

    monkeypatch.setenv("RANK", "0")

    class A:
        workload = "tiny_w4a4"
        steps = 1
        warmup = 0
        gpus = 1

    bench.run_reference(A())
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["metric"] == bench.METRIC and j["unit"] == "tokens/s"
    assert j["value"] > 0 and j["higher_is_better"] is True and j["n_gpus"] == 1
    assert j["config"]["workload"] == "tiny_w4a4"
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["cores"] >= 1
    assert j["cpu_baseline"]["value"] == j["value"]
    assert j["e2e"] == {"value": j["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
