"""The multi-GPU path of bench.py on CPU: independent replicas per rank (decode
shards by sequence, no data-path collective); the step time is the maximum
over ranks and the throughput counts the units of every rank."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local_ms = 1.0 + rank * 0.5           # rank 1 is slower
    ms = bench.reduce_max(local_ms, world, torch.device("cpu"))
    q.put((rank, ms, bench.job_throughput(world, 64, ms)))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in out:
        assert ms == 1.5                       # both ranks see the slowest rank's time
        assert value == pytest.approx(2 * 64 / 1.5e-3)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    class A:
        workload = "v2"; steps = 1; warmup = 0; gpus = 2
    assert bench.run_reference(A()) == 0


def test_single_rank_reduce_is_identity():
    import bench
    assert bench.reduce_max(3.25, 1, None) == 3.25
    assert bench.job_throughput(1, 64, 0.5) == pytest.approx(128000.0)


def test_reference_arm_line_keeps_the_contract(capsys, monkeypatch):
    """The reference arm's JSON line carries the contract's keys and the same
    config object as the CUDA arm (both come from bench.workload_config)."""
    import json
    import bench
    monkeypatch.setenv("RANK", "0")

    class A:
        workload = "tiny"; steps = 1; warmup = 0; gpus = 1; ctx = 0; batch = 0
    assert bench.run_reference(A()) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["higher_is_better"] is True
    assert line["config"] == bench.workload_config(A(), 1)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
