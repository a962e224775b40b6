"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

The path does not shard: under torchrun every rank runs an independent replica and
the job's figure is the bytes of all ranks over the slowest rank's time. The reference
arm (the CPU oracle) runs on rank 0 alone; other ranks exit without work.
"""
import datetime
import os
import socket

import pytest

torch = pytest.importorskip("torch")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _aggregate_worker(rank, world, port, out_dir):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench

    b, t = bench.aggregate(local_bytes=(rank + 1) * 1e9, local_ms=10.0 * (rank + 1), world=world)
    with open(os.path.join(out_dir, f"rank{rank}"), "w") as f:
        f.write(f"{b!r} {t!r}")
    dist.barrier()
    dist.destroy_process_group()


def test_aggregate_sums_bytes_and_takes_the_slowest_rank_over_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp

    mp.start_processes(_aggregate_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    for r in range(2):
        b, t = (float(v) for v in (tmp_path / f"rank{r}").read_text().split())
        assert b == 3e9  # 1 GB + 2 GB
        assert t == 20.0  # max(10 ms, 20 ms)


def test_single_rank_aggregate_is_the_local_figure():
    import bench

    assert bench.aggregate(5e8, 3.5, 1) == (5e8, 3.5)


def test_reference_arm_does_no_work_on_other_ranks(monkeypatch, capsys):
    import argparse

    import bench
    import synth

    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(steps=1, warmup=0, gpus=2, cpu_seconds=1.0)
    assert bench.run_reference(args, synth.WORKLOADS[1]) is None
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_one_contract_line_on_rank_0(monkeypatch, capsys):
    """The reference arm times the CPU oracle on a bounded sample and prints the same
    metric, unit and config as the GPU arm, with its own cpu_baseline and a zero-copy e2e."""
    import argparse
    import json

    import bench
    import synth

    monkeypatch.setenv("RANK", "0")
    wl = synth.WORKLOADS[0]
    bench.run_reference(argparse.Namespace(steps=2, warmup=1, gpus=1), wl)
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["higher_is_better"] is True and d["vs_baseline"] is None and d["dtype"] == "f64"
    assert d["config"]["workload"] == wl.name
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
