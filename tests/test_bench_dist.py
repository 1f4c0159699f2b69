"""bench.py's multi-rank plumbing on CPU: two gloo ranks, as torchrun would start them.

The bench runs one process per GPU and reports whole-job throughput as the
units all ranks processed divided by the slowest rank's time. These tests run
its helpers (process-group set-up, barrier, max and sum over ranks, the JSON
line) in two spawned CPU processes with the gloo backend, and check the
reference arm's rule that ranks other than 0 exit without work.
"""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    ws, r = bench.init_dist("gloo")
    assert (ws, r) == (world, rank)
    bench.barrier()
    # rank r took (r + 1) seconds and moved (r + 1) GB
    t_max = bench.max_over_ranks(float(rank + 1))
    gb_sum = bench.sum_over_ranks(float(rank + 1) * 1e9)
    line = bench.assemble_line(n_gpus=world, steps=4, warmup=3, total_bytes_all_ranks=gb_sum, max_time_s=t_max,
                               workload={"workload": "unit"}, extra={"extra_key": rank})
    bench.barrier()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"t_max": t_max, "gb_sum": gb_sum, "line": line}, f)
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_and_report(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        assert r["t_max"] == 2.0                 # the slowest rank's time
        assert r["gb_sum"] == 3e9                # units of all ranks
        line = r["line"]
        assert line["value"] == pytest.approx(1.5)  # 3 GB / 2 s, whole job
        assert line["n_gpus"] == 2 and line["steps"] == 4 and line["warmup"] == 3
        assert line["scaling"] == "weak"
        assert line["ms_per_step"] == pytest.approx(500.0)
        assert line["higher_is_better"] is True


def test_reference_arm_non_zero_rank_exits_without_work(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")

    class Args:  # never read on rank 1
        pass

    assert bench.run_reference(Args()) == 0


def test_single_process_helpers_are_identities(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    assert bench.dist_env()[0] == 1
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.sum_over_ranks(7.0) == 7.0
