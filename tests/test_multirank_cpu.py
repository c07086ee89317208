"""The multi-GPU bench path on CPU: two gloo ranks exercise the cross-rank timing
(max over ranks) and the rank-0-only reference arm, without a GPU."""
import os
import socket
import sys

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
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # Each rank reports its own step time; the job's time is the slowest rank's.
        got = bench.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))
        out[rank] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5


def test_reference_arm_is_rank0_only(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class A:
        workload, steps, warmup = "tiny", 1, 3
    bench.run_reference(A, rank=1, world=2)   # other ranks exit without work or output
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_one_json_line(capsys):
    import json
    sys.path.insert(0, ROOT)
    import bench

    class A:
        workload, steps, warmup = "tiny", 2, 3
    bench.run_reference(A, rank=0, world=1)
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["higher_is_better"] is True
