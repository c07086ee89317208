"""The multi-GPU paths on CPU, without a GPU: two gloo ranks exercise the cross-rank
timing (max over ranks), the rank-0-only reference arm, and the token split of the
layer with its one exchange step (the value-gradient reduce-scatter of
product_key_memory_b200.sharding), each rank computing its share with the fp64
oracle. Unmeasured on hardware: every run here has one GPU."""
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


def _split_worker(rank, world, port, B, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import numpy as np
    import oracle
    import synth
    from product_key_memory_b200 import sharding
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.WORKLOADS["tiny"].with_(B=B)
        L = synth.make_layer(w)
        gout = synth.make_grad_out(w)
        a, b = sharding.token_range(B, world, rank)
        part = dict(L)
        part["x"] = L["x"][a:b]
        r = oracle.forward(part, w.H, w.dq, w.n, w.k)
        # Forward: no exchange; gather the ranks' rows (padded to one length) to check.
        most = -(-B // world)
        pad = np.zeros((most, w.v))
        pad[: b - a] = r["out"]
        got = [torch.empty(most, w.v, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(got, torch.from_numpy(pad))
        lens = [sharding.token_range(B, world, q)[1] - sharding.token_range(B, world, q)[0]
                for q in range(world)]
        out_all = torch.cat([g[:n] for g, n in zip(got, lens)]).numpy()
        # Value backward: each rank's partial table over all slots, then the
        # reduce-scatter leaves each rank the summed block of rows it owns.
        gv, gs = oracle.backward(L["values"], gout[a:b], r["indices"], r["weights"])
        block = sharding.reduce_value_grads(torch.from_numpy(gv))
        out[rank] = dict(out=out_all, block=block.numpy(), rows=sharding.row_block(
            w.n * w.n, world, rank), idx=r["indices"], gs=gs, span=(a, b))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("B", [64, 63])
def test_token_split_over_two_gloo_ranks_matches_one_rank(B):
    """Two ranks each take half of the tiny batch (63: ragged halves): outputs
    concatenated and value gradients summed equal the single-rank oracle."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_split_worker, args=(world, _free_port(), B, out), nprocs=world, join=True)
    w = synth.WORKLOADS["tiny"].with_(B=B)
    L = synth.make_layer(w)
    gout = synth.make_grad_out(w)
    full = oracle.forward(L, w.H, w.dq, w.n, w.k)
    gv, gs = oracle.backward(L["values"], gout, full["indices"], full["weights"])
    for rank in range(world):
        got = out[rank]
        # Forward rows depend only on their own token: equal bit for bit.
        np.testing.assert_array_equal(got["out"], full["out"])
        a, b = got["span"]
        np.testing.assert_array_equal(got["idx"], full["indices"][a:b])
        np.testing.assert_array_equal(got["gs"], gs[a:b])
        # Summed over ranks in another order than the one-rank sum: fp64 rounding only.
        r0, r1 = got["rows"]
        np.testing.assert_allclose(got["block"], gv[r0:r1], rtol=1e-12, atol=1e-15)
    assert out[0]["span"][1] == out[1]["span"][0] and out[1]["span"][1] == B


def test_token_range_and_row_block_cover_everything():
    sys.path.insert(0, ROOT)
    from product_key_memory_b200 import sharding
    for B in (0, 1, 7, 4096, 16385):
        for world in (1, 2, 3, 8):
            spans = [sharding.token_range(B, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == B
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    assert sharding.row_block(1 << 20, 8, 3) == (3 << 17, 4 << 17)
    with pytest.raises(ValueError):
        sharding.row_block(10, 3, 0)


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
