"""Multi-process host logic of the data-parallel run, on CPU with gloo.

The data-parallel path exchanges exactly one thing: the LoRA gradients dA and
dB are summed over ranks and divided by the world size (the frozen NF4 weight
is replicated, tokens are split). Timing is reported as the slowest rank's.
These checks run bench.py's helpers as two gloo ranks on 127.0.0.1.
"""

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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        ws, rk, local = bench.dist_env()
        assert (ws, rk, local) == (world, rank, rank)
        # slowest rank decides the step time
        t = bench.max_over_ranks(1.5 + rank * 2.25, world)
        # gradients: each rank holds its own dA, dB; afterwards all hold the mean
        g = torch.Generator().manual_seed(100 + rank)
        da = torch.randn(8, 64, generator=g, dtype=torch.float32)
        db = torch.randn(32, 8, generator=g, dtype=torch.float32)
        bench.allreduce_grads([da, db], world)
        out[rank] = (t, da.clone(), db.clone())
    finally:
        dist.destroy_process_group()


def test_two_rank_exchange_and_timing():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    expect_da = sum(torch.randn(8, 64, generator=torch.Generator().manual_seed(100 + r)) for r in range(world)) / world
    gens = [torch.Generator().manual_seed(100 + r) for r in range(world)]
    for gg in gens:
        torch.randn(8, 64, generator=gg)
    expect_db = sum(torch.randn(32, 8, generator=gg) for gg in gens) / world
    for r in range(world):
        t, da, db = res[r]
        assert t == pytest.approx(1.5 + (world - 1) * 2.25)
        torch.testing.assert_close(da, expect_da, rtol=1e-6, atol=1e-6)
        torch.testing.assert_close(db, expect_db, rtol=1e-6, atol=1e-6)
    # every rank ends with identical gradients (replicas stay in step)
    assert torch.equal(res[0][1], res[1][1]) and torch.equal(res[0][2], res[1][2])


def test_single_rank_helpers_are_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
    t = torch.ones(3)
    bench.allreduce_grads([t], 1)
    assert torch.equal(t, torch.ones(3))


def test_bench_launcher_starts_n_ranks(tmp_path):
    # bench.py --gpus N outside a launcher re-runs itself as N ranks under
    # torch.distributed.run; here the same launcher starts a small script
    # that joins a gloo group and reports its rank and the world size
    import json
    import subprocess
    import sys
    sys.path.insert(0, ROOT)
    import bench
    script = tmp_path / "rank_report.py"
    out = tmp_path / "ranks"
    out.mkdir()
    script.write_text(
        "import os, json, torch.distributed as dist\n"
        "from datetime import timedelta\n"
        "dist.init_process_group('gloo', timeout=timedelta(seconds=60))\n"
        "r, w = dist.get_rank(), dist.get_world_size()\n"
        "dist.barrier()\n"
        f"open(os.path.join({str(out)!r}, f'r{{r}}.json'), 'w').write(json.dumps(dict(rank=r, world=w, "
        "local=int(os.environ['LOCAL_RANK']))))\n"
        "dist.destroy_process_group()\n")
    cmd = bench.torchrun_command(2, str(script), [], bench.free_port())
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"] and "--nproc-per-node=2" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    rc = bench.spawn_ranks(2, str(script), [], timeout_s=240)
    assert rc == 0
    got = sorted((json.loads((out / f"r{i}.json").read_text()) for i in range(2)), key=lambda d: d["rank"])
    assert [(d["rank"], d["world"], d["local"]) for d in got] == [(0, 2, 0), (1, 2, 1)]
