"""The benchmark's multi-rank host logic, run as two gloo ranks on the CPU.

With N GPUs every rank prefills its own sequence (weak scaling, no collective on the data path);
the host logic is the barrier around the timed region, the max of the device times over ranks,
per-rank seeds that give every rank different data, and the reference arm running on rank 0
alone.
"""
import contextlib
import io
import os
import socket
import sys

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
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    import bench
    import synth_inputs as SI
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        res = {}
        bench.barrier(world)
        res["max"] = bench.max_over_ranks(1.5 + rank, world)
        x = SI.gret_inputs(1, 8, 2, 16, seed=bench.rank_seed(2, rank))["q"]
        gathered = [torch.empty_like(x) for _ in range(world)]
        dist.all_gather(gathered, x)
        res["distinct"] = all(not torch.equal(gathered[i], gathered[j])
                              for i in range(world) for j in range(i + 1, world))
        # reference arm: only rank 0 runs and prints
        args = type("A", (), dict(cpu_tokens=16, steps=1, warmup=0))()
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.run_reference(args)
        res["ref_lines"] = len([ln for ln in buf.getvalue().splitlines() if ln.strip()])
        bench.barrier(world)
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_two_rank_host_logic():
    pytest.importorskip("numpy")
    oracle_lib = os.path.join(ROOT, "oracle", "libgret_oracle.so")
    if not os.path.exists(oracle_lib):
        pytest.skip("oracle library not built")
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert set(res) == {0, 1}
    for r in range(world):
        assert res[r]["max"] == pytest.approx(2.5)
        assert res[r]["distinct"]
    assert res[0]["ref_lines"] == 1
    assert res[1]["ref_lines"] == 0
