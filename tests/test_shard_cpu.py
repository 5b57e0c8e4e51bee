"""Splitting a prefill's independent chains across ranks (gated_retention_linear_b200.shard), on
the CPU: the partitions cover every head and every packed sequence exactly once, and two gloo
ranks that each run the oracle on their own sequences and heads reassemble the full result."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from gated_retention_linear_b200 import shard  # noqa: E402


@pytest.mark.parametrize("H,world", [(24, 1), (24, 2), (24, 5), (3, 8), (0, 2), (7, 7)])
def test_head_ranges_cover_each_head_once(H, world):
    seen = []
    for r in range(world):
        h0, h1 = shard.head_range(H, r, world)
        assert 0 <= h0 <= h1 <= H
        seen.extend(range(h0, h1))
    assert seen == list(range(H))
    sizes = [shard.head_range(H, r, world)[1] - shard.head_range(H, r, world)[0]
             for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def test_head_range_rejects_bad_ranks():
    with pytest.raises(ValueError):
        shard.head_range(4, 2, 2)


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_sequence_assignment_is_a_balanced_partition(world):
    rng = np.random.default_rng(7)
    lengths = [int(x) for x in rng.integers(1, 65536, size=13)]
    parts = shard.sequence_assignment(lengths, world)
    assert len(parts) == world
    flat = sorted(i for p in parts for i in p)
    assert flat == list(range(len(lengths)))
    assert all(p == sorted(p) for p in parts)
    loads = [sum(lengths[i] for i in p) for p in parts]
    # longest-first greedy: no rank exceeds another by more than one sequence
    assert max(loads) - min(loads) <= max(lengths)


def test_packed_subset_rows_and_offsets():
    cu = [0, 5, 5, 12, 20]
    rows, sub = shard.packed_subset(cu, [3, 0, 1])
    assert rows == [(12, 20), (0, 5), (5, 5)]
    assert sub == [0, 8, 13, 13]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


LENGTHS = [37, 5, 60, 12, 1]
H, D = 3, 8


def _inputs():
    g = torch.Generator().manual_seed(11)
    T = sum(LENGTHS)
    q = torch.randn(T, H, D, generator=g, dtype=torch.float64) / D ** 0.5
    k = torch.randn(T, H, D, generator=g, dtype=torch.float64) / D ** 0.5
    v = torch.randn(T, H, D, generator=g, dtype=torch.float64)
    gl = torch.randn(T, H, generator=g, dtype=torch.float64) + 2.0
    return q.numpy(), k.numpy(), v.numpy(), gl.numpy()


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    from oracle import oracle
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, gl = _inputs()
        cu = [0]
        for n in LENGTHS:
            cu.append(cu[-1] + n)
        # this rank's sequences (all heads) ...
        mine = shard.sequence_assignment(LENGTHS, world)[rank]
        rows, sub = shard.packed_subset(cu, mine)
        take = np.concatenate([np.arange(a, b) for a, b in rows]) if rows else np.zeros(0, int)
        o_seq, s_seq = oracle.gret_recurrent(q[take], k[take], v[take], gl[take], cu_seqlens=sub)
        # ... and this rank's heads (all sequences)
        h0, h1 = shard.head_range(H, rank, world)
        o_head, s_head = oracle.gret_recurrent(q[:, h0:h1], k[:, h0:h1], v[:, h0:h1],
                                               gl[:, h0:h1], cu_seqlens=cu)
        parts = [None] * world
        dist.all_gather_object(parts, (mine, rows, o_seq, s_seq, (h0, h1), o_head, s_head))
        if rank == 0:
            o_full, s_full = oracle.gret_recurrent(q, k, v, gl, cu_seqlens=cu)
            o_a, s_a = np.zeros_like(o_full), np.zeros_like(s_full)
            o_b, s_b = np.zeros_like(o_full), np.zeros_like(s_full)
            for seqs, rws, o_s, s_s, (a0, a1), o_h, s_h in parts:
                t = 0
                for i, (a, b) in zip(seqs, rws):
                    o_a[a:b] = o_s[t:t + b - a]
                    s_a[i] = s_s[seqs.index(i)]
                    t += b - a
                o_b[:, a0:a1] = o_h
                s_b[:, a0:a1] = s_h
            out["seq"] = bool(np.array_equal(o_a, o_full) and np.array_equal(s_a, s_full))
            out["head"] = bool(np.array_equal(o_b, o_full) and np.array_equal(s_b, s_full))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_reassemble_the_full_prefill():
    if not os.path.exists(os.path.join(ROOT, "oracle", "libgret_oracle.so")):
        pytest.skip("oracle library not built")
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res == {"seq": True, "head": True}
