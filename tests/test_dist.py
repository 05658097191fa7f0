"""Multi-rank plumbing on CPU (gloo, world size 2): shard assignment and max-over-ranks timing."""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_deltanet_linear_17_b200 import dist as gdist


def test_shard_sequences_partition():
    import random
    r = random.Random(0)
    for _ in range(200):
        lens = [r.randint(0, 500) for _ in range(r.randint(1, 40))]
        for world in (1, 2, 3, 4, 8):
            parts = [gdist.shard_sequences(lens, world, k) for k in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == len(lens)
            for a, b in zip(parts, parts[1:]):
                assert a[1] == b[0]
            tot = sum(lens)
            if world == 2 and tot > 0 and max(lens) < tot / 4:
                t0 = sum(lens[parts[0][0]:parts[0][1]])
                assert abs(t0 - tot / 2) <= max(lens)


def test_shard_heads_partition():
    for Nqk, Nv in ((16, 32), (4, 8), (2, 4), (3, 9)):
        for world in (1, 2, 4):
            if world > Nqk:
                continue
            got = [gdist.shard_heads(Nqk, Nv, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == Nqk and got[-1][3] == Nv
            for a, b in zip(got, got[1:]):
                assert a[1] == b[0] and a[3] == b[2]
            G = Nv // Nqk
            for a, b, va, vb in got:
                assert va == a * G and vb == b * G


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    try:
        r, local, w = gdist.init(backend="gloo", timeout_s=60)
        assert (r, w) == (rank, world)
        gdist.barrier()
        step_ms = 1.0 + rank          # each rank's own step time
        mx = gdist.max_over_ranks(step_ms)
        total = gdist.sum_over_ranks(100.0)
        lens = [10, 300, 5, 77, 129, 64]
        shard = gdist.shard_sequences(lens, w, r)
        q.put((rank, mx, total, shard))
        dist.destroy_process_group()
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put((rank, "error", repr(e), None))


def test_gloo_world_size_two():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
    res.sort()
    assert all(r[1] != "error" for r in res), res
    assert [r[1] for r in res] == [2.0, 2.0]          # max over ranks seen by both
    assert [r[2] for r in res] == [200.0, 200.0]
    shards = [r[3] for r in res]
    assert shards[0][0] == 0 and shards[0][1] == shards[1][0] and shards[1][1] == 6
