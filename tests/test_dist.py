"""Multi-rank host logic on CPU (gloo, world size 2): the (b, h) sharding
covers every pair once, and the timing takes the slowest rank."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from frame_wise_delta_b200 import dist as vdist


def test_shards_cover_every_pair_once():
    for B, H, world in [(1, 24, 2), (4, 24, 8), (3, 5, 4), (1, 1, 2)]:
        seen = []
        for r in range(world):
            seen += vdist.shard_pairs(B, H, r, world)
        assert sorted(seen) == [(b, h) for b in range(B) for h in range(H)]
        sizes = [len(vdist.shard_pairs(B, H, r, world)) for r in range(world)]
        assert max(sizes) - min(sizes) <= 1


def test_head_ranges_are_contiguous_slices():
    runs = vdist.head_ranges(4, 24, 3, 8)
    pairs = [(b, h) for b, h0, h1 in runs for h in range(h0, h1)]
    assert pairs == vdist.shard_pairs(4, 24, 3, 8)
    with pytest.raises(ValueError):
        vdist.shard_pairs(1, 2, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = vdist.max_over_ranks(1.0 + 2.0 * rank)  # rank 1 is the slower one
        mine = vdist.shard_pairs(1, 24, rank, world)
        out.put((rank, t, len(mine), mine[0]))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [3.0, 3.0]
    assert [r[2] for r in res] == [12, 12]
    assert res[0][3] == (0, 0) and res[1][3] == (0, 12)
    assert vdist.throughput(102, 2, 0.5) == 408.0


def _shard_worker(rank, world, port, out):
    """One rank of a head-sharded problem: its inputs (drawn for its own pairs
    only, as bench.py --shard heads does) through the oracle."""
    import dataclasses

    import numpy as np
    import torch.distributed as dist

    import oracle
    from frame_wise_delta_b200 import synth

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = dataclasses.replace(synth.WORKLOADS["tiny"], B=2, H=3, T=12)
        pairs = vdist.shard_pairs(w.B, w.H, rank, world)
        mine = synth.generate_pairs(w, pairs)
        res = {"O": [], "F": [], "G": []}
        for i in range(len(pairs)):
            r = oracle.vda_head({k: v[0, i] for k, v in mine.items()}, w.chunk, w.anchors)
            for k in res:
                res[k].append(r[k])
        out.put((rank, vdist.pair_range(w.B, w.H, rank, world), {k: np.stack(v) for k, v in res.items()}))
    finally:
        dist.destroy_process_group()


def test_head_shards_reassemble_the_whole_problem_gloo_world2():
    """Two ranks each run their share of one problem's (b, h) pairs (no data
    exchange); their outputs, put side by side in rank order, are the whole
    problem's outputs exactly."""
    import dataclasses

    import numpy as np

    import oracle
    from frame_wise_delta_b200 import synth

    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((out.get(timeout=300) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [(0, 3), (3, 6)]
    w = dataclasses.replace(synth.WORKLOADS["tiny"], B=2, H=3, T=12)
    full = synth.generate_all(w)
    for k in ("O", "F", "G"):
        got = np.concatenate([r[2][k] for r in res]).reshape((w.B, w.H) + res[0][2][k].shape[1:])
        for b in range(w.B):
            for h in range(w.H):
                want = oracle.vda_head({n: v[b, h] for n, v in full.items()}, w.chunk, w.anchors)[k]
                np.testing.assert_array_equal(got[b, h], want)


def test_shard_view_is_the_ranks_pairs():
    import numpy as np

    x = np.arange(4 * 24 * 3).reshape(4, 24, 3)
    for world in (1, 2, 3, 8):
        parts = [vdist.shard_view(x, 4, 24, r, world) for r in range(world)]
        assert np.array_equal(np.concatenate(parts, axis=1).reshape(x.shape), x)
        for r, p in enumerate(parts):
            want = np.stack([x[b, h] for b, h in vdist.shard_pairs(4, 24, r, world)])
            assert np.array_equal(p[0], want)
