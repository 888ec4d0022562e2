"""Multi-GPU plumbing for the frame-wise delta-rule memory.

Every (batch, head) pair of VDA is independent (text state, frame statistics,
factor, composition, scans and readout), so the path shards over GPUs with no
collective on the data path: each rank owns a contiguous share of one
problem's (b, h) pairs (strong scaling: `bench.py --shard heads`) or a whole
problem of its own (weak scaling). torch.distributed is
used only to line ranks up and to take the slowest rank's time.
"""
from __future__ import annotations


def shard_pairs(B: int, H: int, rank: int, world: int) -> list[tuple[int, int]]:
    """Contiguous, balanced share of the B*H (b, h) pairs for `rank`."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} not in a world of {world}")
    n = B * H
    lo = n * rank // world
    hi = n * (rank + 1) // world
    return [(i // H, i % H) for i in range(lo, hi)]


def head_ranges(B: int, H: int, rank: int, world: int) -> list[tuple[int, int, int]]:
    """The rank's pairs as (b, h_begin, h_end) runs, i.e. contiguous slices of
    [B, H, ...] tensors that can be handed to the library as they are."""
    runs: list[tuple[int, int, int]] = []
    for b, h in shard_pairs(B, H, rank, world):
        if runs and runs[-1][0] == b and runs[-1][2] == h:
            runs[-1] = (b, runs[-1][1], h + 1)
        else:
            runs.append((b, h, h + 1))
    return runs


def pair_range(B: int, H: int, rank: int, world: int) -> tuple[int, int]:
    """The rank's share of the B*H pairs as a half-open range [lo, hi) of the
    flattened (b * H + h) index (the pairs of shard_pairs)."""
    pairs = shard_pairs(B, H, rank, world)
    if not pairs:
        return (0, 0)
    return (pairs[0][0] * H + pairs[0][1], pairs[-1][0] * H + pairs[-1][1] + 1)


def shard_view(x, B: int, H: int, rank: int, world: int):
    """The rank's pairs of a [B, H, ...] array or tensor as a [1, n, ...] view:
    a contiguous range of the flattened pairs, which the library takes as one
    batch of n heads (every pair is independent)."""
    lo, hi = pair_range(B, H, rank, world)
    return x.reshape((1, B * H) + tuple(x.shape[2:]))[:, lo:hi]


def max_over_ranks(x: float) -> float:
    """Largest value of x over all ranks (x itself without a process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(units_per_rank: float, world: int, seconds_slowest: float) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return units_per_rank * world / seconds_slowest
