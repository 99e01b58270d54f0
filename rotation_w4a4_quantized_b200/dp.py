"""Host-side helpers for running the ConvLinear4bit path data-parallel over tokens.

Tokens (rows of X) are independent through every step of the path: the group-wise rotation
runs along K, the absmax and scale are per token, and each output row of the GEMM depends on
one activation row ("ConvRot: Rotation-Based Plug-and-Play 4-bit Quantization for Diffusion
Transformers", Fig. 3). A batch therefore shards over ranks by rows with a replicated weight
and no collective on the data path; the only communication is for timing and for gathering
results a caller wants in one place.
"""

from __future__ import annotations

from typing import Tuple


def shard_rows(M: int, rank: int, world: int) -> Tuple[int, int]:
    """Half-open row range [start, stop) of `rank` when M rows split over `world` ranks.

    The first M % world ranks get one extra row, so sizes differ by at most one and the
    ranges tile [0, M) in rank order.
    """
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} for world {world}")
    if M < 0:
        raise ValueError("M must be non-negative")
    base, extra = divmod(M, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start, stop


def local_rows(X, rank: int, world: int):
    """This rank's rows of a batch (a view: no copy), as shard_rows assigns them."""
    start, stop = shard_rows(X.shape[0], rank, world)
    return X[start:stop]


def gather_rows(y_local, M: int, rank: int, world: int, group=None):
    """All ranks' output rows in global order (every rank receives the whole [M, ...] result).

    Shards differ by at most one row; each is padded to the largest before the all-gather
    (collectives move equal-sized buffers) and trimmed after it."""
    import torch
    import torch.distributed as dist

    if world == 1:
        return y_local
    start, stop = shard_rows(M, rank, world)
    if y_local.shape[0] != stop - start:
        raise ValueError(f"rank {rank} holds {y_local.shape[0]} rows, expected {stop - start}")
    rows = -(-M // world)
    pad = torch.zeros((rows,) + tuple(y_local.shape[1:]), dtype=y_local.dtype,
                      device=y_local.device)
    pad[: y_local.shape[0]] = y_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([parts[r][: b - a] for r, (a, b) in
                      enumerate(shard_rows(M, r, world) for r in range(world))])


def run_sharded(X, layer, rank: int, world: int, gather: bool = True, group=None):
    """One global batch split over the ranks by rows: `layer` runs on this rank's rows (no
    communication on the data path); with `gather`, the outputs are all-gathered in row order."""
    y = layer(local_rows(X, rank, world))
    return gather_rows(y, X.shape[0], rank, world, group) if gather else y


def slowest_rank_ms(local_ms: float, group=None) -> float:
    """Max over ranks of a per-rank device time (ms); the job is as fast as its slowest rank."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return float(local_ms)
    backend = dist.get_backend(group)
    device = "cuda" if backend == "nccl" else "cpu"
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def job_throughput(ops_per_rank: float, world: int, slowest_ms: float) -> float:
    """Whole-job rate in ops/s: every rank's work divided by the slowest rank's time."""
    if slowest_ms <= 0:
        raise ValueError("time must be positive")
    return ops_per_rank * world / (slowest_ms * 1e-3)
