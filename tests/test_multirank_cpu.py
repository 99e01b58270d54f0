"""Data-parallel (token-sharded) path on two gloo ranks, CPU only.

Each rank runs the oracle on its row shard of the same workload with the replicated weight;
gathering the shards must reproduce the unsharded layer exactly (rows are independent), and the
job timing must take the slowest rank.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from rotation_w4a4_quantized_b200.dp import job_throughput, shard_rows, slowest_rank_ms


def test_shard_rows_tiles_the_batch():
    for M in (0, 1, 7, 64, 4608, 4609):
        for world in (1, 2, 3, 8):
            ranges = [shard_rows(M, r, world) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == M
            for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
                assert a1 == b0
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_rows(10, 2, 2)


def test_job_throughput():
    assert job_throughput(1e12, 4, 2.0) == pytest.approx(2e15)
    with pytest.raises(ValueError):
        job_throughput(1.0, 1, 0.0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    from oracle import convrot_oracle as O
    from synthetic import CONFIGS, make_inputs

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        w = CONFIGS["tiny"]
        X, W, bias = make_inputs(w, with_bias=True)
        a, b = shard_rows(w.M, rank, world)
        X64 = X.float().numpy().astype(np.float64)
        res = O.w4a4_linear(X64[a:b], W.float().numpy().astype(np.float64), w.group,
                            bias=bias.float().numpy().astype(np.float64))
        y = torch.from_numpy(res["y"])
        sizes = [shard_rows(w.M, r, world) for r in range(world)]
        parts = [torch.zeros(s1 - s0, w.N, dtype=torch.float64) for s0, s1 in sizes]
        dist.all_gather(parts, y)
        # each rank reports its own time; the job time is the slowest one
        slow = slowest_rank_ms(1.0 + rank)
        if rank == 0:
            out.put((torch.cat(parts).numpy(), slow))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _strong_worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    from oracle import convrot_oracle as O
    from rotation_w4a4_quantized_b200.dp import run_sharded
    from synthetic import CONFIGS, make_inputs

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        w = CONFIGS["tiny"]
        X, W, bias = make_inputs(w, with_bias=True)
        X = X[:61]                                  # a batch that does not split evenly
        W64 = W.float().numpy().astype(np.float64)
        b64 = bias.float().numpy().astype(np.float64)
        seen = []

        def layer(x_local):
            # the CPU stand-in for the device layer: the oracle on this rank's rows
            seen.append(x_local.shape[0])
            res = O.w4a4_linear(x_local.float().numpy().astype(np.float64), W64, w.group,
                                bias=b64)
            return torch.from_numpy(res["y"])

        y = run_sharded(X, layer, rank, world)
        out.put((rank, seen[0], y.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_strong_split_and_gather():
    """run_sharded (the split-and-gather bench.py's strong-scaling mode calls): each rank's
    layer sees only its rows, and every rank ends with the unsharded output."""
    from oracle import convrot_oracle as O
    from synthetic import CONFIGS, make_inputs

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_strong_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict((r, (n, y)) for r, n, y in (q.get(timeout=120) for _ in range(2)))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    w = CONFIGS["tiny"]
    X, W, bias = make_inputs(w, with_bias=True)
    ref = O.w4a4_linear(X[:61].float().numpy().astype(np.float64),
                        W.float().numpy().astype(np.float64), w.group,
                        bias=bias.float().numpy().astype(np.float64))["y"]
    assert [got[r][0] for r in (0, 1)] == [31, 30]
    for r in (0, 1):
        assert np.array_equal(got[r][1], ref)


def test_two_rank_token_sharding_matches_unsharded():
    from oracle import convrot_oracle as O
    from synthetic import CONFIGS, make_inputs

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    y_sharded, slow = q.get(timeout=120)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    w = CONFIGS["tiny"]
    X, W, bias = make_inputs(w, with_bias=True)
    ref = O.w4a4_linear(X.float().numpy().astype(np.float64), W.float().numpy().astype(np.float64),
                        w.group, bias=bias.float().numpy().astype(np.float64))
    assert np.array_equal(y_sharded, ref["y"])
    assert slow == 2.0
