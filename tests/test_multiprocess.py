"""The multi-rank host logic on CPU with the gloo backend (world size 2): column shards
of a GEMM gather back to the full product, and timings reduce to the maximum."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from error_compensated_gemm_b200.shard import max_over_ranks, shard_range


def test_shard_range_covers_and_aligns():
    for n in (1, 7, 128, 14336, 14337):
        for world in (1, 2, 3, 8):
            ranges = [shard_range(n, world, r, align=128) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == n
            for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
                assert a1 == b0 and a0 % 128 == 0
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 128


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import synthetic
        from oracle import gemm as G
        X, W = synthetic.gemm_prefill(M=64, K=256, N=1000)
        n0, n1 = shard_range(1000, world, rank, align=128)
        part = torch.from_numpy(G.gemm_ref(X.numpy(), W.numpy()[:, n0:n1]))
        pad = torch.zeros(64, 512, dtype=torch.float64)
        pad[:, : n1 - n0] = part
        parts = [torch.zeros_like(pad) for _ in range(world)]
        dist.all_gather(parts, pad)
        widths = [shard_range(1000, world, r, align=128) for r in range(world)]
        full = torch.cat([p[:, : b - a] for p, (a, b) in zip(parts, widths)], dim=1)
        mx = max_over_ranks([1.0 + rank, 10.0 - rank])
        if rank == 0:
            ref = torch.from_numpy(G.gemm_ref(X.numpy(), W.numpy()))
            out_q.put((bool(torch.equal(full, ref)), mx))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_sharded_gemm_and_timing_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    equal, mx = q.get(timeout=10)
    assert equal
    assert mx == [2.0, 10.0]
