"""Host-side helpers for running the hot path on several GPUs, one process per GPU.

The path has no exchange step: GEMM output columns (or rows) and attention's (batch,
KV head) pairs are independent, so each rank takes a contiguous shard and no collective
touches the data.  torch.distributed is used only to line the ranks up and to take the
maximum of their device timings.
"""
import torch


def shard_range(n, world, rank, align=1):
    """Contiguous [start, end) of n items for `rank` of `world`; boundaries are multiples of
    `align` (except the end of the last shard), and shard sizes differ by at most `align`."""
    if world < 1 or not (0 <= rank < world) or align < 1:
        raise ValueError("bad world/rank/align")
    units = (n + align - 1) // align
    u0 = units * rank // world
    u1 = units * (rank + 1) // world
    return min(n, u0 * align), min(n, u1 * align)


def max_over_ranks(values, device=None):
    """Element-wise maximum of a list of floats over all ranks (identity without a process
    group)."""
    import torch.distributed as dist
    vals = [float(v) for v in values]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]
