"""Host-side helpers for running the layer on several GPUs of one node.

H-BitLinear acts on each token row independently (norm, transform and
quantisation are per row; output row m depends only on its own codes), so the
layer shards by token rows with no collective on the data path: each rank
holds the packed weights and processes its own rows.  Only timing uses a
collective (a max over ranks of the measured time).
"""
import os


def env_rank():
    """(rank, local_rank, world_size) from the torchrun environment (defaults: one process)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def shard_rows(M, world, rank):
    """Contiguous, balanced [start, stop) row range of `rank` among `world` ranks."""
    if world < 1 or not (0 <= rank < world) or M < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(M, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value, device=None):
    """Max of a float over all ranks of the default process group (value itself if none)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value, device=None):
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def gather_rows(Y_local, M, group=None):
    """All-gather of row shards (the shard_rows split of M rows) into one [M, N]
    tensor on every rank: the optional step for a caller that wants the whole
    output on each device.  The layer itself needs no collective.  Shards may
    differ by one row, so each is padded to the largest before the all-gather
    (NCCL on GPUs, gloo on CPU) and the padding is dropped afterwards."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return Y_local
    world = dist.get_world_size(group)
    spans = [shard_rows(M, world, r) for r in range(world)]
    rows = max(b - a for a, b in spans)
    pad = torch.zeros((rows,) + tuple(Y_local.shape[1:]), dtype=Y_local.dtype,
                      device=Y_local.device)
    pad[: Y_local.shape[0]] = Y_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([parts[r][: b - a] for r, (a, b) in enumerate(spans)])
