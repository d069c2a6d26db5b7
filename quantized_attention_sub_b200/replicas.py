"""Rank plumbing of the multi-GPU run: one process per GPU, each an
independent replica over its own (b, h) slices.  The quantized attention
forward has no exchange step between slices, so nothing crosses ranks on
the data path; ranks meet only to start and stop the clock together and to
report the slowest rank's time.

Works with the "nccl" backend on GPUs and "gloo" on CPU (the tests)."""
import datetime
import os

import torch

RANK_SEED_STRIDE = 7919  # prime stride between the ranks' input seeds


def init(backend: str = "nccl", timeout_s: float = 120.0):
    """Join the process group named by the torchrun environment (RANK,
    WORLD_SIZE, LOCAL_RANK, MASTER_ADDR/PORT).  Returns (world, rank, local)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return ws, rank, local


def barrier(ws: int) -> None:
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int, device="cuda") -> float:
    """The largest value of x over all ranks (the slowest rank's time)."""
    if ws == 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's synthetic inputs: every rank draws its own slices."""
    return int(base_seed) + RANK_SEED_STRIDE * int(rank)


def job_throughput(units_per_rank: float, ms_max: float, ws: int) -> float:
    """Whole-job rate: the units all ranks processed over the slowest rank's
    time (per second)."""
    return float(units_per_rank) * ws / (ms_max * 1e-3)


def shutdown(ws: int) -> None:
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
