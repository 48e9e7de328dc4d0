"""Process-group plumbing for running the looped mixer on several GPUs of one node.

Every (loop, batch, head) unit of the mixer is an independent recurrence ("LT2 transformer
looped a tempo lineare", section "Sostituire il motore": one state per sequence and head,
re-run in each loop of section "Profondita presa in prestito"), so several GPUs either run
replicas of a workload (weak scaling) or split its units between them; the data path has no
collective.  What remains is host plumbing: rank discovery, the timing barrier, the maximum of
the per-rank step times, the split of units between ranks and the whole-job throughput.  The
functions take the backend and device explicitly, so the same code runs on NCCL (one process
per GPU) and on gloo (the CPU tests).
"""
import datetime
import os

import torch


def env_ranks():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 when absent)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend="nccl", timeout_s=120, device=None):
    """Join the process group when WORLD_SIZE > 1.  `device` (a torch.device) is bound to the
    group for NCCL.  Returns (world, rank, local_rank)."""
    world, rank, local = env_ranks()
    if world > 1 and not torch.distributed.is_initialized():
        kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
        if device is not None and backend == "nccl":
            kw["device_id"] = device
        torch.distributed.init_process_group(backend, **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world, device="cpu"):
    """The largest value of a per-rank float (the step time of the slowest rank)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def split_units(n_units, world, rank):
    """Contiguous, near-equal share [start, stop) of n_units for `rank`: the first
    n_units % world ranks take one unit more.  The shares of all ranks cover every unit once."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def whole_job_rate(items_per_rank, world, ms_max):
    """Items per second of the whole job: every rank's items over the slowest rank's time."""
    if ms_max <= 0:
        raise ValueError("step time must be positive")
    return items_per_rank * world / (ms_max * 1e-3)
