"""Multi-process plumbing for running independent attention layers on several GPUs.

The hot path has no exchange step: every (layer, batch row, KV head) cache is
independent ("Learning how to Forget", §3.1: the policy may differ per batch row
and head).  So ranks never talk on the data path; this module only partitions
the layers, synchronizes the timed region and combines the per-rank timings:
the job's time is the slowest rank's, its throughput the sum of all ranks'
tokens over that time.
"""

from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_rank():
    """(world_size, rank, local_rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: int = 120):
    """Join the process group when launched with more than one rank."""
    ws, rank, local = env_rank()
    if ws > 1 and not dist.is_initialized():
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return ws, rank, local


def _device():
    return torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" \
        else torch.device("cpu")


def barrier():
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float) -> float:
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float) -> float:
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_device())
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def layers_for_rank(n_layers: int, world: int, rank: int):
    """Round-robin partition of independent layers over ranks."""
    return list(range(rank, n_layers, world))


def job_throughput(tokens_this_rank: float, ms_this_rank: float) -> tuple[float, float]:
    """(tokens per second of the whole job, the job's milliseconds = max over ranks)."""
    ms = max_over_ranks(ms_this_rank)
    tokens = sum_over_ranks(tokens_this_rank)
    return tokens / (ms / 1e3), ms


def shutdown():
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
