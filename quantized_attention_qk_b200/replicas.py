"""Coordination of replicas when the forward runs on several GPUs of one node.

The attention of one (batch, head) pair needs nothing from any other, so the
GPUs share no data: every rank runs its own replica of the workload on its own
device and the ranks only agree on timing (a barrier on both sides of the timed
region and the maximum of the per-rank times).  The job's throughput is then
the work of all ranks divided by that maximum (weak scaling).

One process per GPU, launched by torchrun (RANK, LOCAL_RANK, WORLD_SIZE,
MASTER_ADDR, MASTER_PORT in the environment).  NCCL carries the two collectives
on GPUs; gloo carries them in the CPU tests.  Every rank takes the same
collective steps in the same order; a short process-group timeout turns a rank
that died or never arrived into an error on the others instead of a hang.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_int(name: str, default: int) -> int:
    v = os.environ.get(name)
    return int(v) if v not in (None, "") else default


class Replicas:
    """This process's place among the replicas, and the two collectives they use."""

    def __init__(self, device: torch.device | None = None, backend: str | None = None, timeout_s: float = 120.0):
        self.world = env_int("WORLD_SIZE", 1)
        self.rank = env_int("RANK", 0)
        self.local_rank = env_int("LOCAL_RANK", 0)
        self.device = device
        if self.world < 1 or not 0 <= self.rank < self.world:
            raise ValueError(f"bad rank {self.rank} of world size {self.world}")
        if backend is None:
            backend = "nccl" if device is not None and device.type == "cuda" else "gloo"
        self.backend = backend
        self._own_group = False
        if self.world > 1 and not dist.is_initialized():
            kwargs = {"timeout": datetime.timedelta(seconds=timeout_s)}
            if backend == "nccl" and device is not None:
                kwargs["device_id"] = device
            dist.init_process_group(backend, **kwargs)
            self._own_group = True

    @property
    def is_root(self) -> bool:
        return self.rank == 0

    def barrier(self) -> None:
        if self.world > 1:
            dist.barrier()

    def max(self, x: float) -> float:
        """Largest value of x over all ranks (x itself on one rank)."""
        if self.world == 1:
            return float(x)
        dev = self.device if self.backend == "nccl" else torch.device("cpu")
        t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self) -> None:
        if self._own_group and dist.is_initialized():
            dist.destroy_process_group()
        self._own_group = False


def whole_job_tops(world: int, ops_per_step: float, steps: int, max_total_ms: float) -> float:
    """Throughput of the whole job in tera-operations per second: the work of all
    `world` replicas over `steps` steps divided by the slowest rank's time."""
    if max_total_ms <= 0:
        raise ValueError("the timed region must have a positive duration")
    return world * ops_per_step * steps / (max_total_ms * 1e-3) / 1e12
