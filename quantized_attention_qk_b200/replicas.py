"""Running the forward on several GPUs of one node.

The attention of one (batch, head) pair needs nothing from any other, so the
GPUs share no data on the way in.  Two uses:

* replicas (what bench.py measures): every rank runs its own copy of the
  workload and the ranks only agree on timing (a barrier on both sides of the
  timed region and the maximum of the per-rank times); the job's throughput is
  the work of all ranks divided by that maximum (weak scaling);
* head sharding (`sharded_forward`): one problem split by heads, rank r
  computing heads `head_range(H, world, r)` of every batch row on its own
  device, optionally followed by one all-gather of the bf16 outputs so that
  every rank holds the whole result (strong scaling).

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


def head_range(H: int, world: int, rank: int) -> tuple[int, int]:
    """Heads [h0, h1) of `rank` when H heads are split over `world` ranks as
    evenly as possible (the first H mod world ranks take one more)."""
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def sharded_forward(q, k, v, reps: Replicas, sm_scale=None, gather: bool = True, attn=None, out_dtype=None):
    """Head-sharded forward of one problem over the ranks of `reps`.

    Every rank holds q, k, v ([B,H,N,d] views, any strides) and computes its
    heads `head_range(H, world, rank)` of every batch row through `attn`
    (default: the library's sage_attn_fwd) on strided views of them, without
    copies.  With `gather` the ranks then exchange their outputs (one
    all-gather, outputs padded to the largest share) and each returns the
    whole [B,H,N,d] result; without it each returns its own [B,h1-h0,N,d]
    part.  A rank whose share is empty computes nothing.  `out_dtype` is the
    dtype `attn` returns (default q's, as sage_attn_fwd does); an empty share
    takes it, so that all ranks gather the same type."""
    if attn is None:
        from quantized_attention_qk_b200 import sage_attn_fwd as attn
    B, H, N, d = q.shape
    h0, h1 = head_range(H, reps.world, reps.rank)
    if h1 > h0:
        part = attn(q[:, h0:h1], k[:, h0:h1], v[:, h0:h1], sm_scale=sm_scale)
    else:
        part = torch.empty(B, 0, N, d, dtype=out_dtype or q.dtype, device=q.device)
    if not gather or reps.world == 1:
        return part
    hmax = -(-H // reps.world)
    buf = torch.zeros(B, hmax, N, d, dtype=part.dtype, device=part.device)
    buf[:, : h1 - h0] = part
    parts = [torch.empty_like(buf) for _ in range(reps.world)]
    dist.all_gather(parts, buf)
    out = torch.empty(B, H, N, d, dtype=part.dtype, device=part.device)
    for r in range(reps.world):
        a, b = head_range(H, reps.world, r)
        out[:, a:b] = parts[r][:, : b - a]
    return out


def timed_sharded(q, k, v, reps: Replicas, steps: int, warmup: int, sm_scale=None, attn=None, out_dtype=None,
                  before_step=None):
    """Time `steps` head-sharded forwards of one problem (each with the
    all-gather) after `warmup` untimed ones.  On CUDA tensors each step is
    timed with events on the current stream (which waits for the collective);
    on CPU tensors with the host clock.  `before_step` (e.g. an L2 flush) runs
    before every timed step, outside its timing.  Every rank takes the same
    collective steps.  Returns (the last gathered output, this rank's total
    ms, the maximum of the totals over the ranks)."""
    import time

    cuda = q.is_cuda
    out = None
    for _ in range(warmup):
        out = sharded_forward(q, k, v, reps, sm_scale=sm_scale, attn=attn, out_dtype=out_dtype)
    if cuda:
        torch.cuda.synchronize()
    reps.barrier()
    if cuda:
        torch.cuda.synchronize()
    total = 0.0
    for _ in range(steps):
        if before_step is not None:
            before_step()
        if cuda:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            out = sharded_forward(q, k, v, reps, sm_scale=sm_scale, attn=attn, out_dtype=out_dtype)
            e1.record()
            e1.synchronize()
            total += e0.elapsed_time(e1)
        else:
            t0 = time.perf_counter()
            out = sharded_forward(q, k, v, reps, sm_scale=sm_scale, attn=attn, out_dtype=out_dtype)
            total += (time.perf_counter() - t0) * 1e3
    if cuda:
        torch.cuda.synchronize()
    reps.barrier()
    return out, total, reps.max(total)
