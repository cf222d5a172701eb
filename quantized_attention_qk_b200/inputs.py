"""Seeded synthetic attention inputs (bf16 Q, K, V) for tests, smoke and bench.

This module is shared by the CUDA path's callers and by the CPU oracle's
callers, so it holds no step of the attention method: it only draws numbers.

Recipe (every workload):
  * ``torch.Generator`` on the CPU, seeded per workload; fields are drawn in a
    fixed order: Q noise, K noise, V noise (each [B,H,N,d], N(0,1), fp32), then
    the K bias, then the outlier channel set.
  * K bias: one N(0, sigma^2) draw per (head, channel), shared by every batch
    and token (a per-channel offset, the structure K smoothing removes).
  * Outliers: round(frac * H * d) (head, channel) pairs drawn without
    replacement; the whole K channel (bias included) is multiplied by 8.
  * Values are rounded to bf16 (round-to-nearest-even, torch's cast).
  * Layout "contiguous": separate [B,H,N,d] tensors.  Layout "fused": one
    [B,N,3,H,d] buffer (the output of a fused qkv projection) and q/k/v are
    strided [B,H,N,d] views of it with strides (N*3*H*d, d, 3*H*d, 1).

The workloads mirror the shapes the pages talk about: a Flux-like image DiT
(4096 image + 512 text tokens), an SDXL-like UNet self-attention, the
864x480 5 s video of the MiniMax H3 measurement (latent 54x30x21 = 34020
tokens), and the 8K/16K/65K-token lengths of the Sol-Attn timings.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    layout: str = "contiguous"   # or "fused"
    bias_sigma: float = 0.0
    outlier_frac: float = 0.0
    seed: int = 0

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def ops(self) -> int:
        """4*B*H*N^2*d: the two dense contractions (QK^T and PV), 2 ops per MAC."""
        return 4 * self.B * self.H * self.N * self.N * self.d

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 256, 64, "contiguous", 2.0, 0.0, 1001),
    "flux": Workload("flux", 1, 24, 4608, 128, "fused", 4.0, 0.01, 1002),
    "sdxl": Workload("sdxl", 4, 10, 4096, 64, "contiguous", 2.0, 0.0, 1003),
    "video": Workload("video", 1, 40, 34020, 128, "fused", 4.0, 0.01, 1004),
    "long8k": Workload("long8k", 1, 24, 8192, 128, "contiguous", 4.0, 0.0, 5013),
    "long16k": Workload("long16k", 1, 24, 16384, 128, "contiguous", 4.0, 0.0, 5014),
    "long64k": Workload("long64k", 1, 24, 65536, 128, "contiguous", 4.0, 0.0, 5016),
}


def make_qkv(w: Workload, device="cpu"):
    """Return (q, k, v, storage): bf16 [B,H,N,d] tensors (views for the fused
    layout) on ``device`` plus the list of underlying buffers."""
    B, H, N, d = w.B, w.H, w.N, w.d
    g = torch.Generator().manual_seed(int(w.seed))
    qf = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    kf = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    vf = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    bias = torch.randn(H, d, generator=g, dtype=torch.float32) * float(w.bias_sigma)
    kf += bias.view(1, H, 1, d)
    n_out = int(round(w.outlier_frac * H * d))
    if n_out > 0:
        idx = torch.randperm(H * d, generator=g)[:n_out]
        mult = torch.ones(H * d)
        mult[idx] = 8.0
        kf *= mult.view(1, H, 1, d)
    if w.layout == "fused":
        qkv = torch.empty(B, N, 3, H, d, dtype=torch.bfloat16)
        qkv[:, :, 0].copy_(qf.permute(0, 2, 1, 3))
        del qf
        qkv[:, :, 1].copy_(kf.permute(0, 2, 1, 3))
        del kf
        qkv[:, :, 2].copy_(vf.permute(0, 2, 1, 3))
        del vf
        qkv = qkv.to(device)
        q, k, v = (qkv[:, :, i].permute(0, 2, 1, 3) for i in range(3))
        return q, k, v, [qkv]
    if w.layout != "contiguous":
        raise ValueError(f"unknown layout {w.layout!r}")
    q = qf.to(torch.bfloat16).to(device)
    k = kf.to(torch.bfloat16).to(device)
    v = vf.to(torch.bfloat16).to(device)
    return q, k, v, [q, k, v]


def tiny_custom(B, H, N, d, seed, layout="contiguous", bias_sigma=0.0, outlier_frac=0.0) -> Workload:
    """A small ad-hoc workload (for edge-case tests: ragged N, one head, ...)."""
    return Workload(f"custom_{B}x{H}x{N}x{d}", B, H, N, d, layout, bias_sigma, outlier_frac, seed)
