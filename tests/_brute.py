"""Independent pure-Python restatements used to pin the C oracle.

Nothing here imports the oracle or the CUDA library.  These are written from
the definitions, in a different shape from the oracle (explicit loops, tiled
online evaluation), so that a dropped term, a wrong sign or a transposed
operand in either one shows up as a mismatch.  Library casts (torch's float8
and bfloat16 conversions) stand in for the number formats where used.
"""
from __future__ import annotations

import math

import numpy as np
import torch

LOG2E = 1.4426950408889634


def bf16_values(t: torch.Tensor):
    """bf16 tensor [N,d] -> nested Python float lists (exact)."""
    return t.float().tolist()


def exact_attention_loops(q, k, v, sm_scale):
    """softmax(q k^T * sm_scale) v with explicit loops and math.exp (natural base)."""
    N = len(k)
    out = []
    for qi in q:
        scores = [sm_scale * math.fsum(a * b for a, b in zip(qi, kj)) for kj in k]
        mx = max(scores)
        e = [math.exp(s - mx) for s in scores]
        z = math.fsum(e)
        row = []
        for c in range(len(v[0])):
            row.append(math.fsum(e[j] * v[j][c] for j in range(N)) / z)
        out.append(row)
    return out


def _e4m3_torch(x: np.ndarray) -> np.ndarray:
    """Round fp32 values (|x| <= 448) to e4m3 with torch's cast; return the values."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).to(torch.float64).numpy()


def quant_codes_numpy(q: np.ndarray, k: np.ndarray, v: np.ndarray):
    """Block quantization written with numpy fp32 arithmetic.
    q,k,v: float32 [N,d] (bf16-exact values)."""
    N, d = q.shape
    f32 = np.float32
    # K mean over tokens, accumulated exactly then rounded to fp32
    mu = np.array([f32(math.fsum(k[:, c].astype(np.float64)) / N) for c in range(d)], dtype=f32)
    qc = np.zeros((N, d), np.int64)
    qs = []
    for b0 in range(0, N, 128):
        blk = q[b0:b0 + 128]
        amax = f32(np.max(np.abs(blk)))
        if amax == 0:
            qs.append(f32(0))
            continue
        inv = f32(f32(127) / amax)
        qs.append(f32(amax / f32(127)))
        qc[b0:b0 + 128] = np.clip(np.rint((blk * inv).astype(f32)), -127, 127)
    ksm = (k - mu[None, :]).astype(f32)
    kc = np.zeros((N, d), np.int64)
    ks = []
    for b0 in range(0, N, 64):
        blk = ksm[b0:b0 + 64]
        amax = f32(np.max(np.abs(blk)))
        if amax == 0:
            ks.append(f32(0))
            continue
        inv = f32(f32(127) / amax)
        ks.append(f32(amax / f32(127)))
        kc[b0:b0 + 64] = np.clip(np.rint((blk * inv).astype(f32)), -127, 127)
    vamax = np.max(np.abs(v), axis=0).astype(f32)
    vval = np.zeros((N, d), np.float64)
    vs = np.zeros(d, f32)
    for c in range(d):
        if vamax[c] == 0:
            continue
        inv = f32(f32(448) / vamax[c])
        vs[c] = f32(vamax[c] / f32(448))
        vval[:, c] = _e4m3_torch((v[:, c] * inv).astype(f32)) * float(vs[c])
    return qc, np.array(qs, f32), kc, np.array(ks, f32), mu, vval, vs


def tiled_online_quant(q: np.ndarray, k: np.ndarray, v: np.ndarray, sm_scale: float, bkv: int):
    """The quantized scheme evaluated tile by tile with an online softmax whose
    running max lives on the integer (log2) grid: m' = max(m, ceil(tile max)),
    O and l rescaled by 2^(m - m') when it moves.  Returns fp64 [N,d] before
    the final bf16 rounding."""
    N, d = q.shape
    f32 = np.float32
    qc, qs, kc, ks, _mu, vval, _vs = quant_codes_numpy(q, k, v)
    S = qc @ kc.T  # exact int64
    s_l2 = f32(f32(sm_scale) * f32(LOG2E))
    out = np.zeros((N, d), np.float64)
    for i in range(N):
        cq = f32(qs[i // 128] * s_l2)
        m = -math.inf
        l = 0.0
        o = np.zeros(d, np.float64)
        for j0 in range(0, N, bkv):
            j1 = min(N, j0 + bkv)
            c = np.array([f32(cq * ks[j // 64]) for j in range(j0, j1)], dtype=np.float64)
            x = S[i, j0:j1].astype(np.float64) * c
            m_new = max(m, math.ceil(float(np.max(x))))
            alpha = 2.0 ** (m - m_new) if m != -math.inf else 0.0
            p = np.exp2(x - m_new)
            P = _e4m3_torch((p * 448.0).astype(np.float32))
            l = l * alpha + math.fsum(p)
            o = o * alpha + P @ vval[j0:j1]
            m = m_new
        out[i] = o / (448.0 * l)
    return out
