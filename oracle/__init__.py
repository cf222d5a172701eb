"""CPU oracle for SageAttention-style quantized attention -- TEST INFRASTRUCTURE.

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never calls it and
shares no code with it; the one thing both sides use is the seeded input
generator in ``quantized_attention_qk_b200.inputs``, which holds none of the
method's arithmetic.

The arithmetic lives in ``sage_oracle.c`` (plain C, single-threaded, fp64 plus
IEEE fp32 where the scheme fixes fp32).  This module only marshals torch /
numpy arrays into it, one (batch, head) slab at a time.

Readings of the pages that the oracle follows are named C1..C9 in the C file;
the pins that tie it to the mathematics are in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sage_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-fexcess-precision=standard", "-Wall", "-Wextra"]

Q_BLOCK = 128
K_BLOCK = 64
SEL_TILE = 128  # query / key tile of the block-sparse selection (reading S1)


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to its source (gcc); return its path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Flags(ctypes.Structure):
    _fields_ = [("int8_qk", ctypes.c_int), ("fp8_p", ctypes.c_int), ("fp8_v", ctypes.c_int),
                ("round_bf16", ctypes.c_int), ("smooth_k", ctypes.c_int), ("k_residual", ctypes.c_int)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P, I64, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.oracle_attn_exact.argtypes = [P, I64, P, I64, P, I64, I32, I32, ctypes.c_double, P, I32, P, P]
        L.oracle_quantize.argtypes = [P, I64, P, I64, P, I64, I32, I32, I32, P, P, P, P, P, P, P]
        L.oracle_attn_quant.argtypes = [P, I64, P, I64, P, I64, I32, I32, ctypes.c_float,
                                        ctypes.POINTER(_Flags), P, I32, P, P]
        L.oracle_attn_quant_masked.argtypes = [P, I64, P, I64, P, I64, I32, I32, ctypes.c_float,
                                               ctypes.POINTER(_Flags), P, P, I32, P, P]
        L.oracle_block_scores.argtypes = [P, P, P, P, I32, I32, ctypes.c_float, P]
        L.oracle_block_select.argtypes = [P, I32, ctypes.c_double, P]
        L.oracle_int8_gemm_nt.argtypes = [P, I64, P, I64, I32, I32, I32, P]
        L.oracle_quantize_kres.argtypes = [P, I64, I32, I32, P, P, P]
        L.oracle_e4m3_encode_array.argtypes = [P, I64, P]
        L.oracle_e4m3_decode_array.argtypes = [P, I64, P]
        L.oracle_bf16_rne_array.argtypes = [P, I64, P]
        L.oracle_s3_exp2_array.argtypes = [P, I64, P]
        for f in ("oracle_attn_exact", "oracle_quantize", "oracle_attn_quant", "oracle_int8_gemm_nt",
                  "oracle_quantize_kres", "oracle_attn_quant_masked", "oracle_block_scores", "oracle_block_select"):
            getattr(L, f).restype = I32
        _lib = L
    return _lib


# --------------------------------------------------------------------------
# marshalling helpers
# --------------------------------------------------------------------------

def _slab(t: torch.Tensor, b: int, h: int):
    """(pointer, row stride) of the [N, d] slab (b, h) of a [B,H,N,d] bf16 CPU tensor."""
    assert t.dtype == torch.bfloat16 and t.device.type == "cpu" and t.stride(3) == 1
    ptr = t.data_ptr() + (b * t.stride(0) + h * t.stride(1)) * 2
    return ctypes.c_void_p(ptr), t.stride(2)


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def _rows_array(rows, N):
    if rows is None:
        rows = np.arange(N, dtype=np.int32)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int32))


# --------------------------------------------------------------------------
# public functions (per whole [B,H,N,d] tensors)
# --------------------------------------------------------------------------

def attn_exact(q, k, v, sm_scale, rows=None, want_weights=False):
    """Exact fp64 attention.  q,k,v: bf16 [B,H,N,d] on CPU (any strides, channel stride 1).
    Returns out [B,H,R,d] float64 (and weights [B,H,R,N] if asked)."""
    B, H, N, d = q.shape
    r = _rows_array(rows, N)
    out = np.zeros((B, H, len(r), d), dtype=np.float64)
    w = np.zeros((B, H, len(r), N), dtype=np.float64) if want_weights else None
    L = lib()
    for b in range(B):
        for h in range(H):
            (qp, qs), (kp, ks), (vp, vs) = _slab(q, b, h), _slab(k, b, h), _slab(v, b, h)
            ob = np.zeros((len(r), d), dtype=np.float64)
            wb = np.zeros((len(r), N), dtype=np.float64) if want_weights else None
            _check(L.oracle_attn_exact(qp, qs, kp, ks, vp, vs, N, d, float(sm_scale), _ptr(r), len(r),
                                       _ptr(ob), _ptr(wb) if wb is not None else None), "attn_exact")
            out[b, h] = ob
            if want_weights:
                w[b, h] = wb
    return (out, w) if want_weights else out


def quantize(q, k, v, smooth_k=True):
    """Block quantization of every slab.  Returns a dict of numpy arrays:
    q_i8 [B,H,N,d] int8, q_scale [B,H,ceil(N/128)] f32, k_i8, k_scale [B,H,ceil(N/64)],
    k_mean [B,H,d] f32, v_e4m3 [B,H,N,d] uint8 (token-major), v_scale [B,H,d] f32."""
    B, H, N, d = q.shape
    nqb, nkb = -(-N // Q_BLOCK), -(-N // K_BLOCK)
    res = dict(q_i8=np.zeros((B, H, N, d), np.int8), q_scale=np.zeros((B, H, nqb), np.float32),
               k_i8=np.zeros((B, H, N, d), np.int8), k_scale=np.zeros((B, H, nkb), np.float32),
               k_mean=np.zeros((B, H, d), np.float32), v_e4m3=np.zeros((B, H, N, d), np.uint8),
               v_scale=np.zeros((B, H, d), np.float32))
    L = lib()
    for b in range(B):
        for h in range(H):
            (qp, qs), (kp, ks), (vp, vs) = _slab(q, b, h), _slab(k, b, h), _slab(v, b, h)
            slab = {kk: np.ascontiguousarray(vv[b, h]) for kk, vv in res.items()}
            _check(L.oracle_quantize(qp, qs, kp, ks, vp, vs, N, d, int(bool(smooth_k)),
                                     _ptr(slab["q_i8"]), _ptr(slab["q_scale"]),
                                     _ptr(slab["k_i8"]), _ptr(slab["k_scale"]), _ptr(slab["k_mean"]),
                                     _ptr(slab["v_e4m3"]), _ptr(slab["v_scale"])), "quantize")
            for kk in res:
                res[kk][b, h] = slab[kk]
    return res


def quantize_kres(k):
    """K-residual codes of every slab ("ComfyUI-sol-attn", 核心亮点 item 1).
    Returns dict k_i8 [B,H,N,d] int8, k_scale [B,H,ceil(N/64)] f32,
    k_bmean [B,H,ceil(N/64),d] bf16 bit patterns (uint16)."""
    B, H, N, d = k.shape
    nkb = -(-N // K_BLOCK)
    res = dict(k_i8=np.zeros((B, H, N, d), np.int8), k_scale=np.zeros((B, H, nkb), np.float32),
               k_bmean=np.zeros((B, H, nkb, d), np.uint16))
    L = lib()
    for b in range(B):
        for h in range(H):
            kp, ks = _slab(k, b, h)
            slab = {kk: np.ascontiguousarray(vv[b, h]) for kk, vv in res.items()}
            _check(L.oracle_quantize_kres(kp, ks, N, d, _ptr(slab["k_i8"]), _ptr(slab["k_scale"]),
                                          _ptr(slab["k_bmean"])), "quantize_kres")
            for kk in res:
                res[kk][b, h] = slab[kk]
    return res


def attn_quant(q, k, v, sm_scale, rows=None, int8_qk=True, fp8_p=True, fp8_v=True,
               round_bf16=True, smooth_k=True, heads=None, k_residual=False, kv_keep=None):
    """Quant-emulation attention.  Returns (out_f64 [B,H,R,d], out_bf16 bits [B,H,R,d] uint16).
    ``heads`` optionally restricts the work to a list of (b, h) pairs (others stay zero).
    ``k_residual``: K-residual quantization with the block-mean term kept
    (oracle_quantize_kres) instead of the smoothing.
    ``kv_keep``: block-sparse skipping, [B,H,nt,nt] (nt = ceil(N/128)), nonzero
    where query tile i attends to key tile j; a row whose tile keeps nothing
    returns 0 (oracle_attn_quant_masked)."""
    B, H, N, d = q.shape
    r = _rows_array(rows, N)
    nt = -(-N // SEL_TILE)
    if kv_keep is not None:
        kv_keep = np.asarray(kv_keep)
        assert kv_keep.shape == (B, H, nt, nt), kv_keep.shape
    f = _Flags(int(int8_qk), int(fp8_p), int(fp8_v), int(round_bf16), int(smooth_k), int(k_residual))
    out = np.zeros((B, H, len(r), d), dtype=np.float64)
    outb = np.zeros((B, H, len(r), d), dtype=np.uint16)
    L = lib()
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in pairs:
        (qp, qs), (kp, ks), (vp, vs) = _slab(q, b, h), _slab(k, b, h), _slab(v, b, h)
        ob = np.zeros((len(r), d), dtype=np.float64)
        obb = np.zeros((len(r), d), dtype=np.uint16)
        keep = None if kv_keep is None else np.ascontiguousarray(kv_keep[b, h] != 0, dtype=np.uint8)
        _check(L.oracle_attn_quant_masked(qp, qs, kp, ks, vp, vs, N, d, ctypes.c_float(sm_scale),
                                          ctypes.byref(f), _ptr(keep) if keep is not None else None,
                                          _ptr(r), len(r), _ptr(ob), _ptr(obb)), "attn_quant")
        out[b, h] = ob
        outb[b, h] = obb
    return out, outb


def block_scores(q, k, v, sm_scale, codes=None):
    """Tile-pair scores of the block-sparse selection (reading S2,
    oracle_block_scores): [B,H,nt,nt] float32, from the oracle's own codes
    (``codes`` = a result of quantize(q, k, v), computed if not given)."""
    B, H, N, d = q.shape
    nt = -(-N // SEL_TILE)
    c = quantize(q, k, v) if codes is None else codes
    out = np.zeros((B, H, nt, nt), dtype=np.float32)
    L = lib()
    for b in range(B):
        for h in range(H):
            qc = np.ascontiguousarray(c["q_i8"][b, h])
            kc = np.ascontiguousarray(c["k_i8"][b, h])
            qs = np.ascontiguousarray(c["q_scale"][b, h], dtype=np.float32)
            ks = np.ascontiguousarray(c["k_scale"][b, h], dtype=np.float32)
            sb = np.zeros((nt, nt), dtype=np.float32)
            _check(L.oracle_block_scores(_ptr(qc), _ptr(qs), _ptr(kc), _ptr(ks), N, d,
                                         ctypes.c_float(sm_scale), _ptr(sb)), "block_scores")
            out[b, h] = sb
    return out


def block_select(sbar, N, tau):
    """Kept key tiles per query tile (reading S3, oracle_block_select):
    uint8 [B,H,nt,nt] from scores [B,H,nt,nt]."""
    sbar = np.asarray(sbar, dtype=np.float32)
    B, H, nt, _ = sbar.shape
    assert nt == -(-N // SEL_TILE)
    keep = np.zeros((B, H, nt, nt), dtype=np.uint8)
    L = lib()
    for b in range(B):
        for h in range(H):
            sb = np.ascontiguousarray(sbar[b, h])
            kb = np.zeros((nt, nt), dtype=np.uint8)
            _check(L.oracle_block_select(_ptr(sb), N, float(tau), _ptr(kb)), "block_select")
            keep[b, h] = kb
    return keep


def tau_schedule(step, n_steps, tau_start, tau_end):
    """Reading S4: tau at sampling step ``step`` of ``n_steps``, moving linearly
    from tau_start (first step) to tau_end (last step); steps outside the
    range take the nearer end ("ComfyUI-sol-attn", 核心亮点 item 4: sparse
    early, dense late)."""
    if n_steps <= 1:
        return float(tau_end)
    t = min(max(step, 0), n_steps - 1) / (n_steps - 1)
    return float(tau_start) + (float(tau_end) - float(tau_start)) * t


def int8_gemm_nt(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """s[i,j] = sum_c a[i,c] b[j,c] for int8 row-major a [m,d], b [n,d] -> int32 [m,n]."""
    a = np.ascontiguousarray(a, dtype=np.int8)
    b = np.ascontiguousarray(b, dtype=np.int8)
    m, d = a.shape
    n = b.shape[0]
    s = np.zeros((m, n), dtype=np.int32)
    _check(lib().oracle_int8_gemm_nt(_ptr(a), d, _ptr(b), d, m, n, d, _ptr(s)), "int8_gemm_nt")
    return s


def e4m3_encode(x) -> np.ndarray:
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64).ravel())
    c = np.zeros(x.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_array(_ptr(x), x.size, _ptr(c))
    return c


def e4m3_decode(c) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(c, dtype=np.uint8).ravel())
    x = np.zeros(c.shape, dtype=np.float64)
    lib().oracle_e4m3_decode_array(_ptr(c), c.size, _ptr(x))
    return x


def s3_exp2(x) -> np.ndarray:
    """The fp32 exponential of the selection's masses (reading S3) for x <= 0."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32).ravel())
    y = np.zeros(x.shape, dtype=np.float32)
    lib().oracle_s3_exp2_array(_ptr(x), x.size, _ptr(y))
    return y


def bf16_rne(x) -> np.ndarray:
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64).ravel())
    h = np.zeros(x.shape, dtype=np.uint16)
    lib().oracle_bf16_rne_array(_ptr(x), x.size, _ptr(h))
    return h


def bf16_bits_to_f64(h) -> np.ndarray:
    h = np.asarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
