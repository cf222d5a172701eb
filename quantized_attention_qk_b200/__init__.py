"""quantized_attention_qk_b200 -- SageAttention-style quantized attention on B200.

Thin Python binding of ``lib/libsage.so`` (include/sage.h).  Every function
here only marshals torch tensors into pointers, strides and sizes and calls the
C ABI function of the same name; all arithmetic runs in the library's CUDA
kernels.  torch provides device memory and streams.  There is no fallback: if
the library is missing or a call fails, an exception is raised.

Tensors are [B, H, N, d] bf16 views with channel stride 1 (e.g. slices of a
fused [B, N, 3, H, d] qkv buffer, read in place).
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "SageError", "lib", "sage_attn_fwd", "sage_attn_quantized", "sage_quant_qk", "sage_quant_v",
    "sage_attn_dense_ref_gpu", "sage_debug_qk_tile", "sage_quant_qk_noalloc", "sage_attn_workspace_bytes",
    "sage_quant_workspace_bytes", "sage_check", "sage_attn_fwd_host", "n_pad",
    "sage_block_select", "sage_attn_fwd_sparse", "sage_tau_schedule", "sage_block_mask_bytes",
    "sage_attn_sparse_workspace_bytes", "n_tiles", "mask_words", "mask_to_keep", "keep_to_mask",
    "sage_attn_fwd_kres", "sage_quant_k_residual", "sage_attn_kres_workspace_bytes", "sage_attn_fwd_fused_q",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libsage.so")
Q_BLOCK, K_BLOCK = 128, 64

SAGE_STATUS = {0: "SAGE_OK", 1: "SAGE_ERR_INVALID_ARG", 2: "SAGE_ERR_UNSUPPORTED", 3: "SAGE_ERR_WORKSPACE",
               4: "SAGE_ERR_CUDA", 5: "SAGE_ERR_TIMEOUT"}


class SageError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{SAGE_STATUS.get(status, status)}: {message}")
        self.status = status


_lib = None
_P, _I64P, _I32, _SZ = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64), ctypes.c_int, ctypes.c_size_t
_SIGS = {
    "sage_status_string": ([_I32], ctypes.c_char_p),
    "sage_last_error_message": ([], ctypes.c_char_p),
    "sage_check": ([_P], _I32),
    "sage_attn_workspace_bytes": ([_I32] * 4, _SZ),
    "sage_quant_workspace_bytes": ([_I32] * 4, _SZ),
    "sage_quant_qk": ([_P, _I64P, _P, _I64P, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P, _SZ, _P], _I32),
    "sage_quant_qk_noalloc": ([_P, _I64P, _P, _I64P, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P], _I32),
    "sage_quant_v": ([_P, _I64P, _I32, _I32, _I32, _I32, _P, _P, _P, _SZ, _P], _I32),
    "sage_attn_quantized": ([_P, _P, _P, _P, _P, _P, _P, _I64P, _I32, _I32, _I32, _I32, ctypes.c_float, _P], _I32),
    "sage_attn_fwd": ([_P, _I64P, _P, _I64P, _P, _I64P, _P, _I64P, _I32, _I32, _I32, _I32, ctypes.c_float,
                       _P, _SZ, _P], _I32),
    "sage_attn_fwd_ev": ([_P, _I64P, _P, _I64P, _P, _I64P, _P, _I64P, _I32, _I32, _I32, _I32, ctypes.c_float,
                          _P, _SZ, _P, _P, _P], _I32),
    "sage_attn_dense_ref_gpu": ([_P, _I64P, _P, _I64P, _P, _I64P, _P, _I64P, _I32, _I32, _I32, _I32,
                                 ctypes.c_float, _P], _I32),
    "sage_debug_qk_tile": ([_P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _P, _P], _I32),
    "sage_attn_fwd_host_scratch_bytes": ([_I32, _I32, _I32, _I32], _SZ),
    "sage_attn_fwd_host": ([_P, _I32, _P, _I32, _I32, _I32, _I32, ctypes.c_float, _P, _SZ, _P], _I32),
    "sage_block_mask_bytes": ([_I32, _I32, _I32], _SZ),
    "sage_block_select_workspace_bytes": ([_I32] * 4, _SZ),
    "sage_block_select": ([_P, _P, _P, _P, _I32, _I32, _I32, _I32, ctypes.c_float, ctypes.c_float, _P, _P, _P, _SZ,
                           _P], _I32),
    "sage_attn_sparse_workspace_bytes": ([_I32] * 4, _SZ),
    "sage_attn_fwd_sparse": ([_P, _I64P, _P, _I64P, _P, _I64P, _P, _I64P, _I32, _I32, _I32, _I32, ctypes.c_float,
                              ctypes.c_float, _P, _P, _P, _SZ, _P, _P, _P], _I32),
    "sage_tau_schedule": ([_I32, _I32, ctypes.c_float, ctypes.c_float], ctypes.c_float),
    "sage_attn_kres_workspace_bytes": ([_I32] * 4, _SZ),
    "sage_debug_wait_timeout": ([_I32, _P], _I32),
    "sage_debug_ex2_probe": ([_P, _I32, _I32, _P], _I32),
    "sage_attn_fwd_fused_q": ([_P, _I64P, _P, _I64P, _P, _I64P, _P, _I64P, _I32, _I32, _I32, _I32, ctypes.c_float,
                               _P, _SZ, _P, _P, _P], _I32),
    "sage_quant_k_residual": ([_P, _I64P, _I32, _I32, _I32, _I32, _P, _P, _P, _P], _I32),
    "sage_attn_fwd_kres": ([_P, _I64P, _P, _I64P, _P, _I64P, _P, _I64P, _I32, _I32, _I32, _I32, ctypes.c_float,
                            _P, _SZ, _P, _P, _P], _I32),
}


def lib():
    """Load libsage.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with quantized_attention_qk_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _raise(status: int):
    if status != 0:
        raise SageError(status, lib().sage_last_error_message().decode(errors="replace"))


def _run(dev, fn, *args):
    """Call library function ``fn`` with ``dev`` as the current device: the
    library launches its kernels on, and keeps its per-device state for, the
    current device, and rejects tensors that live elsewhere."""
    with torch.cuda.device(dev):
        _raise(fn(*args))


def _strides(t: torch.Tensor):
    return (ctypes.c_int64 * 4)(*t.stride())


def _stream(stream, device):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def n_pad(N: int) -> int:
    return -(-N // Q_BLOCK) * Q_BLOCK


def _check_qkv(*ts):
    for t in ts:
        if t.dim() != 4 or t.dtype != torch.bfloat16 or not t.is_cuda:
            raise ValueError("expected bf16 CUDA tensors of shape [B, H, N, d]")


def sage_attn_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(lib().sage_attn_workspace_bytes(B, H, N, d))


def sage_quant_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(lib().sage_quant_workspace_bytes(B, H, N, d))


def sage_check(stream=None, device=None):
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    _run(dev, lib().sage_check, _stream(stream, dev))


def sage_quant_qk(q, k, workspace=None, stream=None):
    """Smoothing + block INT8 quantization.  Returns dict of device tensors:
    q_i8 [B,H,N_pad,d] int8, q_scale [B,H,N_pad/128], k_i8, k_scale [B,H,N_pad/64], k_mean [B,H,d]."""
    _check_qkv(q, k)
    B, H, N, d = q.shape
    dev = q.device
    npd = n_pad(N)
    r = dict(q_i8=torch.empty(B, H, npd, d, dtype=torch.int8, device=dev),
             q_scale=torch.empty(B, H, npd // Q_BLOCK, dtype=torch.float32, device=dev),
             k_i8=torch.empty(B, H, npd, d, dtype=torch.int8, device=dev),
             k_scale=torch.empty(B, H, npd // K_BLOCK, dtype=torch.float32, device=dev),
             k_mean=torch.empty(B, H, d, dtype=torch.float32, device=dev))
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _run(dev, lib().sage_quant_qk, _ptr(q), _strides(q), _ptr(k), _strides(k), B, H, N, d,
                               _ptr(r["q_i8"]), _ptr(r["q_scale"]), _ptr(r["k_i8"]), _ptr(r["k_scale"]),
                               _ptr(r["k_mean"]), _ptr(workspace), ws_bytes, _stream(stream, dev))
    return r


def sage_quant_qk_noalloc(q, k, out=None, stream=None):
    """sage_quant_qk without a workspace and without any device allocation in
    the library: its statistics scratch is a fixed 4 MiB array in the library's
    device memory (shared by all calls on a device; calls that overlap on the
    GPU race; shapes needing more scratch raise with status 3).  ``out`` optionally supplies the output dict (same keys/shapes as
    sage_quant_qk returns) so that the caller owns every buffer."""
    _check_qkv(q, k)
    B, H, N, d = q.shape
    dev = q.device
    npd = n_pad(N)
    r = out if out is not None else dict(
        q_i8=torch.empty(B, H, npd, d, dtype=torch.int8, device=dev),
        q_scale=torch.empty(B, H, npd // Q_BLOCK, dtype=torch.float32, device=dev),
        k_i8=torch.empty(B, H, npd, d, dtype=torch.int8, device=dev),
        k_scale=torch.empty(B, H, npd // K_BLOCK, dtype=torch.float32, device=dev),
        k_mean=torch.empty(B, H, d, dtype=torch.float32, device=dev))
    _run(dev, lib().sage_quant_qk_noalloc, _ptr(q), _strides(q), _ptr(k), _strides(k), B, H, N, d,
                                       _ptr(r["q_i8"]), _ptr(r["q_scale"]), _ptr(r["k_i8"]), _ptr(r["k_scale"]),
                                       _ptr(r["k_mean"]), _stream(stream, dev))
    return r


def sage_quant_v(v, workspace=None, stream=None):
    """V -> e4m3 with per-channel scales.  Returns (v_e4m3 uint8 [B,H,N_pad,d], v_scale [B,H,d])."""
    _check_qkv(v)
    B, H, N, d = v.shape
    dev = v.device
    v_e4m3 = torch.empty(B, H, n_pad(N), d, dtype=torch.uint8, device=dev)
    v_scale = torch.empty(B, H, d, dtype=torch.float32, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _run(dev, lib().sage_quant_v, _ptr(v), _strides(v), B, H, N, d, _ptr(v_e4m3), _ptr(v_scale), _ptr(workspace),
                              ws_bytes, _stream(stream, dev))
    return v_e4m3, v_scale


def sage_attn_quantized(q_i8, q_scale, k_i8, k_scale, v_e4m3, v_scale, N: int, sm_scale=None, out=None, stream=None):
    """The fused attention kernel on existing codes; returns bf16 [B,H,N,d]."""
    B, H, _, d = q_i8.shape
    dev = q_i8.device
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=dev)
    for t in (q_i8, q_scale, k_i8, k_scale, v_e4m3, v_scale):
        if not t.is_contiguous():
            raise ValueError("code and scale tensors must be contiguous")
    _run(dev, lib().sage_attn_quantized, _ptr(q_i8), _ptr(q_scale), _ptr(k_i8), _ptr(k_scale), _ptr(v_e4m3),
                                     _ptr(v_scale), _ptr(out), _strides(out), B, H, N, d,
                                     ctypes.c_float(sm_scale), _stream(stream, dev))
    return out


def sage_attn_fwd(q, k, v, sm_scale=None, out=None, workspace=None, stream=None, attn_events=None):
    """Quantized attention forward on device tensors; returns bf16 [B,H,N,d].
    ``attn_events``: optional pair of recorded-once torch.cuda.Event objects that
    the library records right before / after the fused attention kernel."""
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    dev = q.device
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    if attn_events is None:
        _run(dev, lib().sage_attn_fwd, _ptr(q), _strides(q), _ptr(k), _strides(k), _ptr(v), _strides(v),
                                   _ptr(out), _strides(out), B, H, N, d, ctypes.c_float(sm_scale),
                                   _ptr(workspace), ws_bytes, _stream(stream, dev))
    else:
        e0, e1 = (ctypes.c_void_p(e.cuda_event) for e in attn_events)
        _run(dev, lib().sage_attn_fwd_ev, _ptr(q), _strides(q), _ptr(k), _strides(k), _ptr(v), _strides(v),
                                      _ptr(out), _strides(out), B, H, N, d, ctypes.c_float(sm_scale),
                                      _ptr(workspace), ws_bytes, _stream(stream, dev), e0, e1)
    return out


def sage_attn_dense_ref_gpu(q, k, v, sm_scale=None, out=None, stream=None):
    """Dense fp32 CUDA-core attention (A/B reference); returns bf16 [B,H,N,d]."""
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=q.device)
    _run(q.device, lib().sage_attn_dense_ref_gpu, _ptr(q), _strides(q), _ptr(k), _strides(k), _ptr(v), _strides(v),
                                         _ptr(out), _strides(out), B, H, N, d, ctypes.c_float(sm_scale),
                                         _stream(stream, q.device))
    return out


def sage_debug_qk_tile(q_i8, k_i8, N: int, b: int, h: int, q_tile: int, kv_tile: int, stream=None):
    """int32 [128,128] S tile of slab (b,h) computed on the tcgen05 INT8 path."""
    B, H, _, d = q_i8.shape
    s = torch.empty(128, 128, dtype=torch.int32, device=q_i8.device)
    _run(q_i8.device, lib().sage_debug_qk_tile, _ptr(q_i8), _ptr(k_i8), B, H, N, d, b, h, q_tile, kv_tile, _ptr(s),
                                    _stream(stream, q_i8.device))
    return s


LAYOUTS = {"fused": 0, "contiguous": 1}  # SAGE_LAYOUT_FUSED, SAGE_LAYOUT_CONTIGUOUS


def sage_attn_fwd_host_scratch_bytes(B, H, N, d):
    return lib().sage_attn_fwd_host_scratch_bytes(B, H, N, d)


def sage_attn_fwd_host(qkv_host, B, H, N, d, layout="fused", sm_scale=None, device="cuda", out_host=None,
                       workspace=None, stream=None):
    """End-to-end call on HOST memory (the library's sage_attn_fwd_host): the
    bf16 input goes to the device chunk by chunk, the forward runs, and the bf16
    result lands in ``out_host``.

    ``qkv_host`` is one contiguous bf16 host buffer: [B,N,3,H,d] for layout
    "fused", [3,B,H,N,d] for "contiguous" (pinned for asynchronous copies).
    ``workspace``: optional device scratch of sage_attn_fwd_host_scratch_bytes
    bytes.  Returns ``out_host`` ([B,H,N,d]); it is complete once ``stream``
    (default: the current stream of ``device``) reaches the end of the call."""
    if layout not in LAYOUTS:
        raise ValueError(f"layout must be one of {sorted(LAYOUTS)}")
    want = (B, N, 3, H, d) if layout == "fused" else (3, B, H, N, d)
    if qkv_host.device.type != "cpu" or qkv_host.dtype != torch.bfloat16 or not qkv_host.is_contiguous() or \
            tuple(qkv_host.shape) != want:
        raise ValueError(f"qkv_host must be a contiguous bf16 host tensor of shape {want}")
    if out_host is None:
        out_host = torch.empty(B, H, N, d, dtype=torch.bfloat16, pin_memory=True)
    if out_host.device.type != "cpu" or out_host.dtype != torch.bfloat16 or not out_host.is_contiguous() or \
            tuple(out_host.shape) != (B, H, N, d):
        raise ValueError("out_host must be a contiguous bf16 host tensor of shape [B,H,N,d]")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    dev = torch.device(device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    with torch.cuda.device(dev):
        _raise(lib().sage_attn_fwd_host(_ptr(qkv_host), LAYOUTS[layout], _ptr(out_host), B, H, N, d,
                                        ctypes.c_float(sm_scale), _ptr(workspace), ws_bytes, _stream(stream, dev)))
    return out_host


# --------------------------------------------------------------------------
# block-sparse skipping (readings S1-S4 of the sol-attn page's scheduled
# sparsity; the layout of a mask is described in include/sage.h)
# --------------------------------------------------------------------------

TILE = 128  # query / key tile of the block-sparse mask


def n_tiles(N: int) -> int:
    return -(-N // TILE)


def mask_words(N: int) -> int:
    return -(-n_tiles(N) // 32)


def sage_block_mask_bytes(B: int, H: int, N: int) -> int:
    return int(lib().sage_block_mask_bytes(B, H, N))


def sage_attn_sparse_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(lib().sage_attn_sparse_workspace_bytes(B, H, N, d))


def sage_tau_schedule(step: int, n_steps: int, tau_start: float, tau_end: float) -> float:
    return float(lib().sage_tau_schedule(step, n_steps, ctypes.c_float(tau_start), ctypes.c_float(tau_end)))


def keep_to_mask(keep: torch.Tensor) -> torch.Tensor:
    """[B,H,T,T] bool/int (nonzero = query tile i keeps key tile j) -> int32
    mask words [B,H,T,W] in the library's layout (bit j % 32 of word j // 32).
    Argument marshalling only: packs bits, on the tensor's device."""
    B, H, T, T2 = keep.shape
    assert T == T2
    W = -(-T // 32)
    k = torch.zeros(B, H, T, W * 32, dtype=torch.int64, device=keep.device)
    k[..., :T] = (keep != 0).to(torch.int64)
    weights = (torch.ones(32, dtype=torch.int64, device=keep.device) << torch.arange(32, device=keep.device))
    words = (k.view(B, H, T, W, 32) * weights).sum(-1)
    return torch.where(words >= 2 ** 31, words - 2 ** 32, words).to(torch.int32)


def mask_to_keep(mask: torch.Tensor, T: int) -> torch.Tensor:
    """int32 mask words [B,H,T,W] -> bool [B,H,T,T] (the inverse of keep_to_mask)."""
    m = mask.to(torch.int64) & 0xFFFFFFFF
    bits = (m.unsqueeze(-1) >> torch.arange(32, device=mask.device)) & 1
    return bits.flatten(-2)[..., :T].bool()


def sage_block_select(codes, N: int, sm_scale: float, tau: float, want_scores=False, workspace=None, stream=None):
    """Key-tile mask of every query tile from the codes of sage_quant_qk
    (readings S2, S3).  Returns int32 mask words [B,H,T,W] (and the fp32 tile
    scores [B,H,T,T] with want_scores)."""
    q_i8, k_i8 = codes["q_i8"], codes["k_i8"]
    B, H, _, d = q_i8.shape
    dev = q_i8.device
    T, W = n_tiles(N), mask_words(N)
    mask = torch.empty(B, H, T, W, dtype=torch.int32, device=dev)
    scores = torch.empty(B, H, T, T, dtype=torch.float32, device=dev) if want_scores else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _run(dev, lib().sage_block_select, _ptr(q_i8), _ptr(codes["q_scale"]), _ptr(k_i8), _ptr(codes["k_scale"]),
                                   B, H, N, d, ctypes.c_float(sm_scale), ctypes.c_float(tau), _ptr(mask),
                                   _ptr(scores), _ptr(workspace), ws_bytes, _stream(stream, dev))
    return (mask, scores) if want_scores else mask


def sage_attn_fwd_sparse(q, k, v, tau=1.0, sm_scale=None, mask=None, return_mask=False, out=None, workspace=None,
                         stream=None, attn_events=None):
    """Quantized attention forward with block-sparse skipping.  ``mask``:
    optional int32 mask words [B,H,T,W] (then ``tau`` is not used); otherwise
    the library selects with ``tau``.  Returns out (and the mask used, with
    return_mask)."""
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    dev = q.device
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=dev)
    mask_out = None
    if return_mask:
        mask_out = torch.empty(B, H, n_tiles(N), mask_words(N), dtype=torch.int32, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    e0, e1 = (ctypes.c_void_p(e.cuda_event) for e in attn_events) if attn_events is not None else (None, None)
    _run(dev, lib().sage_attn_fwd_sparse, _ptr(q), _strides(q), _ptr(k), _strides(k), _ptr(v), _strides(v),
                                      _ptr(out), _strides(out), B, H, N, d, ctypes.c_float(sm_scale),
                                      ctypes.c_float(tau), _ptr(mask), _ptr(mask_out), _ptr(workspace), ws_bytes,
                                      _stream(stream, dev), e0, e1)
    return (out, mask_out) if return_mask else out


# --------------------------------------------------------------------------
# K-residual quantization (the sol-attn page's item 1; include/sage.h)
# --------------------------------------------------------------------------

def sage_attn_kres_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(lib().sage_attn_kres_workspace_bytes(B, H, N, d))


def sage_quant_k_residual(k, stream=None):
    """Residual codes of K: dict k_i8 [B,H,N_pad,d] int8, k_scale [B,H,N_pad/64]
    fp32, k_bmean [B,H,N_pad/64,d] bf16 bit patterns (int16 tensor)."""
    _check_qkv(k)
    B, H, N, d = k.shape
    dev = k.device
    npd = n_pad(N)
    r = dict(k_i8=torch.empty(B, H, npd, d, dtype=torch.int8, device=dev),
             k_scale=torch.empty(B, H, npd // K_BLOCK, dtype=torch.float32, device=dev),
             k_bmean=torch.empty(B, H, npd // K_BLOCK, d, dtype=torch.int16, device=dev))
    _run(dev, lib().sage_quant_k_residual, _ptr(k), _strides(k), B, H, N, d, _ptr(r["k_i8"]), _ptr(r["k_scale"]),
                                       _ptr(r["k_bmean"]), _stream(stream, dev))
    return r


def sage_attn_fwd_kres(q, k, v, sm_scale=None, out=None, workspace=None, stream=None, attn_events=None):
    """Quantized attention forward with K-residual quantization; returns bf16 [B,H,N,d]."""
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    dev = q.device
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    e0, e1 = (ctypes.c_void_p(e.cuda_event) for e in attn_events) if attn_events is not None else (None, None)
    _run(dev, lib().sage_attn_fwd_kres, _ptr(q), _strides(q), _ptr(k), _strides(k), _ptr(v), _strides(v),
                                    _ptr(out), _strides(out), B, H, N, d, ctypes.c_float(sm_scale),
                                    _ptr(workspace), ws_bytes, _stream(stream, dev), e0, e1)
    return out


def sage_attn_fwd_fused_q(q, k, v, sm_scale=None, out=None, workspace=None, stream=None, attn_events=None):
    """sage_attn_fwd with Q quantized in the attention kernel's prologue (the
    same result bit for bit); returns bf16 [B,H,N,d]."""
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    dev = q.device
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    e0, e1 = (ctypes.c_void_p(e.cuda_event) for e in attn_events) if attn_events is not None else (None, None)
    _run(dev, lib().sage_attn_fwd_fused_q, _ptr(q), _strides(q), _ptr(k), _strides(k), _ptr(v), _strides(v),
                                       _ptr(out), _strides(out), B, H, N, d, ctypes.c_float(sm_scale),
                                       _ptr(workspace), ws_bytes, _stream(stream, dev), e0, e1)
    return out


def sage_debug_wait_timeout(microseconds: int = 10000, stream=None, device=None):
    """Launch the bounded-wait probe (include/sage.h): the next sage_check on
    the stream reports SAGE_ERR_TIMEOUT."""
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    _run(dev, lib().sage_debug_wait_timeout, int(microseconds), _stream(stream, dev))


def sage_debug_ex2_probe(sink, blocks: int, iters: int, stream=None):
    """Launch the exponential-unit throughput probe: ``blocks`` CTAs of 256
    threads, each running eight chains of ``iters`` base-2 exponentials
    (blocks * 256 * iters * 8 in all) into ``sink`` (float32 device tensor of
    at least blocks * 256 elements).  The caller times it."""
    if sink.dtype != torch.float32 or not sink.is_cuda or sink.numel() < blocks * 256:
        raise ValueError("sink must be a float32 CUDA tensor of at least blocks * 256 elements")
    dev = sink.device
    _run(dev, lib().sage_debug_ex2_probe, _ptr(sink), int(blocks), int(iters), _stream(stream, dev))
