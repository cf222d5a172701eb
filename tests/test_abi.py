"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/sage.h declares, sizes its scratch as documented, and
rejects bad arguments before touching a device (only validation paths run)."""
import ctypes
import os
import re

import pytest

import quantized_attention_qk_b200 as sage
from quantized_attention_qk_b200 import build as sage_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    sage_build.build()
    return sage.lib()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "sage.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sage_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("sage_quant_qk", "sage_attn_fwd", "sage_attn_dense_ref_gpu", "sage_debug_qk_tile",
                     "sage_attn_workspace_bytes", "sage_status_string", "sage_last_error_message"):
        assert required in names


def test_library_exports_every_declared_function(L):
    for name in _declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code, name in sage.SAGE_STATUS.items():
        assert L.sage_status_string(code).decode() == name


def test_workspace_sizes(L):
    # codes: 3 * BH * N_pad * d bytes plus scales and statistics
    for (B, H, N, d) in [(1, 2, 256, 64), (1, 24, 4608, 128), (1, 40, 34020, 128)]:
        npd = -(-N // 128) * 128
        ws = sage.sage_attn_workspace_bytes(B, H, N, d)
        assert ws >= 3 * B * H * npd * d
        assert ws <= 3 * B * H * npd * d + 64 * 1024 * 1024
        assert sage.sage_quant_workspace_bytes(B, H, N, d) > 0
    assert sage.sage_attn_workspace_bytes(1, 1, 128, 96) == 0
    assert sage.sage_attn_workspace_bytes(1, 1, 0, 64) == 0
    # every size query answers 0 for the shapes the calls reject (B*H past
    # 65535, N past 2^24), and no size arithmetic runs for them
    for fn in (sage.sage_attn_workspace_bytes, sage.sage_quant_workspace_bytes,
               sage.sage_attn_sparse_workspace_bytes, sage.sage_attn_fwd_host_scratch_bytes):
        assert fn(2, 32768, 128, 64) == 0 and fn(1, 1, (1 << 24) + 1, 64) == 0
        assert fn(65535, 1, 128, 64) > 0 and fn(1, 65535, 128, 64) > 0
        assert fn(46341, 46341, 128, 64) == 0      # B*H past 2^31 too
    L.sage_block_select_workspace_bytes.restype = ctypes.c_size_t
    assert L.sage_block_select_workspace_bytes(2, 32768, 128, 64) == 0
    assert sage.sage_block_mask_bytes(2, 32768, 128) == 0 and sage.sage_block_mask_bytes(1, 65535, 128) > 0


def _call_fwd(L, q=16 * 4096, strides=(8 * 4096, 4096 * 8, 8 * 8, 1), B=1, H=1, N=128, d=64, scale=0.125):
    st = (ctypes.c_int64 * 4)(*strides)
    p = ctypes.c_void_p(q)
    return L.sage_attn_fwd(p, st, p, st, p, st, p, st, B, H, N, d, ctypes.c_float(scale), None, 0, None)


def test_validation_rejects_before_launch(L):
    # every case below fails in argument checking, before any CUDA call
    assert _call_fwd(L, d=96) == 2                       # unsupported head dim
    assert b"d=96" in L.sage_last_error_message()
    assert _call_fwd(L, N=0) == 1
    assert _call_fwd(L, q=0) == 1                          # null pointer
    assert _call_fwd(L, q=16 * 4096 + 2) == 1              # not 16-byte aligned
    assert _call_fwd(L, strides=(8 * 4096, 4096 * 8, 8 * 8, 2)) == 1   # channel stride != 1
    assert _call_fwd(L, strides=(8 * 4096, 4096 * 8, 65, 1)) == 1      # row stride not a multiple of 8
    assert _call_fwd(L, scale=float("nan")) == 1
    assert _call_fwd(L, scale=0.0) == 1
    assert _call_fwd(L, scale=-1.0) == 1


def test_debug_tile_rejects_out_of_range(L):
    p = ctypes.c_void_p(16 * 4096)
    assert L.sage_debug_qk_tile(p, p, 1, 1, 200, 64, 0, 0, 2, 0, p, None) == 1   # q_tile 2 of 2 tiles
    assert L.sage_debug_qk_tile(p, p, 1, 1, 200, 64, 1, 0, 0, 0, p, None) == 1   # b out of range


def test_binding_raises_without_fallback(L):
    with pytest.raises(sage.SageError) as e:
        sage._raise(2)
    assert e.value.status == 2


def test_host_forward_rejects_bad_arguments_before_any_launch(L):
    buf = ctypes.create_string_buffer(4096)
    p = ctypes.cast(buf, ctypes.c_void_p)
    f = L.sage_attn_fwd_host
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    f.restype = ctypes.c_int
    assert f(None, 0, p, 1, 1, 8, 64, 0.125, None, 0, None) == 1          # null input
    assert f(p, 2, p, 1, 1, 8, 64, 0.125, None, 0, None) == 1             # unknown layout
    assert f(p, 0, p, 1, 1, 8, 96, 0.125, None, 0, None) == 2             # head dim
    assert f(p, 1, p, 1, 0, 8, 64, 0.125, None, 0, None) == 1             # shape
    assert f(p, 1, p, 2, 32768, 8, 64, 0.125, None, 0, None) == 2         # B*H past 65535
    assert f(p, 1, p, 1, 1, (1 << 24) + 1, 64, 0.125, None, 0, None) == 2  # N past 2^24
    assert f(p, 1, p, 1, 1, 8, 64, float("nan"), None, 0, None) == 1      # sm_scale
    assert f(p, 1, p, 1, 1, 8, 64, 0.125, p, 16, None) == 3               # scratch too small
    L.sage_attn_fwd_host_scratch_bytes.restype = ctypes.c_size_t
    assert L.sage_attn_fwd_host_scratch_bytes(1, 24, 4608, 128) > 3 * 24 * 4608 * 128 * 2 + 24 * 4608 * 128 * 2
    assert L.sage_attn_fwd_host_scratch_bytes(1, 24, 4608, 96) == 0
    assert L.sage_attn_fwd_host_scratch_bytes(2, 32768, 8, 64) == 0
    assert L.sage_attn_fwd_host_scratch_bytes(1, 1, (1 << 24) + 1, 64) == 0
    assert L.sage_attn_fwd_host_scratch_bytes(1, 65535, 8, 64) > 0


def _call_sparse(L, tau=0.5, N=128, d=64, mask_in=None, mask_out=None, q=16 * 4096):
    st = (ctypes.c_int64 * 4)(8 * 4096, 4096 * 8, 8 * 8, 1)
    p = ctypes.c_void_p(q)
    return L.sage_attn_fwd_sparse(p, st, p, st, p, st, p, st, 1, 1, N, d, ctypes.c_float(0.125), ctypes.c_float(tau),
                                  mask_in, mask_out, None, 0, None, None, None)


def test_sparse_sizes_and_schedule(L):
    # one mask row of ceil(T/32) words per (b,h, query tile)
    for (B, H, N) in [(1, 2, 256), (1, 24, 4608), (1, 40, 34020), (2, 3, 4097)]:
        T = -(-N // 128)
        assert sage.sage_block_mask_bytes(B, H, N) == B * H * T * (-(-T // 32)) * 4
        assert sage.sage_attn_sparse_workspace_bytes(B, H, N, 128) > sage.sage_attn_workspace_bytes(B, H, N, 128)
    assert sage.sage_block_mask_bytes(1, 1, 4096 * 128) > 0
    assert sage.sage_block_mask_bytes(1, 1, 4096 * 128 + 1) == 0
    assert sage.sage_attn_sparse_workspace_bytes(1, 1, 128, 96) == 0
    assert sage.sage_tau_schedule(0, 11, 0.5, 1.0) == 0.5
    assert sage.sage_tau_schedule(10, 11, 0.5, 1.0) == 1.0
    assert sage.sage_tau_schedule(5, 11, 0.5, 1.0) == pytest.approx(0.75, abs=1e-7)
    assert sage.sage_tau_schedule(-4, 11, 0.5, 1.0) == 0.5
    assert sage.sage_tau_schedule(40, 11, 0.5, 1.0) == 1.0
    assert sage.sage_tau_schedule(3, 1, 0.2, 0.9) == pytest.approx(0.9)


def test_sparse_calls_reject_bad_arguments_before_any_launch(L):
    for tau in (0.0, -1.0, float("nan"), float("inf")):
        assert _call_sparse(L, tau=tau) == 1, tau
        assert "tau" in L.sage_last_error_message().decode()
    assert _call_sparse(L, N=4096 * 128 + 1) == 2                       # too many tiles
    assert _call_sparse(L, mask_in=ctypes.c_void_p(4 * 4096 + 2)) == 1  # misaligned mask
    assert _call_sparse(L, mask_out=ctypes.c_void_p(4 * 4096 + 1)) == 1
    assert _call_sparse(L, d=96) == 2
    st = ctypes.c_void_p(16 * 4096)
    assert L.sage_block_select(st, st, st, st, 1, 1, 256, 64, ctypes.c_float(0.125), ctypes.c_float(0.0), st, None,
                               None, 0, None) == 1
    assert L.sage_block_select(st, st, st, st, 1, 1, 256, 64, ctypes.c_float(0.125), ctypes.c_float(0.5), None, None,
                               None, 0, None) == 1                      # null mask
    import torch
    with pytest.raises(ValueError):  # host tensors: refused, never computed elsewhere
        sage.sage_attn_fwd_sparse(*(torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16) for _ in range(3)), tau=0.5)


def test_mask_packing_round_trips():
    import torch
    g = torch.Generator().manual_seed(3)
    for T in (1, 31, 32, 33, 70):
        keep = torch.rand(2, 1, T, T, generator=g) < 0.4
        m = sage.keep_to_mask(keep)
        assert m.shape == (2, 1, T, -(-T // 32)) and m.dtype == torch.int32
        assert torch.equal(sage.mask_to_keep(m, T), keep)
        # bit j of word j // 32
        j = T - 1
        assert bool(((m[0, 0, 0, j // 32].item() & 0xFFFFFFFF) >> (j % 32)) & 1) == bool(keep[0, 0, 0, j])


def test_probes_reject_out_of_range_arguments_before_any_launch(L):
    for us in (0, -5, 1000001):
        assert L.sage_debug_wait_timeout(us, None) == 1
        assert "microseconds" in L.sage_last_error_message().decode()
    p = ctypes.c_void_p(16 * 4096)
    for blocks, iters in ((0, 10), (70000, 10), (1, 0), (1, (1 << 20) + 1)):
        assert L.sage_debug_ex2_probe(p, blocks, iters, None) == 1
    assert L.sage_debug_ex2_probe(None, 1, 1, None) == 1
    assert L.sage_debug_ex2_probe(ctypes.c_void_p(16 * 4096 + 2), 1, 1, None) == 1


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """No library, no result: the binding raises instead of computing anything
    another way."""
    monkeypatch.setattr(sage, "LIB_PATH", str(tmp_path / "libsage.so"))
    monkeypatch.setattr(sage, "_lib", None)
    with pytest.raises(ImportError):
        sage.lib()
    with pytest.raises(ImportError):
        sage.sage_attn_workspace_bytes(1, 1, 128, 64)
