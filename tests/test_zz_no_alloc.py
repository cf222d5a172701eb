"""sage_quant_qk_noalloc: the quantize pass for callers that cannot allocate
device memory while they run (a plugin or server path whose device memory is
budgeted up front, or code whose allocator belongs to a host framework).  Its
statistics scratch is a fixed array inside the library; these tests check that
it gives the same outputs as sage_quant_qk, the entry point that takes a
workspace, on two calls in a row (the second call sees the scratch the first
one left behind), and that it rejects shapes whose scratch does not fit.

This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import quantized_attention_qk_b200 as sage
from quantized_attention_qk_b200 import build as sage_build
from quantized_attention_qk_b200.inputs import WORKLOADS, make_qkv, tiny_custom


@pytest.fixture(scope="module")
def L():
    sage_build.build()
    return sage.lib()


def test_noalloc_rejects_a_shape_beyond_its_scratch(L):
    st = (ctypes.c_int64 * 4)(128 * 128 * 128, 128 * 128, 128, 1)
    p = ctypes.c_void_p(16 * 4096)
    # with B*H = 4096 heads the statistics slots need about 7 MB, more than the array
    assert sage.sage_quant_workspace_bytes(32, 128, 128, 128) > 4 << 20
    rc = L.sage_quant_qk_noalloc(p, st, p, st, 32, 128, 128, 128, p, p, p, p, None, None)
    assert rc == 3
    assert b"scratch" in L.sage_last_error_message()


def test_noalloc_scratch_bound_on_the_workloads(L):
    """The scratch a shape needs is the documented formula; every workload
    fits the 4 MiB array, and the largest head count that fits is the one the
    header states (about 2200 heads at d = 128, 4900 at d = 64): one more head
    is rejected with status 3 before any launch."""
    up = lambda x: -(-x // 1024) * 1024

    def need(B, H, N, d):
        S = B * H + min(512, B * H * -(-N // 128))
        return up(8 * S * d) + up(4 * S * d) + up(8 * S)

    for name, w in WORKLOADS.items():
        assert sage.sage_quant_workspace_bytes(w.B, w.H, w.N, w.d) == need(w.B, w.H, w.N, w.d), name
        assert need(w.B, w.H, w.N, w.d) <= 4 << 20, name
    for d, near in ((128, 2200), (64, 4900)):
        fit = max(h for h in range(near - 50, near + 50) if need(1, h, 4096, d) <= 4 << 20)
        assert abs(fit - near) <= 10, (d, fit)
        assert sage.sage_quant_workspace_bytes(1, fit + 1, 4096, d) > 4 << 20
        st = (ctypes.c_int64 * 4)((fit + 1) * 4096 * d, 4096 * d, d, 1)
        p = ctypes.c_void_p(16 * 4096)
        rc = L.sage_quant_qk_noalloc(p, st, p, st, 1, fit + 1, 4096, d, p, p, p, p, None, None)
        assert rc == 3, (d, rc)
        assert b"scratch" in L.sage_last_error_message()
    # a shape the library does not take at all is reported as such, not as scratch
    st = (ctypes.c_int64 * 4)(128 * 70000 * 128, 128 * 128, 128, 1)
    p = ctypes.c_void_p(16 * 4096)
    assert L.sage_quant_qk_noalloc(p, st, p, st, 1, 70000, 128, 128, p, p, p, p, None, None) == 2


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_noalloc_matches_the_workspace_entry_point_twice(L):
    cases = [WORKLOADS["flux"], tiny_custom(2, 3, 1000, 64, seed=901, bias_sigma=3.0, outlier_frac=0.02)]
    for call, w in enumerate(cases):  # two calls in a row, different shapes
        q, k, _, _ = make_qkv(w, device="cuda")
        ref = sage.sage_quant_qk(q, k)
        got = sage.sage_quant_qk_noalloc(q, k)
        torch.cuda.synchronize()
        sage.sage_check()
        for key in ("q_i8", "q_scale", "k_i8", "k_scale", "k_mean"):
            a, b = got[key], ref[key]
            assert a.shape == b.shape, (call, key)
            # the quantize pass is deterministic: the two entry points must agree bit for bit
            assert torch.equal(a.view(torch.uint8) if a.dtype == torch.int8 else a,
                               b.view(torch.uint8) if b.dtype == torch.int8 else b), (call, key)
