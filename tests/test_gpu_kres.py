"""GPU parity of K-residual quantization ("ComfyUI-sol-attn", 核心亮点 item 1)
through the C ABI.

* residual codes, block scales and bf16 block means bit for bit against the
  oracle (the same arithmetic: exact fp64 block sums, bf16 RNE means, fp32
  residuals, the int8 rule of reading C2);
* the whole forward (mean term on the tensor cores, added to every score of
  its block) against the oracle's K-residual quant emulation, within the
  scheme's tolerances (relative L2 <= 2e-3, max |diff| <= 1e-2), on ragged,
  fused-layout, outlier and multi-batch cases, and on sampled rows of flux;
* its error against exact attention on flux, next to the smoothing scheme's.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_attention_qk_b200 as sage
from quantized_attention_qk_b200.inputs import WORKLOADS, make_qkv, tiny_custom
from tests import _gpu_util as U

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"

CASES = [
    tiny_custom(1, 2, 300, 64, 601, bias_sigma=2.0),
    tiny_custom(1, 2, 777, 128, 602, layout="fused", bias_sigma=4.0, outlier_frac=0.01),
    tiny_custom(2, 3, 200, 128, 603, bias_sigma=4.0, outlier_frac=0.02),
    tiny_custom(1, 1, 50, 64, 604),
    tiny_custom(1, 2, 1, 64, 605, bias_sigma=1.0),
    WORKLOADS["tiny"],
]


@pytest.fixture(scope="module", autouse=True)
def _built():
    from quantized_attention_qk_b200 import build
    build.build()
    oracle.build()


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_residual_codes_match_the_oracle(w):
    q, k, v, _ = make_qkv(w)
    kd = make_qkv(w, device=DEV)[1]
    got = sage.sage_quant_k_residual(kd)
    torch.cuda.synchronize()
    sage.sage_check()
    want = oracle.quantize_kres(k)
    nkb = -(-w.N // 64)
    assert np.array_equal(got["k_bmean"][:, :, :nkb].cpu().numpy().view(np.uint16), want["k_bmean"])
    assert np.array_equal(got["k_scale"][:, :, :nkb].cpu().numpy(), want["k_scale"])
    assert np.array_equal(got["k_i8"][:, :, :w.N].cpu().numpy(), want["k_i8"])
    assert torch.count_nonzero(got["k_i8"][:, :, w.N:]).item() == 0      # padded rows
    assert torch.count_nonzero(got["k_scale"][:, :, nkb:]).item() == 0   # padded blocks


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_forward_matches_the_k_residual_oracle(w):
    q, k, v, _ = make_qkv(w)
    qd, kd, vd, _ = make_qkv(w, device=DEV)
    out = sage.sage_attn_fwd_kres(qd, kd, vd, sm_scale=w.sm_scale)
    torch.cuda.synchronize()
    sage.sage_check()
    got = U.bf16_to_f64(out)
    _, bits = oracle.attn_quant(q, k, v, w.sm_scale, k_residual=True)
    want = oracle.bf16_bits_to_f64(bits)
    ok, rel, mx, nstep = U.within_tol(got, want, label="K-residual " + w.name)
    assert np.isfinite(got).all()
    assert ok, (w.name, rel, mx, nstep)


def test_flux_sampled_rows_and_error_against_exact():
    w = WORKLOADS["flux"]
    q, k, v, _ = make_qkv(w)
    qd, kd, vd, _ = make_qkv(w, device=DEV)
    out_k = sage.sage_attn_fwd_kres(qd, kd, vd, sm_scale=w.sm_scale)
    out_s = sage.sage_attn_fwd(qd, kd, vd, sm_scale=w.sm_scale)
    torch.cuda.synchronize()
    sage.sage_check()
    heads = [(0, 0), (0, 11), (0, 23)]
    rows = U.sample_rows(w.N, 40, 11)
    got = U.stack(U.gather(out_k, heads, rows), heads)
    want = []
    for (b, h) in heads:
        sl = (slice(b, b + 1), slice(h, h + 1))
        _, bits = oracle.attn_quant(q[sl], k[sl], v[sl], w.sm_scale, rows=rows, k_residual=True)
        want.append(oracle.bf16_bits_to_f64(bits[0, 0]))
    ok, rel, mx, nstep = U.within_tol(got, np.stack(want), label="K-residual flux")
    assert ok, (rel, mx, nstep)
    exact = U.stack(U.oracle_exact_rows(q, k, v, w.sm_scale, heads, rows), heads)
    err_k = U.compare(got, exact)[0]
    err_s = U.compare(U.stack(U.gather(out_s, heads, rows), heads), exact)[0]
    # both schemes sit at their intrinsic error (about 0.05 on this workload)
    assert err_k < 0.08 and err_s < 0.08, (err_k, err_s)
    print(f"flux vs exact: K-residual {err_k:.4f}, smoothing {err_s:.4f}")


@pytest.mark.parametrize("name,heads", [("video", [(0, 0), (0, 39)]), ("long64k", [(0, 5)])])
def test_long_sequences_sampled_rows(name, heads):
    """Sequences whose K blocks fill more than one of the attention prologue's
    chunks of 256 block means (video: 532 blocks, three chunks; 65K tokens:
    1024 blocks, four chunks) against the oracle's K-residual emulation on
    sampled rows (first, last, tail and random)."""
    w = WORKLOADS[name]
    assert -(-w.N // 64) > 256
    q, k, v, _ = make_qkv(w)
    qd, kd, vd, _ = make_qkv(w, device=DEV)
    out = sage.sage_attn_fwd_kres(qd, kd, vd, sm_scale=w.sm_scale)
    torch.cuda.synchronize()
    sage.sage_check()
    rows = U.sample_rows(w.N, 24, 13)
    got = U.stack(U.gather(out, heads, rows), heads)
    want = []
    for (b, h) in heads:
        sl = (slice(b, b + 1), slice(h, h + 1))
        _, bits = oracle.attn_quant(q[sl], k[sl], v[sl], w.sm_scale, rows=rows, k_residual=True)
        want.append(oracle.bf16_bits_to_f64(bits[0, 0]))
    ok, rel, mx, nstep = U.within_tol(got, np.stack(want), label="K-residual " + name)
    assert np.isfinite(got).all()
    assert ok, (name, rel, mx, nstep)
