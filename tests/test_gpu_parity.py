"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

  * quantize pass: every code and scale bit-exact (Q, K, V codes, their
    scales and the K mean: the K column sums are exact fp64 sums on both
    sides), on heads of every workload including the full-size ones.
  * S = Q K^T tiles from the tcgen05 INT8 path: bit-exact against the integer
    products of the GPU's own codes (closed form).
  * attention output against the quant-emulation oracle: relative L2 <= 2e-3
    and max |diff| <= 1e-2 (tolerances of the scheme's specification).
  * attention output against exact fp64 attention: within the scheme's own
    error (the oracle's quant-vs-exact gap) plus a small margin.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import quantized_attention_qk_b200 as sage
from quantized_attention_qk_b200.inputs import WORKLOADS, make_qkv, tiny_custom
from tests import _gpu_util as U

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from quantized_attention_qk_b200 import build
    build.build()
    oracle.build()


def _inputs(w):
    """CPU copies for the oracle and device copies of the same bits (the
    device views keep the workload's layout, e.g. the fused qkv strides)."""
    q, k, v, bufs = make_qkv(w)
    dbufs = [b.to(DEV) for b in bufs]
    if w.layout == "fused":
        qd, kd, vd = (dbufs[0][:, :, i].permute(0, 2, 1, 3) for i in range(3))
    else:
        qd, kd, vd = dbufs
    return (q, k, v), (qd, kd, vd), dbufs


def _check_attn(w, heads=None, nrows=None, seed=0):
    (q, k, v), (qd, kd, vd), _ = _inputs(w)
    heads = heads or [(b, h) for b in range(w.B) for h in range(w.H)]
    rows = np.arange(w.N, dtype=np.int32) if nrows is None else U.sample_rows(w.N, nrows, seed)
    out = sage.sage_attn_fwd(qd, kd, vd, sm_scale=w.sm_scale)
    torch.cuda.synchronize()
    sage.sage_check()
    got = U.stack(U.gather(out, heads, rows), heads)
    ref = U.oracle_quant_rows(q, k, v, w.sm_scale, heads, rows)
    want_bf16 = np.stack([ref[x][1] for x in heads])
    ok, rel, mx, nstep = U.within_tol(got, want_bf16, label=w.name)
    assert np.isfinite(got).all()
    assert ok, (w.name, rel, mx, nstep)
    return got, (q, k, v), heads, rows


# --------------------------------------------------------------------------- quantize pass

@pytest.mark.parametrize("name,hs", [("tiny", [0, 1]), ("flux", [0, 11, 23]), ("sdxl", [0, 39]),
                                     ("video", [0, 39]), ("long8k", [5]), ("long64k", [0, 23])])
def test_quant_codes_match_oracle(name, hs):
    """Every code and scale of the quantize pass equals the oracle's bit for
    bit, the K mean included (heads hs, counted over b*H + h)."""
    _check_quant(WORKLOADS[name], hs)


@pytest.mark.parametrize("B,H,N,d", [(8, 64, 100, 64), (2, 300, 130, 128), (1, 3, 20000, 64), (3, 1, 4097, 128)])
def test_quant_codes_match_oracle_on_many_heads_and_ragged_lengths(B, H, N, d):
    """The quantize kernel splits all heads' rows evenly over its CTAs, so
    with many short heads a CTA covers several heads in both of its phases,
    and with few long ones many CTAs share a head's statistics; every head's
    codes and scales must still equal the oracle's bit for bit."""
    w = tiny_custom(B, H, N, d, seed=1201 + N, bias_sigma=2.0, outlier_frac=0.02)
    hs = list(range(B * H)) if B * H <= 8 else [0, 1, B * H // 2, B * H - 2, B * H - 1]
    _check_quant(w, hs)


def _check_quant(w, hs):
    (q, k, v), (qd, kd, vd), _ = _inputs(w)
    r = sage.sage_quant_qk(qd, kd)
    v_e4m3, v_scale = sage.sage_quant_v(vd)
    torch.cuda.synchronize()
    sage.sage_check()
    for bh in hs:
        b, h = divmod(bh, w.H)
        sl = (slice(b, b + 1), slice(h, h + 1))
        o = oracle.quantize(q[sl], k[sl], v[sl])
        _assert_head_codes(r, v_e4m3, v_scale, b, h, w.N, o, f"{w.name} head {bh}")


def _assert_head_codes(r, v_e4m3, v_scale, b, h, N, o, label):
    """Head (b, h) of the quantize pass's outputs against the oracle's codes
    of that head alone (o, from oracle.quantize on [1,1,N,d] inputs): every
    code and scale equal, padded rows and blocks zero."""
    nqb, nkb = -(-N // 128), -(-N // 64)
    for key in ("q_i8", "k_i8"):
        g = r[key][b, h].cpu().numpy()
        np.testing.assert_array_equal(g[:N], o[key][0, 0], err_msg=f"{label} {key}")
        assert (g[N:] == 0).all()
    np.testing.assert_array_equal(r["q_scale"][b, h, :nqb].cpu().numpy(), o["q_scale"][0, 0])
    assert (r["q_scale"][b, h, nqb:] == 0).all()
    np.testing.assert_array_equal(r["k_mean"][b, h].cpu().numpy(), o["k_mean"][0, 0])
    np.testing.assert_array_equal(r["k_scale"][b, h, :nkb].cpu().numpy(), o["k_scale"][0, 0])
    assert (r["k_scale"][b, h, nkb:] == 0).all()
    gv = v_e4m3[b, h].cpu().numpy()          # [N_pad, d]
    np.testing.assert_array_equal(gv[:N], o["v_e4m3"][0, 0])
    assert (gv[N:] == 0).all()
    np.testing.assert_array_equal(v_scale[b, h].cpu().numpy(), o["v_scale"][0, 0])


# --------------------------------------------------------------------------- S tiles

@pytest.mark.parametrize("d,N", [(64, 256), (128, 300), (128, 4608)])
def test_debug_qk_tile_is_exact_integer_product(d, N):
    w = tiny_custom(1, 2, N, d, seed=100 + N, bias_sigma=3.0, outlier_frac=0.02)
    _, (qd, kd, vd), _ = _inputs(w)
    r = sage.sage_quant_qk(qd, kd)
    qi = r["q_i8"].cpu().numpy()
    ki = r["k_i8"].cpu().numpy()
    nt = sage.n_pad(N) // 128
    tiles = {(0, 0), (nt - 1, nt - 1), (0, nt - 1), (nt - 1, 0)}
    for (qt, kt) in sorted(tiles):
        for h in range(2):
            s = sage.sage_debug_qk_tile(r["q_i8"], r["k_i8"], N, 0, h, qt, kt).cpu().numpy()
            want = oracle.int8_gemm_nt(qi[0, h, qt * 128:(qt + 1) * 128], ki[0, h, kt * 128:(kt + 1) * 128])
            np.testing.assert_array_equal(s, want)


# --------------------------------------------------------------------------- attention output

def test_tiny_all_rows():
    _check_attn(WORKLOADS["tiny"])


def test_sdxl_sampled():
    heads = [(0, 0), (0, 9), (1, 3), (1, 7), (2, 4), (2, 5), (3, 0), (3, 9)]
    _check_attn(WORKLOADS["sdxl"], heads=heads, nrows=96)


def test_flux_full_size_sampled():
    _check_attn(WORKLOADS["flux"], heads=[(0, 0), (0, 13), (0, 23)], nrows=96)


def test_video_full_size_sampled():
    _check_attn(WORKLOADS["video"], heads=[(0, 0), (0, 39)], nrows=48)


@pytest.mark.parametrize("name", ["long8k", "long16k", "long64k"])
def test_long_sweep_full_size_sampled(name):
    """The 8K / 16K / 64K-token sweep at full size: two heads, sampled rows
    (first, last, the ragged tail tile and random ones)."""
    _check_attn(WORKLOADS[name], heads=[(0, 0), (0, 23)], nrows=48, seed=len(name))


@pytest.mark.parametrize("N", [1, 17, 63, 64, 65, 127, 128, 129, 255, 383, 1000])
@pytest.mark.parametrize("d", [64, 128])
def test_ragged_and_short_sequences(N, d):
    _check_attn(tiny_custom(1, 1, N, d, seed=7 * N + d, bias_sigma=2.0))


@pytest.mark.parametrize("B,H,N,d", [(1, 65535, 1, 64), (5, 13107, 3, 128)])
def test_the_largest_head_count(B, H, N, d):
    """B*H at its limit (65535 heads, the attention grid's second dimension)
    with very short heads: every CTA of the quantize kernel covers hundreds of
    heads in both of its phases.  Codes, scales and the forward's rows equal
    the oracle's on heads at the start, the middle and the end."""
    w = tiny_custom(B, H, N, d, seed=991 + N, bias_sigma=2.0)
    hs = [0, 1, B * H // 2, B * H - 2, B * H - 1]
    _check_quant(w, hs)
    heads = [divmod(x, H) for x in hs]
    _check_attn(w, heads=heads, nrows=None)


def _wide_inputs(B, H, N, d, layout, P=61, seed=1777):
    """B*H distinct heads without drawing them all on the host: P heads from
    the seeded generator (bias and outlier channels as in the workloads), and
    head x = b*H + h is base head x mod P with its tokens rotated by
    (7919 x) mod N, so that neighbouring heads, and heads 2^31 elements
    apart, hold different rows.  The device tensors are assembled from the
    base heads by an index gather (data movement only).  Returns the device
    q, k, v views in the layout and head(x) -> its (q, k, v) as CPU bf16
    [1,1,N,d], rebuilt from the same base heads."""
    bq, bk, bv, _ = make_qkv(tiny_custom(1, P, N, d, seed=seed, bias_sigma=2.0, outlier_frac=0.02))
    BH = B * H

    def head(x):
        p, r = x % P, (7919 * x) % N
        return tuple(t[0, p].roll(-r, dims=0).contiguous().view(1, 1, N, d) for t in (bq, bk, bv))

    x = torch.arange(BH, device=DEV)
    rows = (torch.arange(N, device=DEV).view(1, N) + ((7919 * x) % N).view(BH, 1)) % N
    pidx = (x % P).view(BH, 1)
    if layout == "fused":
        buf = torch.empty(B, N, 3, H, d, dtype=torch.bfloat16, device=DEV)
        views = tuple(buf[:, :, i].permute(0, 2, 1, 3) for i in range(3))
    else:
        views = tuple(torch.empty(B, H, N, d, dtype=torch.bfloat16, device=DEV) for _ in range(3))
    for t, dst in zip((bq, bk, bv), views):
        dst.copy_(t[0].to(DEV)[pidx, rows].view(B, H, N, d))
    return views, head


@pytest.mark.parametrize("layout", ["contiguous", "fused"])
def test_tensors_past_2_31_elements(layout):
    """65535 heads of 300 tokens (B=3, H=21845, d=128): the inputs and the
    output hold 2.5e9 elements and the codes 3.2e9, so element offsets pass
    2^31 (and byte offsets of the bf16 tensors 2^32); in the fused layout a
    token's stride alone is 8.4 M elements and rows of the first batch cross
    2^31.  Codes and scales equal the oracle's bit for bit, the forward and
    the K-residual forward are within the parity bar, on heads at the start,
    astride the 2^31-byte, 2^31-code and 2^31-input-element boundaries, and
    at the end."""
    B, H, N, d = 3, 21845, 300, 128
    sm_scale = 1.0 / math.sqrt(d)
    (qd, kd, vd), head = _wide_inputs(B, H, N, d, layout)
    assert qd.numel() > 2 ** 31 and B * H * sage.n_pad(N) * d > 2 ** 31
    xs = [0, 1, 27962, 43690, 55924, B * H - 2, B * H - 1]
    cpu = {x: head(x) for x in xs}
    for x in xs:  # the device copies hold the same bits as the oracle's inputs
        b, h = divmod(x, H)
        for dv, cv in zip((qd, kd, vd), cpu[x]):
            assert torch.equal(dv[b, h].cpu(), cv[0, 0])
    r = sage.sage_quant_qk(qd, kd)
    v_e4m3, v_scale = sage.sage_quant_v(vd)
    torch.cuda.synchronize()
    sage.sage_check()
    for x in xs:
        b, h = divmod(x, H)
        _assert_head_codes(r, v_e4m3, v_scale, b, h, N, oracle.quantize(*cpu[x]), f"{layout} head {x}")
    del r, v_e4m3, v_scale
    for kres in (False, True):
        fwd = sage.sage_attn_fwd_kres if kres else sage.sage_attn_fwd
        out = fwd(qd, kd, vd, sm_scale=sm_scale)
        torch.cuda.synchronize()
        sage.sage_check()
        for x in xs:
            b, h = divmod(x, H)
            got = U.bf16_to_f64(out[b, h])
            _, bits = oracle.attn_quant(*cpu[x], sm_scale, k_residual=kres)
            label = f"{layout} {'K-residual ' if kres else ''}head {x}"
            ok, rel, mx, nstep = U.within_tol(got, oracle.bf16_bits_to_f64(bits[0, 0]), label=label)
            assert np.isfinite(got).all()
            assert ok, (label, rel, mx, nstep)
        del out
    del qd, kd, vd
    torch.cuda.empty_cache()


def test_batched_heads_d64():
    _check_attn(tiny_custom(3, 2, 200, 64, seed=77, bias_sigma=1.0), nrows=None)


def test_growing_scores_exercise_the_rescale():
    """Keys whose scores grow along the sequence: the running max moves at
    almost every step, so O and l are rescaled many times."""
    N, d = 1024, 128
    g = torch.Generator().manual_seed(9)
    q = torch.randn(1, 1, N, d, generator=g)
    k = torch.randn(1, 1, N, d, generator=g) * torch.linspace(0.2, 4.0, N).view(1, 1, N, 1)
    v = torch.randn(1, 1, N, d, generator=g)
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    out = sage.sage_attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV))
    torch.cuda.synchronize()
    rows = np.arange(N, dtype=np.int32)
    ref = U.oracle_quant_rows(q, k, v, 1 / math.sqrt(d), [(0, 0)], rows)[(0, 0)][1]
    ok, rel, mx, nstep = U.within_tol(U.bf16_to_f64(out[0, 0]), ref, label="growing scores")
    assert ok, (rel, mx, nstep)


def test_zero_query_gives_mean_of_quantized_v():
    N, d = 300, 64
    g = torch.Generator().manual_seed(10)
    q = torch.zeros(1, 1, N, d, dtype=torch.bfloat16)
    k = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    out = sage.sage_attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV))
    torch.cuda.synchronize()
    ref = U.oracle_quant_rows(q, k, v, 0.125, [(0, 0)], np.arange(N, dtype=np.int32))[(0, 0)][1]
    ok, rel, mx, nstep = U.within_tol(U.bf16_to_f64(out[0, 0]), ref, label="zero query")
    assert ok, (rel, mx, nstep)
    # every row is the same (uniform softmax)
    assert (out[0, 0] == out[0, 0, :1]).all()


def _one_head_against_oracle(q, k, v, sm_scale, label, kres=False):
    """The forward (or the K-residual forward) on one [1,1,N,d] head against
    the oracle's quant emulation on all rows; returns (GPU output, oracle
    output) as float64 [N,d]."""
    fwd = sage.sage_attn_fwd_kres if kres else sage.sage_attn_fwd
    out = fwd(q.to(DEV), k.to(DEV), v.to(DEV), sm_scale=sm_scale)
    torch.cuda.synchronize()
    sage.sage_check()
    got = U.bf16_to_f64(out[0, 0])
    _, bits = oracle.attn_quant(q, k, v, sm_scale, k_residual=kres)
    want = oracle.bf16_bits_to_f64(bits[0, 0])
    ok, rel, mx, nstep = U.within_tol(got, want, label=label)
    assert np.isfinite(got).all()
    assert ok, (label, rel, mx, nstep)
    return got, want


@pytest.mark.parametrize("kres", [False, True], ids=["smoothing", "k_residual"])
def test_scores_far_below_the_row_max_get_no_weight(kres):
    """Hard attention: channel 0 of the keys is +1 or -1 at random and the
    queries point along it, so half of the keys score about 140 (in log2
    units) below the others.  Their exponent offsets fall far below the range
    where the FMA-pipe exponential clamps its input (and the MUFU flushes to
    zero), in both kinds of lanes: they must get no weight, and every row is
    a weighted mean of the top keys' V rows, as in the oracle (also with
    K-residual quantization, where the block means carry much of the score)."""
    N, d = 1000, 128
    g = torch.Generator().manual_seed(21)
    top = torch.rand(N, generator=g) < 0.5
    q = 0.05 * torch.randn(1, 1, N, d, generator=g)
    q[..., 0] = 4.0
    k = 0.05 * torch.randn(1, 1, N, d, generator=g)
    k[0, 0, :, 0] = torch.where(top, 1.0, -1.0)
    v = torch.randn(1, 1, N, d, generator=g)
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    got, want = _one_head_against_oracle(q, k, v, 12.0, "scores far below the max", kres=kres)
    # the bottom keys carry nothing: the oracle's rows lie in the span of the
    # top keys' values (their mean, within the spread of the top weights)
    vt = U.bf16_to_f64(v[0, 0])[top.numpy()]
    assert np.abs(want - vt.mean(axis=0)).max() < 0.25


def test_identical_keys_give_uniform_weights():
    """Every key the same row: the smoothed keys are exactly zero, so are the K
    codes and scales, every score is 0 and every row is the mean of the
    quantized V rows."""
    N, d = 700, 64
    g = torch.Generator().manual_seed(22)
    q = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    k = (3.0 * torch.randn(1, 1, 1, d, generator=g)).expand(1, 1, N, d).contiguous().to(torch.bfloat16)
    v = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    got, _ = _one_head_against_oracle(q, k, v, 1 / math.sqrt(d), "identical keys")
    assert (got == got[:1]).all()


def test_zero_values_give_a_zero_output():
    N, d = 333, 128
    g = torch.Generator().manual_seed(23)
    q = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    v = torch.zeros(1, 1, N, d, dtype=torch.bfloat16)
    got, want = _one_head_against_oracle(q, k, v, 1 / math.sqrt(d), "zero values")
    assert (got == 0).all() and (want == 0).all()


def test_a_tiny_softmax_scale_gives_near_uniform_weights():
    N, d = 500, 128
    g = torch.Generator().manual_seed(24)
    q, k, v = (torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
    _one_head_against_oracle(q, k, v, 1e-6, "tiny softmax scale")


def test_attention_kernel_on_oracle_codes():
    """Feed the oracle's own codes and scales to the attention kernel alone: this
    isolates the tcgen05 attention from the quantize pass."""
    w = tiny_custom(1, 2, 700, 128, seed=55, bias_sigma=4.0, outlier_frac=0.02)
    (q, k, v), _, _ = _inputs(w)
    o = oracle.quantize(q, k, v)
    N, npd = w.N, sage.n_pad(w.N)

    def pad_rows(a, n):
        z = np.zeros(a.shape[:2] + (n,) + a.shape[3:], dtype=a.dtype)
        z[:, :, :a.shape[2]] = a
        return z

    q_i8 = torch.from_numpy(pad_rows(o["q_i8"], npd)).to(DEV)
    k_i8 = torch.from_numpy(pad_rows(o["k_i8"], npd)).to(DEV)
    v_e4m3 = torch.from_numpy(pad_rows(o["v_e4m3"], npd)).to(DEV)
    qs = np.zeros((1, 2, npd // 128), np.float32); qs[..., :o["q_scale"].shape[-1]] = o["q_scale"]
    ks = np.zeros((1, 2, npd // 64), np.float32); ks[..., :o["k_scale"].shape[-1]] = o["k_scale"]
    out = sage.sage_attn_quantized(q_i8, torch.from_numpy(qs).to(DEV), k_i8, torch.from_numpy(ks).to(DEV),
                                   v_e4m3, torch.from_numpy(o["v_scale"]).to(DEV), N, w.sm_scale)
    torch.cuda.synchronize()
    rows = np.arange(N, dtype=np.int32)
    ref = U.oracle_quant_rows(q, k, v, w.sm_scale, [(0, 0), (0, 1)], rows)
    got = U.stack(U.gather(out, [(0, 0), (0, 1)], rows), [(0, 0), (0, 1)])
    want = np.stack([ref[(0, 0)][1], ref[(0, 1)][1]])
    ok, rel, mx, nstep = U.within_tol(got, want, rel_tol=1e-3, label="attention on oracle codes")
    assert ok, (rel, mx, nstep)


def test_fused_and_contiguous_layouts_give_identical_bits():
    w = tiny_custom(1, 3, 500, 128, seed=31, layout="fused", bias_sigma=4.0, outlier_frac=0.01)
    _, (qd, kd, vd), _ = _inputs(w)
    out_f = sage.sage_attn_fwd(qd, kd, vd)
    out_c = sage.sage_attn_fwd(qd.contiguous(), kd.contiguous(), vd.contiguous())
    torch.cuda.synchronize()
    assert torch.equal(out_f.view(torch.int16), out_c.view(torch.int16))


@pytest.mark.parametrize("N,d,layout", [(4608, 128, "fused"), (1000, 128, "contiguous"), (200, 64, "contiguous"),
                                         (777, 64, "fused"), (129, 128, "fused"), (1, 64, "contiguous")])
def test_forward_matches_the_explicit_quantize_then_attention_path(N, d, layout):
    """sage_attn_fwd against its own steps called one by one through the C ABI
    (sage_quant_qk, sage_quant_v, sage_attn_quantized): the same bits."""
    w = tiny_custom(1, 3, N, d, seed=40 + N, layout=layout, bias_sigma=4.0, outlier_frac=0.01)
    _, (qd, kd, vd), _ = _inputs(w)
    fused = sage.sage_attn_fwd(qd, kd, vd, sm_scale=w.sm_scale)
    c = sage.sage_quant_qk(qd, kd)
    v_e4m3, v_scale = sage.sage_quant_v(vd)
    explicit = sage.sage_attn_quantized(c["q_i8"], c["q_scale"], c["k_i8"], c["k_scale"], v_e4m3, v_scale, N,
                                        sm_scale=w.sm_scale)
    torch.cuda.synchronize()
    sage.sage_check()
    assert torch.equal(fused.view(torch.int16), explicit.view(torch.int16))


@pytest.mark.parametrize("B,H,N,d,layout,pinned", [(1, 24, 1000, 128, "fused", True), (2, 5, 777, 64, "contiguous", True),
                                                   (2, 3, 300, 128, "fused", False), (1, 1, 129, 64, "fused", True)])
def test_host_memory_forward_matches_the_device_forward(B, H, N, d, layout, pinned):
    """sage_attn_fwd_host (head chunks on three streams, host<->device copies
    inside) gives the device forward's bits."""
    w = tiny_custom(B, H, N, d, seed=70 + N, layout=layout, bias_sigma=4.0, outlier_frac=0.01)
    _, (qd, kd, vd), bufs = _inputs(w)
    want = sage.sage_attn_fwd(qd, kd, vd, sm_scale=w.sm_scale)
    host_in = (bufs[0] if layout == "fused" else torch.stack(bufs)).cpu()
    if pinned:
        host_in = host_in.pin_memory()
    got = sage.sage_attn_fwd_host(host_in, B, H, N, d, layout=layout, sm_scale=w.sm_scale, device=DEV)
    torch.cuda.synchronize()
    sage.sage_check()
    assert torch.equal(got.view(torch.int16), want.cpu().view(torch.int16))
    small = torch.empty(64, dtype=torch.uint8, device=DEV)
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_fwd_host(host_in, B, H, N, d, layout=layout, sm_scale=w.sm_scale, device=DEV, workspace=small)
    assert e.value.status == 3


@pytest.mark.parametrize("world", [2, 3])
def test_head_shares_reproduce_the_whole_forward(world):
    """Each rank's head share (as sharded_forward computes it, on strided
    views) equals the whole forward's heads bit for bit: the shares of a
    head-sharded run need no communication but the final gather."""
    from types import SimpleNamespace
    from quantized_attention_qk_b200.replicas import head_range, sharded_forward
    w = tiny_custom(2, 5, 700, 128, seed=81, layout="fused", bias_sigma=4.0, outlier_frac=0.01)
    _, (qd, kd, vd), _ = _inputs(w)
    whole = sage.sage_attn_fwd(qd, kd, vd, sm_scale=w.sm_scale)
    for r in range(world):
        part = sharded_forward(qd, kd, vd, SimpleNamespace(world=world, rank=r), sm_scale=w.sm_scale, gather=False)
        h0, h1 = head_range(5, world, r)
        torch.cuda.synchronize()
        assert torch.equal(part.view(torch.int16), whole[:, h0:h1].view(torch.int16))


def test_strided_output_and_explicit_workspace():
    w = tiny_custom(2, 2, 333, 64, seed=32, bias_sigma=2.0)
    _, (qd, kd, vd), _ = _inputs(w)
    ref = sage.sage_attn_fwd(qd, kd, vd)
    ws = torch.empty(sage.sage_attn_workspace_bytes(2, 2, 333, 64), dtype=torch.uint8, device=DEV)
    big = torch.zeros(2, 333, 2, 64, dtype=torch.bfloat16, device=DEV)      # [B,N,H,d] storage
    out = big.permute(0, 2, 1, 3)
    sage.sage_attn_fwd(qd, kd, vd, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(out.contiguous().view(torch.int16), ref.view(torch.int16))
    small = torch.empty(100, dtype=torch.uint8, device=DEV)
    with pytest.raises(sage.SageError) as e:
        sage.sage_attn_fwd(qd, kd, vd, workspace=small)
    assert e.value.status == 3


def test_repeat_calls_are_deterministic():
    w = WORKLOADS["tiny"]
    _, (qd, kd, vd), _ = _inputs(w)
    a = sage.sage_attn_fwd(qd, kd, vd)
    b = sage.sage_attn_fwd(qd, kd, vd)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_back_to_back_forwards_sharing_a_workspace_do_not_interfere():
    """The kernels after the first of a forward may start before their
    predecessor ends (programmatic dependent launch); the first kernel of a
    forward may not, so the next forward cannot overwrite the codes the previous
    forward's attention kernel still reads.  Several forwards of different
    inputs go out back to back on one stream into one workspace, with no
    synchronisation between them; each output must equal its own forward run
    alone, bit for bit."""
    ws_ = [tiny_custom(1, 24, 4608, 128, seed=70 + i, layout="fused", bias_sigma=2.0) for i in range(3)]
    ins = [_inputs(w)[1] for w in ws_]
    alone = []
    for (qd, kd, vd) in ins:
        alone.append(sage.sage_attn_fwd(qd, kd, vd))
        torch.cuda.synchronize()
    ws = torch.empty(sage.sage_attn_workspace_bytes(1, 24, 4608, 128), dtype=torch.uint8, device=DEV)
    outs = [torch.empty(1, 24, 4608, 128, dtype=torch.bfloat16, device=DEV) for _ in ins]
    for rep in range(3):
        for (qd, kd, vd), o in zip(ins, outs):
            sage.sage_attn_fwd(qd, kd, vd, out=o, workspace=ws)
    torch.cuda.synchronize()
    sage.sage_check()
    for a, o in zip(alone, outs):
        assert torch.equal(a.view(torch.int16), o.view(torch.int16))


@pytest.mark.parametrize("B,H,N,d,layout", [(1, 24, 4608, 128, "fused"), (1, 2, 16384, 128, "contiguous"),
                                             (2, 5, 1000, 64, "contiguous")])
def test_quantize_pass_ignores_what_the_workspace_held(B, H, N, d, layout):
    """The quantize kernel's CTAs publish their statistics through flags in the
    workspace, stamped per call; whatever the workspace held before (zeros,
    all ones, random bytes, or the leftovers of another shape's call) must not
    change a bit of the result.  (1, 2, 16384) puts ~74 CTAs on each head, so
    every flag has many readers."""
    w = tiny_custom(B, H, N, d, seed=811, layout=layout, bias_sigma=2.0, outlier_frac=0.02)
    _, (qd, kd, vd), _ = _inputs(w)
    ref = sage.sage_attn_fwd(qd, kd, vd)
    ref_q = sage.sage_quant_qk(qd, kd)
    torch.cuda.synchronize()
    nbytes = sage.sage_attn_workspace_bytes(B, H, N, d)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(5)
    other = tiny_custom(1, 3, 700, d, seed=812)
    _, (qo, ko, vo), _ = _inputs(other)
    fills = [lambda: ws.fill_(0), lambda: ws.fill_(255),
             lambda: ws.copy_(torch.randint(0, 256, (nbytes,), dtype=torch.uint8, device=DEV, generator=g)),
             lambda: sage.sage_attn_fwd(qo, ko, vo, workspace=ws)]
    for fill in fills:
        fill()
        out = sage.sage_attn_fwd(qd, kd, vd, workspace=ws)
        qws = torch.empty(sage.sage_quant_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=DEV)
        qws.fill_(255)
        got_q = sage.sage_quant_qk(qd, kd, workspace=qws)
        torch.cuda.synchronize()
        sage.sage_check()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
        for key in ("q_i8", "q_scale", "k_i8", "k_scale", "k_mean"):
            assert torch.equal(got_q[key], ref_q[key]), key


def test_forward_replays_from_a_cuda_graph():
    """A captured forward replays the same kernel arguments, so the quantize
    kernel's per-call stamp repeats; its flags are cleared by their last
    reader within each launch, so every replay waits for its own statistics.
    Three inputs are copied into the captured buffers in turn; each replay
    must equal the eager forward of the same input bit for bit."""
    ws_ = [tiny_custom(1, 24, 4608, 128, seed=90 + i, layout="contiguous", bias_sigma=2.0) for i in range(3)]
    ins = [_inputs(w)[1] for w in ws_]
    eager = []
    for (qd, kd, vd) in ins:
        eager.append(sage.sage_attn_fwd(qd, kd, vd))
    q, k, v = (t.clone() for t in ins[0])
    out = torch.empty_like(eager[0])
    ws = torch.empty(sage.sage_attn_workspace_bytes(1, 24, 4608, 128), dtype=torch.uint8, device=DEV)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up on the capture stream (first-call set-up outside the capture)
        sage.sage_attn_fwd(q, k, v, out=out, workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        sage.sage_attn_fwd(q, k, v, out=out, workspace=ws)
    for rep in range(2):
        for (qd, kd, vd), want in zip(ins, eager):
            q.copy_(qd)
            k.copy_(kd)
            v.copy_(vd)
            graph.replay()
            torch.cuda.synchronize()
            sage.sage_check()
            assert torch.equal(out.view(torch.int16), want.view(torch.int16)), rep
    del graph


# --------------------------------------------------------------------------- dense reference and exact

@pytest.mark.parametrize("name", ["tiny", "sdxl"])
def test_dense_ref_against_exact(name):
    w = WORKLOADS[name]
    (q, k, v), (qd, kd, vd), _ = _inputs(w)
    out = sage.sage_attn_dense_ref_gpu(qd, kd, vd, sm_scale=w.sm_scale)
    torch.cuda.synchronize()
    heads = [(0, 0), (w.B - 1, w.H - 1)]
    rows = U.sample_rows(w.N, 64, 3)
    ex = U.oracle_exact_rows(q, k, v, w.sm_scale, heads, rows)
    got = U.stack(U.gather(out, heads, rows), heads)
    want = U.stack(ex, heads)
    want_bf16 = oracle.bf16_bits_to_f64(oracle.bf16_rne(want)).reshape(want.shape)
    # only bf16 rounding separates them: at most one bf16 step apart, rarely even that
    step = np.abs(want_bf16) * 2.0 ** -7 + 1e-30
    assert np.all(np.abs(got - want_bf16) <= step * 1.01)
    assert np.mean(got != want_bf16) < 0.02
    rel, _ = U.compare(got, want)
    assert rel < 3e-3


def test_quantized_against_exact_is_the_schemes_own_error():
    w = WORKLOADS["flux"]
    got, (q, k, v), heads, rows = _check_attn(w, heads=[(0, 5)], nrows=64, seed=4)
    ex = U.stack(U.oracle_exact_rows(q, k, v, w.sm_scale, heads, rows), heads)
    emu = np.stack([U.oracle_quant_rows(q, k, v, w.sm_scale, heads, rows)[x][1] for x in heads])
    gpu_err, _ = U.compare(got, ex)
    emu_err, _ = U.compare(emu, ex)
    assert gpu_err <= 1.05 * emu_err + 1e-3, (gpu_err, emu_err)


def test_device_error_word_is_clear():
    sage.sage_check()


@pytest.mark.parametrize("w", [
    WORKLOADS["tiny"],
    tiny_custom(1, 2, 300, 64, 701, layout="fused", bias_sigma=2.0),
    tiny_custom(2, 3, 777, 128, 702, bias_sigma=4.0, outlier_frac=0.01),
    tiny_custom(1, 1, 50, 128, 703, layout="fused"),
    tiny_custom(1, 2, 1, 64, 704),
    WORKLOADS["flux"],
], ids=lambda w: w.name)
def test_prologue_q_quantization_forward_is_bit_identical(w):
    """sage_attn_fwd_fused_q (Q coded inside the attention kernel) against the
    forward with the quantize pass coding Q: the same codes, so the same bits."""
    _, (qd, kd, vd), _ = _inputs(w)
    ref = sage.sage_attn_fwd(qd, kd, vd, sm_scale=w.sm_scale)
    got = sage.sage_attn_fwd_fused_q(qd, kd, vd, sm_scale=w.sm_scale)
    torch.cuda.synchronize()
    sage.sage_check()
    assert torch.equal(got, ref)
