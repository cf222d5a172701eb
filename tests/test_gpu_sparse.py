"""GPU parity of block-sparse skipping (readings S1-S4 of the sol-attn page's
scheduled sparsity) through the C ABI.

* every key tile kept (tau = 1, or an all-ones mask): bit for bit the dense
  forward;
* a mask the test draws (seeded; rows that keep nothing, only the ragged tail
  tile, everything; the two query tiles of a CTA with disjoint masks): the
  output against the oracle's masked quant emulation with that same mask,
  within the scheme's tolerances (relative L2 <= 2e-3, max |diff| <= 1e-2);
* the GPU's tile scores and kept sets against the oracle's on the same codes:
  equal bit for bit (readings S2 and S3 fix every fp32 operation);
* the full flux workload with a drawn mask on sampled heads and rows.
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
T = 128


@pytest.fixture(scope="module", autouse=True)
def _built():
    from quantized_attention_qk_b200 import build
    build.build()
    oracle.build()


def _inputs(w, planted=False):
    q, k, v, _ = make_qkv(w)
    if planted:
        q, k = _plant(q, k, w.seed)
    return (q, k, v), tuple(t.to(DEV) for t in (q, k, v))


def _plant(q, k, seed):
    """Give each query / key tile its own offset vector so that tile scores
    differ (iid inputs make every tile pair look alike)."""
    B, H, N, d = q.shape
    nt = -(-N // T)
    g = torch.Generator().manual_seed(seed + 99)
    uq = torch.randn(B, H, nt, d, generator=g) * 0.6
    uk = torch.randn(B, H, nt, d, generator=g) * 0.6
    q = q.float() + uq.repeat_interleave(T, dim=2)[:, :, :N]
    k = k.float() + uk.repeat_interleave(T, dim=2)[:, :, :N]
    return q.to(torch.bfloat16), k.to(torch.bfloat16)


def _draw_keep(B, H, N, seed, density=0.5):
    nt = -(-N // T)
    rng = np.random.default_rng(seed)
    keep = (rng.random((B, H, nt, nt)) < density).astype(np.uint8)
    keep[..., 0, :] = 0                       # a query tile that keeps nothing
    if nt > 1:
        keep[..., 1, :] = 0
        keep[..., 1, nt - 1] = 1              # one that keeps only the ragged tail tile
    if nt > 2:
        keep[..., 2, :] = 1                   # one that keeps everything
    if nt > 4:                                # CTA of tiles 4, 5: disjoint rows
        keep[..., 4, :] = 0
        keep[..., 4, ::2] = 1
        keep[..., 5, :] = 0
        keep[..., 5, 1::2] = 1
    return keep


def _run_masked(dev_qkv, w, keep):
    mask = sage.keep_to_mask(torch.from_numpy(keep).to(DEV))
    out, used = sage.sage_attn_fwd_sparse(*dev_qkv, sm_scale=w.sm_scale, mask=mask, return_mask=True)
    torch.cuda.synchronize()
    sage.sage_check()
    assert torch.equal(used, mask)
    return out


@pytest.mark.parametrize("w", [
    tiny_custom(1, 2, 300, 64, 501, bias_sigma=2.0),
    tiny_custom(2, 1, 520, 128, 502, layout="fused", bias_sigma=4.0, outlier_frac=0.01),
    WORKLOADS["tiny"],
], ids=lambda w: w.name)
def test_every_tile_kept_is_the_dense_forward_bit_for_bit(w):
    _, dev = _inputs(w)
    dense = sage.sage_attn_fwd(*dev, sm_scale=w.sm_scale)
    sp = sage.sage_attn_fwd_sparse(*dev, tau=1.0, sm_scale=w.sm_scale)
    nt = -(-w.N // T)
    ones = _run_masked(dev, w, np.ones((w.B, w.H, nt, nt), np.uint8))
    torch.cuda.synchronize()
    sage.sage_check()
    assert torch.equal(sp, dense)
    assert torch.equal(ones, dense)


@pytest.mark.parametrize("w,density", [
    (tiny_custom(1, 2, 300, 64, 511, bias_sigma=2.0), 0.5),
    (tiny_custom(1, 2, 777, 128, 512, layout="fused", bias_sigma=4.0, outlier_frac=0.01), 0.4),
    (tiny_custom(2, 1, 1280, 64, 513, bias_sigma=2.0), 0.25),
    (tiny_custom(1, 1, 129, 128, 514), 0.5),
], ids=lambda x: getattr(x, "name", str(x)))
def test_drawn_mask_matches_the_masked_oracle(w, density):
    (q, k, v), dev = _inputs(w)
    keep = _draw_keep(w.B, w.H, w.N, w.seed, density)
    out = _run_masked(dev, w, keep)
    got = U.bf16_to_f64(out)
    _, bits = oracle.attn_quant(q, k, v, w.sm_scale, kv_keep=keep)
    want = oracle.bf16_bits_to_f64(bits)
    ok, rel, mx, nstep = U.within_tol(got, want, label="drawn mask " + w.name)
    assert np.isfinite(got).all()
    assert ok, (w.name, rel, mx, nstep)
    assert np.all(got[:, :, :T] == 0.0)       # tile 0 keeps nothing


def _oracle_codes_on_gpu(codes, N):
    """The oracle's codes and scales, padded to the library's layout (rows past
    N zero, padded blocks with scale 0), as device tensors."""
    npd = sage.n_pad(N)

    def pad(a, n, axis):
        z = np.zeros(a.shape[:axis] + (n,) + a.shape[axis + 1:], dtype=a.dtype)
        z[(slice(None),) * axis + (slice(0, a.shape[axis]),)] = a
        return torch.from_numpy(z).to(DEV)

    return dict(q_i8=pad(codes["q_i8"], npd, 2), k_i8=pad(codes["k_i8"], npd, 2),
                q_scale=pad(codes["q_scale"], npd // 128, 2), k_scale=pad(codes["k_scale"], npd // 64, 2))


@pytest.mark.parametrize("w", [
    tiny_custom(1, 3, 1500, 128, 521, bias_sigma=4.0, outlier_frac=0.01),
    tiny_custom(2, 2, 2100, 64, 522, bias_sigma=2.0),
    tiny_custom(1, 2, 4608, 128, 523, layout="fused", bias_sigma=4.0, outlier_frac=0.01),
], ids=lambda w: w.name)
def test_selection_matches_the_oracle(w):
    """Readings S2 and S3 fix every fp32 operation and its order, so on the
    same codes the GPU's tile scores equal the oracle's bit for bit and the
    kept sets are the same on every row.  The codes are the oracle's own
    (passed to both sides), and then the GPU's quantize pass's (equal to the
    oracle's: the K mean is an exact sum on both sides)."""
    (q, k, v), dev = _inputs(w, planted=True)
    oc = oracle.quantize(q, k, v)
    sbar_o = oracle.block_scores(q, k, v, w.sm_scale, codes=oc)
    nt = sbar_o.shape[-1]
    codes_o = _oracle_codes_on_gpu(oc, w.N)
    codes_g = sage.sage_quant_qk(dev[0], dev[1])
    for tau in (0.3, 0.6, 0.9, 0.999):
        keep_o = oracle.block_select(sbar_o, w.N, tau)
        for codes in (codes_o, codes_g):
            mask, sbar_g = sage.sage_block_select(codes, w.N, w.sm_scale, tau, want_scores=True)
            torch.cuda.synchronize()
            sage.sage_check()
            np.testing.assert_array_equal(sbar_g.cpu().numpy(), sbar_o)
            keep_g = sage.mask_to_keep(mask, nt).cpu().numpy()
            assert np.array_equal(keep_g, keep_o.astype(bool)), tau
        assert keep_o.sum() < keep_o.size or tau > 0.99
    # the forward's own selection is the same mask
    out, used = sage.sage_attn_fwd_sparse(*dev, tau=0.6, sm_scale=w.sm_scale, return_mask=True)
    again = sage.sage_block_select(codes_g, w.N, w.sm_scale, 0.6)
    torch.cuda.synchronize()
    assert torch.equal(used, again)


def test_tied_tile_scores_keep_the_lowest_key_tiles():
    """Every key the same row: the smoothed K codes are all zero, so every
    tile score ties at 0 and the ranking falls back to the key tile's index
    (reading S3: lower index first).  Each query tile keeps the shortest
    prefix of key tiles whose token count reaches tau of N (the last tile is
    ragged), the same mask as the oracle's, and the forward with it equals
    the oracle's masked emulation."""
    B, H, N, d = 1, 2, 1100, 128
    g = torch.Generator().manual_seed(541)
    q = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    k = (2.0 * torch.randn(B, H, 1, d, generator=g)).expand(B, H, N, d).contiguous().to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    sm_scale = d ** -0.5
    nt = -(-N // T)
    sizes = np.minimum(T, N - T * np.arange(nt))
    sbar_o = oracle.block_scores(q, k, v, sm_scale)
    assert (sbar_o == 0).all()
    dev = tuple(t.to(DEV) for t in (q, k, v))
    codes = sage.sage_quant_qk(dev[0], dev[1])
    for tau in (0.05, 0.5, 0.93, 1.0):
        keep_o = oracle.block_select(sbar_o, N, tau).astype(bool)
        n_keep = int(np.searchsorted(np.cumsum(sizes), tau * N - 1e-9) + 1)  # shortest prefix reaching tau*N
        assert (keep_o == (np.arange(nt) < min(n_keep, nt))).all(), tau
        mask = sage.sage_block_select(codes, N, sm_scale, tau)
        out, used = sage.sage_attn_fwd_sparse(*dev, tau=tau, sm_scale=sm_scale, return_mask=True)
        torch.cuda.synchronize()
        sage.sage_check()
        assert np.array_equal(sage.mask_to_keep(mask, nt).cpu().numpy(), keep_o), tau
        assert torch.equal(used, mask)
        _, bits = oracle.attn_quant(q, k, v, sm_scale, kv_keep=keep_o.astype(np.uint8))
        ok, rel, mx, nstep = U.within_tol(U.bf16_to_f64(out), oracle.bf16_bits_to_f64(bits), label=f"ties tau {tau}")
        assert ok, (tau, rel, mx, nstep)


@pytest.mark.parametrize("d", [64, 128])
def test_the_largest_tile_count(d):
    """N = 4096 * 128 tokens: the most key tiles one selection ranks (4096,
    in shared memory), and at d = 128 the attention kernel's largest shared
    memory (its step lists for 4096 query tiles on top of the tiles).  The
    tile scores and the kept sets equal the oracle's bit for bit on every
    query tile, the selecting forward uses that mask, and its sampled rows
    are within the bar.  The keys carry an offset that falls along the
    sequence, so every row of scores is sorted up to local disorder (which
    keeps the oracle's insertion-sort ranking quick)."""
    B, H, N = 1, 1, 4096 * T
    nt = N // T
    g = torch.Generator().manual_seed(561)
    u = torch.randn(d, generator=g)
    u = u / u.norm() * 4.0
    fall = torch.linspace(1.0, -1.0, nt).repeat_interleave(T).view(1, 1, N, 1)
    q = (0.5 * torch.randn(B, H, N, d, generator=g) + u).to(torch.bfloat16)
    k = (0.5 * torch.randn(B, H, N, d, generator=g) + fall * u).to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    sm_scale, tau = d ** -0.5, 0.3
    sbar_o = oracle.block_scores(q, k, v, sm_scale)
    keep_o = oracle.block_select(sbar_o, N, tau)
    assert 0.02 < keep_o.mean() < 0.5
    dev = tuple(t.to(DEV) for t in (q, k, v))
    codes = sage.sage_quant_qk(dev[0], dev[1])
    mask, sbar_g = sage.sage_block_select(codes, N, sm_scale, tau, want_scores=True)
    out, used = sage.sage_attn_fwd_sparse(*dev, tau=tau, sm_scale=sm_scale, return_mask=True)
    torch.cuda.synchronize()
    sage.sage_check()
    np.testing.assert_array_equal(sbar_g.cpu().numpy(), sbar_o)
    assert np.array_equal(sage.mask_to_keep(mask, nt).cpu().numpy(), keep_o.astype(bool))
    assert torch.equal(used, mask)
    rows = U.sample_rows(N, 24, seed=5)
    _, bits = oracle.attn_quant(q, k, v, sm_scale, rows=rows, kv_keep=keep_o)
    got = U.bf16_to_f64(out[0, 0, torch.from_numpy(rows).long().to(DEV)])
    ok, rel, mx, nstep = U.within_tol(got, oracle.bf16_bits_to_f64(bits[0, 0]), label="4096 tiles")
    assert ok, (rel, mx, nstep)


def test_tau_forward_matches_the_oracle():
    """The selecting forward against the oracle's selection and masked
    emulation: the same kept sets on every row, outputs within the
    tolerances."""
    w = tiny_custom(1, 2, 1100, 128, 531, bias_sigma=4.0)
    (q, k, v), dev = _inputs(w, planted=True)
    out, mask = sage.sage_attn_fwd_sparse(*dev, tau=0.5, sm_scale=w.sm_scale, return_mask=True)
    torch.cuda.synchronize()
    sage.sage_check()
    nt = -(-w.N // T)
    keep_g = sage.mask_to_keep(mask, nt).cpu().numpy()
    keep_o = oracle.block_select(oracle.block_scores(q, k, v, w.sm_scale), w.N, 0.5)
    assert np.array_equal(keep_g, keep_o.astype(bool))
    assert keep_o.sum() < 0.8 * keep_o.size              # the selection really skips tiles
    _, bits = oracle.attn_quant(q, k, v, w.sm_scale, kv_keep=keep_o)
    ok, rel, mx, nstep = U.within_tol(U.bf16_to_f64(out), oracle.bf16_bits_to_f64(bits), label="tau forward")
    assert ok, (rel, mx, nstep)


def test_flux_workload_with_a_drawn_mask_on_sampled_rows():
    w = WORKLOADS["flux"]
    (q, k, v), dev = _inputs(w)
    keep = _draw_keep(w.B, w.H, w.N, 541, density=0.5)
    out = _run_masked(dev, w, keep)
    heads = [(0, 0), (0, 13), (0, 23)]
    rows = U.sample_rows(w.N, 48, 7)
    got = U.stack(U.gather(out, heads, rows), heads)
    want = []
    for (b, h) in heads:
        sl = (slice(b, b + 1), slice(h, h + 1))
        _, bits = oracle.attn_quant(q[sl], k[sl], v[sl], w.sm_scale, rows=rows, kv_keep=keep[sl])
        want.append(oracle.bf16_bits_to_f64(bits[0, 0]))
    ok, rel, mx, nstep = U.within_tol(got, np.stack(want), label="flux drawn mask")
    assert ok, (rel, mx, nstep)


def test_single_tile_sequences():
    w = tiny_custom(1, 2, 77, 64, 551, layout="fused", bias_sigma=2.0)
    _, dev = _inputs(w)
    dense = sage.sage_attn_fwd(*dev, sm_scale=w.sm_scale)
    full = _run_masked(dev, w, np.ones((1, 2, 1, 1), np.uint8))
    empty = _run_masked(dev, w, np.zeros((1, 2, 1, 1), np.uint8))
    sel, mask = sage.sage_attn_fwd_sparse(*dev, tau=0.2, sm_scale=w.sm_scale, return_mask=True)
    torch.cuda.synchronize()
    sage.sage_check()
    assert torch.equal(full, dense)
    assert torch.count_nonzero(empty).item() == 0
    assert torch.equal(sel, dense)  # one tile: every tau keeps it
    assert sage.mask_to_keep(mask, 1).all()


@pytest.mark.parametrize("w", [WORKLOADS["flux"], WORKLOADS["sdxl"], tiny_custom(2, 3, 1000, 128, 561, bias_sigma=3.0)],
                         ids=lambda w: w.name)
def test_forward_selection_equals_the_standalone_selection_on_its_codes(w):
    """The selecting forward pools the tiles' codes inside its quantize pass;
    sage_block_select pools them from the codes in a kernel of its own.  On
    the same inputs (whose codes both sides share bit for bit) the two kept
    sets must be the same on every row, for several tau."""
    _, dev = _inputs(w, planted=True)
    codes = sage.sage_quant_qk(dev[0], dev[1])
    for tau in (0.3, 0.5, 0.9):
        _, mask = sage.sage_attn_fwd_sparse(*dev, tau=tau, sm_scale=w.sm_scale, return_mask=True)
        alone = sage.sage_block_select(codes, w.N, w.sm_scale, tau)
        torch.cuda.synchronize()
        sage.sage_check()
        assert torch.equal(mask, alone), (w.name, tau)
