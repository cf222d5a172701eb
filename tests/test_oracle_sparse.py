"""Pins of the oracle's block-sparse skipping (readings S1-S4 of the
"ComfyUI-sol-attn" page, 核心亮点 item 4) against facts it does not itself
define:

* the tile-pair score equals the mean of the dequantized score matrix over
  the tile pair, computed here in fp64 from the codes (a closed form of the
  pooled dot product);
* the kept set is the unique set with the defining properties of reading S3
  (non-empty, a prefix of the score ranking, enough mass, no redundant tile),
  checked on random scores with ties and a ragged last tile;
* a planted strongly-aligned tile pair is the one a small tau keeps;
* masked attention with every rounding off is the plain softmax over the kept
  keys (fp64 brute force), an all-ones mask changes nothing, and a tile that
  keeps nothing returns zeros;
* the tau schedule's endpoints, midpoint and clamping.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from quantized_attention_qk_b200.inputs import make_qkv, tiny_custom

pytestmark = pytest.mark.usefixtures("oracle_lib")

T = oracle.SEL_TILE
LOG2E = 1.4426950408889634


def _tile_sizes(N):
    nt = -(-N // T)
    return np.array([min(T, N - j * T) for j in range(nt)], dtype=np.float64)


def _dequantized_scores(codes, b, h, N, sm_scale):
    """x[r, s] in log2 units from the codes, fp64."""
    qd = codes["q_i8"][b, h].astype(np.float64) * np.repeat(codes["q_scale"][b, h].astype(np.float64), 128)[:N, None]
    kd = codes["k_i8"][b, h].astype(np.float64) * np.repeat(codes["k_scale"][b, h].astype(np.float64), 64)[:N, None]
    s_l2 = float(np.float32(np.float32(sm_scale) * np.float32(LOG2E)))
    return (qd @ kd.T) * s_l2


def _planted(N, d, seed, tile_q, tile_k, gain):
    """Inputs with one strongly aligned (query tile, key tile) pair."""
    w = tiny_custom(1, 1, N, d, seed, bias_sigma=2.0)
    q, k, v, _ = make_qkv(w)
    g = torch.Generator().manual_seed(seed + 7)
    u = torch.randn(d, generator=g)
    u = u / u.norm() * gain
    q = q.float()
    k = k.float()
    q[0, 0, tile_q * T:(tile_q + 1) * T] += u
    k[0, 0, tile_k * T:(tile_k + 1) * T] += u
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v, w.sm_scale


@pytest.mark.parametrize("N,d,seed", [(300, 64, 11), (257, 128, 12), (512, 64, 13)])
def test_tile_score_is_the_mean_dequantized_score(N, d, seed):
    q, k, v, sm = _planted(N, d, seed, tile_q=1, tile_k=0, gain=6.0)
    codes = oracle.quantize(q, k, v)
    sbar = oracle.block_scores(q, k, v, sm, codes=codes)[0, 0]
    x = _dequantized_scores(codes, 0, 0, N, sm)
    nt = -(-N // T)
    for i in range(nt):
        for j in range(nt):
            blk = x[i * T:(i + 1) * T, j * T:(j + 1) * T]
            want = blk.mean()
            # fp32 pipeline: a handful of roundings per channel on values of
            # size |mean q| |mean k|; bound them by the absolute products
            mag = np.abs(blk).mean() + abs(want)
            assert abs(float(sbar[i, j]) - want) <= 1e-5 * mag + 1e-9, (i, j, sbar[i, j], want)
    # the planted pair stands out
    assert np.argmax(sbar[1]) == 0


def _ranked(row):
    return sorted(range(len(row)), key=lambda j: (-float(row[j]), j))


@pytest.mark.parametrize("seed", range(6))
def test_selection_has_the_defining_properties(seed):
    rng = np.random.default_rng(seed)
    N = int(rng.integers(200, 1400))
    nt = -(-N // T)
    sbar = (rng.standard_normal((1, 2, nt, nt)) * rng.uniform(0.1, 4.0)).astype(np.float32)
    sbar[0, 1, :, ::3] = sbar[0, 1, :, :1]          # ties, broken by the lower index
    n = _tile_sizes(N)
    prev = None
    for tau in [1e-6, 0.2, 0.5, 0.8, 0.95, 0.999999, 1.0, 3.0]:
        keep = oracle.block_select(sbar, N, tau)
        for h in range(2):
            for i in range(nt):
                row, kr = sbar[0, h, i], keep[0, h, i].astype(bool)
                order = _ranked(row)
                kcount = int(kr.sum())
                assert kcount >= 1
                assert set(np.nonzero(kr)[0]) == set(order[:kcount]), "kept set is not a ranking prefix"
                if tau >= 1.0:
                    assert kcount == nt
                    continue
                wts = n * np.exp2(row.astype(np.float64) - float(row.max()))
                total = wts.sum()
                kept = sum(wts[j] for j in order[:kcount])
                # the selection sums its masses in fp32 (reading S3): allow
                # its accumulated rounding, a few units of 2^-24 per term
                eps = 4 * nt * 2.0 ** -24
                assert kept >= tau * total * (1 - eps), "kept mass below tau"
                assert kept - wts[order[kcount - 1]] < tau * total * (1 + eps), "a redundant tile is kept"
        if prev is not None:
            assert np.all(keep >= prev), "a larger tau dropped a tile"
        prev = keep


def test_selection_exponential_is_2_to_the_x():
    """The fixed fp32 exponential of reading S3's masses against the library
    exp2 in fp64: within 2e-7 relative on [-64, 0], exact at the integers (a
    power of two times the polynomial's value 1 at f = 0), 0 below -64."""
    x = np.concatenate([np.linspace(-64.0, 0.0, 200001, dtype=np.float32),
                        -np.logspace(-8, 0, 2001).astype(np.float32)])
    y = oracle.s3_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y / ref - 1.0)) < 2e-7
    ints = -np.arange(0, 65, dtype=np.float32)
    np.testing.assert_array_equal(oracle.s3_exp2(ints), np.exp2(ints))
    assert np.all(oracle.s3_exp2(np.array([-64.001, -100.0, -1e30], np.float32)) == 0.0)
    # monotone, as the ranking of masses needs
    xs = np.sort(np.random.default_rng(5).uniform(-64, 0, 100000).astype(np.float32))
    assert np.all(np.diff(oracle.s3_exp2(xs)) >= 0)


def test_small_tau_keeps_the_planted_tile():
    N, d = 640, 64
    q, k, v, sm = _planted(N, d, 21, tile_q=3, tile_k=1, gain=8.0)
    keep = oracle.block_select(oracle.block_scores(q, k, v, sm), N, 0.3)[0, 0]
    assert keep[3].tolist() == [0, 1, 0, 0, 0]
    assert keep.sum(axis=1).min() >= 1


def _exact_masked(q, k, v, sm, keep):
    qf, kf, vf = (t[0, 0].double().numpy() for t in (q, k, v))
    N = qf.shape[0]
    out = np.zeros_like(qf)
    for r in range(N):
        cols = [j for j in range(N) if keep[r // T, j // T]]
        if not cols:
            continue
        x = qf[r] @ kf[cols].T * sm
        p = np.exp(x - x.max())
        out[r] = p @ vf[cols] / p.sum()
    return out


@pytest.mark.parametrize("N,d,seed", [(300, 32, 31), (384, 16, 32)])
def test_masked_exact_mode_is_the_softmax_over_kept_keys(N, d, seed):
    w = tiny_custom(1, 1, N, d, seed, bias_sigma=1.0)
    q, k, v, _ = make_qkv(w)
    nt = -(-N // T)
    rng = np.random.default_rng(seed)
    keep = (rng.random((nt, nt)) < 0.5).astype(np.uint8)
    keep[0] = 0                      # a query tile that keeps nothing
    keep[1] = 0
    keep[1, nt - 1] = 1              # one that keeps only the ragged tail tile
    got, _ = oracle.attn_quant(q, k, v, w.sm_scale, int8_qk=False, fp8_p=False, fp8_v=False,
                               round_bf16=False, smooth_k=False, kv_keep=keep[None, None])
    want = _exact_masked(q, k, v, float(np.float32(w.sm_scale)), keep)  # the oracle takes sm_scale as fp32
    np.testing.assert_allclose(got[0, 0], want, rtol=0, atol=1e-12)
    assert np.all(got[0, 0, :T] == 0.0)


def test_all_kept_mask_changes_nothing_and_empty_tiles_are_zero():
    w = tiny_custom(1, 2, 333, 64, 41, bias_sigma=4.0, outlier_frac=0.02)
    q, k, v, _ = make_qkv(w)
    nt = -(-w.N // T)
    ref = oracle.attn_quant(q, k, v, w.sm_scale)[1]
    ones = np.ones((1, 2, nt, nt), np.uint8)
    assert np.array_equal(oracle.attn_quant(q, k, v, w.sm_scale, kv_keep=ones)[1], ref)
    keep = ones.copy()
    keep[0, 1, 2] = 0
    got = oracle.attn_quant(q, k, v, w.sm_scale, kv_keep=keep)[1]
    assert np.all(got[0, 1, 2 * T:] == 0)
    assert np.array_equal(got[0, 0], ref[0, 0])
    assert np.array_equal(got[0, 1, :2 * T], ref[0, 1, :2 * T])


def test_tau_schedule_endpoints_midpoint_and_clamping():
    assert oracle.tau_schedule(0, 11, 0.5, 1.0) == 0.5
    assert oracle.tau_schedule(10, 11, 0.5, 1.0) == 1.0
    assert math.isclose(oracle.tau_schedule(5, 11, 0.5, 1.0), 0.75, rel_tol=0, abs_tol=1e-15)
    assert oracle.tau_schedule(-3, 11, 0.5, 1.0) == 0.5
    assert oracle.tau_schedule(99, 11, 0.5, 1.0) == 1.0
    assert oracle.tau_schedule(0, 1, 0.2, 0.9) == 0.9
    vals = [oracle.tau_schedule(s, 30, 0.3, 1.0) for s in range(30)]
    assert all(a < b for a, b in zip(vals, vals[1:]))
