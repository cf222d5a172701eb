"""Pins of the CPU oracle against mathematics it does not itself define.

Exact mode: brute force, closed forms of softmax, invariants.
Quant mode: equals exact mode with every error source off; an independent
tile-by-tile online replay; closed forms of the int8 codes; the e4m3 and bf16
rounding helpers against the format definitions and torch's casts.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests import _brute
from quantized_attention_qk_b200.inputs import WORKLOADS, make_qkv, tiny_custom

pytestmark = pytest.mark.usefixtures("oracle_lib")


def _rand_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)


def _as4(t):
    return t.view(1, 1, *t.shape)


# --------------------------------------------------------------------------
# exact mode
# --------------------------------------------------------------------------

@pytest.mark.parametrize("N,d", [(1, 1), (2, 3), (5, 4), (16, 8), (13, 7)])
def test_exact_matches_brute_force(N, d):
    q, k, v = (_rand_bf16((N, d), s) for s in (1 + N, 2 + N, 3 + N))
    sm = 1.0 / math.sqrt(d)
    got = oracle.attn_exact(_as4(q), _as4(k), _as4(v), sm)[0, 0]
    want = np.array(_brute.exact_attention_loops(_brute.bf16_values(q), _brute.bf16_values(k),
                                                 _brute.bf16_values(v), sm))
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-14)


def test_exact_closed_forms():
    d = 4
    # q = 0: every score equal -> the plain mean of V.
    N = 9
    q = torch.zeros(N, d, dtype=torch.bfloat16)
    k = _rand_bf16((N, d), 7)
    v = _rand_bf16((N, d), 8)
    out = oracle.attn_exact(_as4(q), _as4(k), _as4(v), 0.5)[0, 0]
    np.testing.assert_allclose(out, np.tile(v.double().mean(0).numpy(), (N, 1)), rtol=1e-14, atol=1e-15)
    # two keys: weight of key 0 is the logistic of the score difference.
    q = torch.tensor([[1.0, 0, 0, 0], [1.0, 0, 0, 0]], dtype=torch.bfloat16)
    k = torch.tensor([[2.0, 0, 0, 0], [0.5, 0, 0, 0]], dtype=torch.bfloat16)
    v = torch.tensor([[1.0, 2, 3, 4], [-1.0, 0, 1, 0.5]], dtype=torch.bfloat16)
    sm = 0.75
    w0 = 1.0 / (1.0 + math.exp(-(2.0 - 0.5) * sm))
    want = w0 * v[0].double().numpy() + (1 - w0) * v[1].double().numpy()
    out = oracle.attn_exact(_as4(q), _as4(k), _as4(v), sm)[0, 0]
    np.testing.assert_allclose(out, np.tile(want, (2, 1)), rtol=1e-14)
    # one key with a score far above the rest -> that key's V row.
    N = 6
    q = torch.zeros(N, d, dtype=torch.bfloat16)
    q[:, 0] = 64.0
    k = torch.zeros(N, d, dtype=torch.bfloat16)
    k[3, 0] = 64.0
    v = _rand_bf16((N, d), 9)
    out = oracle.attn_exact(_as4(q), _as4(k), _as4(v), 1.0)[0, 0]
    np.testing.assert_allclose(out, np.tile(v[3].double().numpy(), (N, 1)), rtol=0, atol=1e-300)


def test_exact_weights_sum_to_one_and_uniform_v():
    N, d = 37, 8
    q, k = _rand_bf16((N, d), 11, 3.0), _rand_bf16((N, d), 12, 3.0)
    row = _rand_bf16((1, d), 13)
    v = row.expand(N, d).contiguous()
    out, w = oracle.attn_exact(_as4(q), _as4(k), _as4(v), 0.3, want_weights=True)
    np.testing.assert_allclose(w[0, 0].sum(axis=1), np.ones(N), rtol=0, atol=1e-12)
    assert (w >= 0).all() and (w <= 1).all()
    np.testing.assert_allclose(out[0, 0], np.tile(row.double().numpy(), (N, 1)), rtol=1e-12, atol=1e-12)


def test_exact_invariant_under_per_channel_k_offset():
    """q.(k_j + b) = q.k_j + q.b: a per-row constant, so softmax is unchanged.
    Values are multiples of 1/8 so that K + b stays exact in bf16."""
    N, d = 20, 8
    g = torch.Generator().manual_seed(5)
    q = (torch.randint(-16, 17, (N, d), generator=g) / 8.0).to(torch.bfloat16)
    k = (torch.randint(-16, 17, (N, d), generator=g) / 8.0).to(torch.bfloat16)
    v = _rand_bf16((N, d), 6)
    b = (torch.randint(-40, 41, (1, d), generator=g) / 8.0)
    kb = (k.float() + b).to(torch.bfloat16)
    assert torch.equal(kb.float() - b, k.float())
    o1 = oracle.attn_exact(_as4(q), _as4(k), _as4(v), 0.35)[0, 0]
    o2 = oracle.attn_exact(_as4(q), _as4(kb), _as4(v), 0.35)[0, 0]
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------

def test_e4m3_decode_table_matches_definition_and_torch():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    for c in range(256):
        s, E, M = c >> 7, (c >> 3) & 15, c & 7
        if E == 15 and M == 7:
            assert math.isnan(got[c])
            continue
        val = (M / 8.0) * 2.0 ** -6 if E == 0 else (1 + M / 8.0) * 2.0 ** (E - 7)
        assert got[c] == (-val if s else val), c
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    assert np.nanmax(got) == 448.0 and np.nanmin(np.abs(got[got != 0])) == 2.0 ** -9


def test_e4m3_encode_roundtrip_midpoints_saturation():
    codes = np.array([c for c in range(256) if (c & 0x7f) != 0x7f], dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    back = oracle.e4m3_encode(vals)
    np.testing.assert_array_equal(back, codes)
    pos = np.sort(np.unique(vals[vals >= 0]))
    mids = (pos[:-1] + pos[1:]) / 2
    enc = oracle.e4m3_encode(mids)
    # a tie goes to the neighbour whose mantissa is even
    assert all((int(c) & 1) == 0 for c in enc)
    assert all(oracle.e4m3_decode([c])[0] in (lo, hi) for c, lo, hi in zip(enc, pos[:-1], pos[1:]))
    np.testing.assert_array_equal(oracle.e4m3_decode(oracle.e4m3_encode([448.0, 460.0, 464.0, 1e6, -1e6])),
                                  [448.0, 448.0, 448.0, 448.0, -448.0])


def test_e4m3_encode_matches_torch_cast():
    g = torch.Generator().manual_seed(3)
    x = torch.cat([torch.randn(200000, generator=g) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)])
    x = x.clamp(-448, 448)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(x.double().numpy())
    np.testing.assert_array_equal(got, ref)


def test_bf16_rne_matches_torch_cast():
    g = torch.Generator().manual_seed(4)
    x = torch.cat([torch.randn(300000, generator=g) * s for s in (1e-30, 1e-3, 1.0, 1e5)])
    # exact ties: a bf16 value plus half of its last place
    base = torch.randn(1000, generator=g).to(torch.bfloat16).float()
    ulp = torch.ldexp(torch.ones_like(base), torch.frexp(base)[1] - 8)
    x = torch.cat([x, base + ulp / 2, base - ulp / 2])
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_rne(x.double().numpy())
    np.testing.assert_array_equal(got, ref)


# --------------------------------------------------------------------------
# quant mode
# --------------------------------------------------------------------------

def test_int8_codes_closed_form():
    d = 4
    # block amax 2.0 -> inv = 63.5 exactly; 1.0 -> 63.5 -> tie to even 64; 0.5 -> 31.75 -> 32
    q = torch.tensor([[2.0, 1.0, 0.5, -1.0], [-2.0, 0.0, 0.25, -0.5]], dtype=torch.bfloat16)
    z = torch.zeros_like(q)
    r = oracle.quantize(_as4(q), _as4(q), _as4(q), smooth_k=False)
    np.testing.assert_array_equal(r["q_i8"][0, 0], [[127, 64, 32, -64], [-127, 0, 16, -32]])
    assert r["q_scale"][0, 0, 0] == np.float32(2.0) / np.float32(127.0)
    # all-zero block: scale 0, codes 0
    r0 = oracle.quantize(_as4(z), _as4(z), _as4(z))
    assert (r0["q_i8"] == 0).all() and (r0["q_scale"] == 0).all() and (r0["v_scale"] == 0).all()


def test_k_smoothing_statistic_and_blocks():
    w = tiny_custom(1, 1, 200, 16, seed=21, bias_sigma=3.0)
    q, k, v, _ = make_qkv(w)
    r = oracle.quantize(q, k, v)
    np.testing.assert_allclose(r["k_mean"][0, 0], k[0, 0].double().mean(0).numpy(), rtol=1e-6, atol=1e-6)
    assert r["q_scale"].shape[-1] == 2 and r["k_scale"].shape[-1] == 4
    # every K block reaches +-127 at its largest smoothed element
    kc = r["k_i8"][0, 0].astype(np.int64)
    for b0 in range(0, 200, 64):
        assert np.abs(kc[b0:b0 + 64]).max() == 127
    # dequantized K is within half a step of the smoothed value
    ks = k[0, 0].float().numpy() - r["k_mean"][0, 0][None, :]
    deq = kc * np.repeat(r["k_scale"][0, 0], 64)[:200, None]
    assert np.all(np.abs(deq - ks) <= np.repeat(r["k_scale"][0, 0], 64)[:200, None] * 0.5 * (1 + 1e-5))


@pytest.mark.parametrize("name,heads", [("tiny", [0, 1]), ("flux", [0, 11, 23]), ("sdxl", [0, 17, 39])])
def test_k_mean_is_the_exact_mean_on_the_workloads(name, heads):
    """Reading C1: the K mean is fp32(fp64(exact column sum) / N).  On the
    workloads every column sum is exact in fp64 whatever the order (a column's
    values span fewer than 53 bits): the sequential, reversed and 256-token
    chunked fp64 sums all equal math.fsum, which is why a GPU summing in its
    own order gets the oracle's mean bit for bit."""
    w = WORKLOADS[name]
    q, k, v, _ = make_qkv(w)
    N = w.N
    for bh in heads:
        b, h = divmod(bh, w.H)
        sl = (slice(b, b + 1), slice(h, h + 1))
        mu = oracle.quantize(q[sl], k[sl], v[sl])["k_mean"][0, 0]
        kk = k[b, h].double().numpy()
        seq = np.cumsum(kk, axis=0)[-1]
        rev = np.cumsum(kk[::-1], axis=0)[-1]
        chunks = np.cumsum(np.array([kk[i:i + 256].sum(axis=0) for i in range(0, N, 256)]), axis=0)[-1]
        for c in range(w.d):
            exact = math.fsum(kk[:, c])
            assert seq[c] == exact and rev[c] == exact and chunks[c] == exact, (bh, c)
            assert mu[c] == np.float32(exact / N), (bh, c)


def test_quant_codes_match_numpy_restatement():
    w = tiny_custom(1, 1, 300, 32, seed=22, bias_sigma=2.0, outlier_frac=0.05)
    q, k, v, _ = make_qkv(w)
    r = oracle.quantize(q, k, v)
    qc, qs, kc, ks, mu, vval, vs = _brute.quant_codes_numpy(q[0, 0].float().numpy(), k[0, 0].float().numpy(),
                                                            v[0, 0].float().numpy())
    np.testing.assert_array_equal(r["q_i8"][0, 0], qc)
    np.testing.assert_array_equal(r["q_scale"][0, 0], qs)
    np.testing.assert_array_equal(r["k_mean"][0, 0], mu)
    np.testing.assert_array_equal(r["k_i8"][0, 0], kc)
    np.testing.assert_array_equal(r["k_scale"][0, 0], ks)
    np.testing.assert_array_equal(r["v_scale"][0, 0], vs)
    np.testing.assert_array_equal(oracle.e4m3_decode(r["v_e4m3"][0, 0]).reshape(300, 32) * vs[None, :], vval)


@pytest.mark.parametrize("smooth", [True, False])
def test_quant_with_error_sources_off_equals_exact(smooth):
    w = tiny_custom(1, 2, 150, 16, seed=23, bias_sigma=2.0)
    q, k, v, _ = make_qkv(w)
    ex = oracle.attn_exact(q, k, v, w.sm_scale)
    f64, _ = oracle.attn_quant(q, k, v, w.sm_scale, int8_qk=False, fp8_p=False, fp8_v=False,
                               round_bf16=False, smooth_k=smooth)
    np.testing.assert_allclose(f64, ex, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("N,d,bkv", [(300, 16, 128), (300, 16, 64), (129, 64, 128), (64, 8, 32)])
def test_quant_equals_tiled_online_replay(N, d, bkv):
    w = tiny_custom(1, 1, N, d, seed=30 + N + d, bias_sigma=2.0, outlier_frac=0.02)
    q, k, v, _ = make_qkv(w)
    f64, _ = oracle.attn_quant(q, k, v, w.sm_scale)
    rep = _brute.tiled_online_quant(q[0, 0].float().numpy(), k[0, 0].float().numpy(), v[0, 0].float().numpy(),
                                    w.sm_scale, bkv)
    np.testing.assert_allclose(f64[0, 0], rep, rtol=1e-12, atol=1e-13)


def test_quant_bf16_output_is_rne_of_f64():
    w = tiny_custom(1, 1, 70, 16, seed=41)
    q, k, v, _ = make_qkv(w)
    f64, bits = oracle.attn_quant(q, k, v, w.sm_scale)
    ref = torch.from_numpy(f64[0, 0].astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    # fp64 -> fp32 -> bf16 may double-round only at exact fp32 ties; none occur here
    np.testing.assert_array_equal(bits[0, 0], ref)


def test_quant_single_key_returns_quantized_v():
    N, d = 1, 8
    q, k, v = (_rand_bf16((N, d), s) for s in (51, 52, 53))
    f64, _ = oracle.attn_quant(_as4(q), _as4(k), _as4(v), 0.3)
    r = oracle.quantize(_as4(q), _as4(k), _as4(v))
    vq = oracle.e4m3_decode(r["v_e4m3"][0, 0]).reshape(N, d) * r["v_scale"][0, 0]
    # one key: p = 2^(x - ceil x) in (1/2, 1], so 448 p is rounded once; the ratio P/(448 p) stays within e4m3's step
    ratio = f64[0, 0] / vq
    assert np.all(np.abs(ratio - 1) <= 2.0 ** -4 + 1e-12)


def test_quant_error_scale_on_tiny_workload():
    """The scheme's own error against exact attention: nonzero, and of the
    size the e4m3/int8 steps imply (a few percent), on the tiny workload."""
    from quantized_attention_qk_b200.inputs import WORKLOADS
    w = WORKLOADS["tiny"]
    q, k, v, _ = make_qkv(w)
    rows = np.arange(0, w.N, 7)
    ex = oracle.attn_exact(q, k, v, w.sm_scale, rows=rows)
    f64, _ = oracle.attn_quant(q, k, v, w.sm_scale, rows=rows)
    rel = np.linalg.norm(f64 - ex) / np.linalg.norm(ex)
    assert 1e-3 < rel < 0.1, rel


# --------------------------------------------------------------------------- K-residual mode
# ("ComfyUI-sol-attn", 核心亮点 item 1: only the residual of K inside each
# block is quantized; the block-mean term keeps bf16 precision)

def test_kres_with_error_sources_off_equals_exact():
    """q.k = q.mean_b + q.(k - mean_b) exactly, so with every rounding switched
    off the K-residual mode must give exact attention."""
    w = tiny_custom(1, 2, 300, 64, seed=91, bias_sigma=4.0, outlier_frac=0.02)
    q, k, v, _ = make_qkv(w)
    rows = np.arange(0, 300, 7).astype(np.int32)
    ex = oracle.attn_exact(q, k, v, w.sm_scale, rows=rows)
    o, _ = oracle.attn_quant(q, k, v, w.sm_scale, rows=rows, int8_qk=False, fp8_p=False, fp8_v=False,
                             round_bf16=False, k_residual=True)
    assert np.max(np.abs(o - ex)) < 1e-12


def test_kres_codes_match_numpy_restatement():
    w = tiny_custom(1, 1, 200, 64, seed=92, bias_sigma=3.0, outlier_frac=0.05)
    _, k, _, _ = make_qkv(w)
    got = oracle.quantize_kres(k)
    kf = k[0, 0].float().numpy()
    for b in range(-(-200 // 64)):
        blk = kf[b * 64:(b + 1) * 64].astype(np.float64)
        mean = blk.mean(axis=0)
        mb = torch.from_numpy(got["k_bmean"][0, 0, b].astype(np.int16)).view(torch.bfloat16).float().numpy()
        # the stored mean is the bf16 nearest the fp64 mean (within half a bf16 step)
        step = np.exp2(np.floor(np.log2(np.maximum(np.abs(mean), 1e-30))) - 7)
        assert np.all(np.abs(mb.astype(np.float64) - mean) <= step / 2 + 1e-30)
        r = (kf[b * 64:(b + 1) * 64] - mb).astype(np.float32)     # exact in fp32
        amax = np.float32(np.abs(r).max())
        inv = np.float32(127.0) / amax
        want = np.clip(np.rint((r * inv).astype(np.float32)), -127, 127).astype(np.int8)
        assert np.array_equal(got["k_i8"][0, 0, b * 64:(b + 1) * 64], want)
        assert got["k_scale"][0, 0, b] == np.float32(amax / np.float32(127.0))


def test_kres_block_mean_term_varies_by_block():
    """The block-mean term must enter the scores: dropping it (a per-row constant
    only for the global mean) would change the result."""
    w = tiny_custom(1, 1, 256, 64, seed=93, bias_sigma=2.0)
    q, k, v, _ = make_qkv(w)
    k = k.clone()
    k[0, 0, 128:] += 2.0          # a block-wise shift of the keys
    rows = np.arange(0, 256, 5).astype(np.int32)
    ex = oracle.attn_exact(q, k, v, w.sm_scale, rows=rows)
    o, _ = oracle.attn_quant(q, k, v, w.sm_scale, rows=rows, fp8_p=False, fp8_v=False, round_bf16=False,
                             k_residual=True)
    assert np.linalg.norm(o - ex) / np.linalg.norm(ex) < 0.03


def test_kres_constant_block_has_zero_residual():
    """A K block whose rows are all equal is its own mean: the residual codes and
    the block scale are 0, and with the remaining rounding switched off the
    scores of that block are the mean term alone, so attention is exact."""
    w = tiny_custom(1, 1, 128, 64, seed=94, bias_sigma=1.0)
    q, k, v, _ = make_qkv(w)
    k = k.clone()
    k[0, 0, :64] = k[0, 0, 5]            # block 0: one repeated bf16 row
    got = oracle.quantize_kres(k)
    assert np.all(got["k_i8"][0, 0, :64] == 0)
    assert got["k_scale"][0, 0, 0] == 0.0
    mb = torch.from_numpy(got["k_bmean"][0, 0, 0].astype(np.int16)).view(torch.bfloat16)
    assert torch.equal(mb, k[0, 0, 5])   # the mean of equal bf16 values is that value
    rows = np.arange(0, 128, 3).astype(np.int32)
    ex = oracle.attn_exact(q, k, v, w.sm_scale, rows=rows)
    o, _ = oracle.attn_quant(q, k, v, w.sm_scale, rows=rows, int8_qk=False, fp8_p=False, fp8_v=False,
                             round_bf16=False, k_residual=True)
    assert np.max(np.abs(o - ex)) < 1e-12


# --------------------------------------------------------------------------
# integer score tiles (the closed form the GPU's S tiles are checked against)
# --------------------------------------------------------------------------

def _int8_codes(shape, rng):
    return rng.integers(-127, 128, size=shape).astype(np.int8)


@pytest.mark.parametrize("m,n,d", [(1, 1, 1), (3, 5, 64), (7, 2, 128), (5, 9, 33)])
def test_int8_gemm_nt_equals_python_integer_loops(m, n, d):
    """s[i][j] = sum_c a[i][c] b[j][c] over Python ints, with rows at +-127."""
    rng = np.random.default_rng(1000 * m + 10 * n + d)
    a, b = _int8_codes((m, d), rng), _int8_codes((n, d), rng)
    a[0] = -127                       # extreme rows: |s| = 127 * 127 * d
    b[-1] = -127
    got = oracle.int8_gemm_nt(a, b)
    assert got.shape == (m, n) and got.dtype == np.int32
    for i in range(m):
        for j in range(n):
            want = sum(int(a[i, c]) * int(b[j, c]) for c in range(d))
            assert int(got[i, j]) == want, (i, j)
    assert int(got[0, n - 1]) == 127 * 127 * d


@pytest.mark.parametrize("m,n,d", [(128, 96, 128), (40, 128, 64), (128, 128, 128)])
def test_int8_gemm_nt_equals_int64_product_not_transposed(m, n, d):
    """Against the int64 matrix product a b^T (m != n catches a swapped
    operand or a transposed result), including the largest magnitudes."""
    rng = np.random.default_rng(7 * m + n + d)
    a, b = _int8_codes((m, d), rng), _int8_codes((n, d), rng)
    a[1] = 127
    a[2] = -127
    b[3] = -127
    got = oracle.int8_gemm_nt(a, b)
    want = a.astype(np.int64) @ b.astype(np.int64).T
    np.testing.assert_array_equal(got.astype(np.int64), want)
    assert got[2, 3] == 127 * 127 * d and got[1, 3] == -127 * 127 * d


def test_int8_gemm_nt_indexes_rows_and_channels():
    """One nonzero code per row: s[i][j] is nonzero only where a's channel of
    row i meets b's channel of row j, so a swapped index shows at once; the
    row strides of the C routine are exercised with padded rows."""
    m, n, d, pad = 6, 4, 16, 24
    a = np.zeros((m, pad), np.int8)
    b = np.zeros((n, pad), np.int8)
    ca = [0, 3, 5, 7, 9, 15]
    cb = [3, 9, 0, 15]
    for i, c in enumerate(ca):
        a[i, c] = i + 1
        a[i, d:] = 99                 # padding past d must not be read
    for j, c in enumerate(cb):
        b[j, c] = -(j + 2)
        b[j, d:] = 99
    s = np.zeros((m, n), np.int32)
    L = oracle.lib()
    rc = L.oracle_int8_gemm_nt(oracle._ptr(a), pad, oracle._ptr(b), pad, m, n, d, oracle._ptr(s))
    assert rc == 0
    for i in range(m):
        for j in range(n):
            want = (i + 1) * -(j + 2) if ca[i] == cb[j] else 0
            assert s[i, j] == want, (i, j)
