/*
 * sage_oracle.c -- CPU oracle for SageAttention-style quantized attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: it is used by the test-suite, by the smoke check and by the
 * CPU-baseline leg of the benchmark.  It shares no code, header, table or
 * constant generator with the CUDA library.
 *
 * It is deliberately plain, slow and single-threaded.  Every function works on
 * ONE (batch, head) slab; the caller loops over slabs.  Inputs are bf16 bit
 * patterns (uint16) with an element stride between token rows; channels are
 * contiguous.
 *
 * What it follows (the pages are cited by title and section):
 *   - "MiniMax H3 接入 SageAttention 实测加速", section 一 (SageAttention 加速了什么):
 *     Attention(Q,K,V) = Softmax(Q K^T / sqrt(d)) V; SageAttention 2 applies
 *     low-bit quantization and outlier smoothing to Q K^T; the sm89 kernel
 *     handles QK in INT8 and PV in FP8.
 *   - "SDPA稠密注意力模式：大模型推理加速的优化方案", section 三.1 (数学基础):
 *     the same dense formula with the 1/sqrt(d_k) scale.
 *   - "GitHub榜单静默期：Attention优化从架构转向推理加速", section 2.2: the
 *     attention matrix is processed block-wise and never written out; low-bit
 *     (INT8) representation of chosen attention operands.
 * Where the pages leave a numeric step open, the reading used here is the one
 * listed (C1..C9) in the project design notes; each step below names it.
 *
 * Two modes:
 *   oracle_attn_exact  -- the plain definition in fp64 (no smoothing, no
 *                         quantization).
 *   (oracle_attn_quant with k_residual set follows "ComfyUI-sol-attn",
 *   核心亮点 item 1 instead of the smoothing: only the residual of K inside
 *   each 64-token block is quantized, and the block mean term stays at bf16
 *   precision -- see oracle_quantize_kres.)
 *   oracle_attn_quant_masked -- the same with block-sparse skipping: each
 *                         128-query tile attends only to the 128-key tiles
 *                         its row of a keep mask selects (see the block
 *                         selection below for how such a mask is chosen).
 *   oracle_attn_quant  -- the quantization scheme, step by step, in the order
 *                         smoothing -> block INT8 of Q and K -> integer Q K^T ->
 *                         dequant -> softmax with an integer-grid (log2) row max
 *                         -> FP8 e4m3 P and V -> fp64 accumulate -> bf16 output.
 *                         Steps the GPU performs order-independently in fp32
 *                         (block amax, scales, codes of Q and V) are emulated
 *                         here in IEEE fp32 so that they can be compared bit
 *                         for bit; everything else is fp64.
 *
 * Pins (tests that tie this file to something other than itself):
 *   exact mode      -- brute force on tiny inputs, softmax closed forms
 *                      (uniform scores, one dominant key, two-key logistic),
 *                      rows of weights summing to one, uniform V returning V,
 *                      invariance under a per-channel K offset.
 *   quant mode      -- with every error source switched off it must equal the
 *                      exact mode; the e4m3 and bf16 rounding helpers against
 *                      the format definitions and a library cast; the int8
 *                      block codes against closed forms; the one-pass
 *                      integer-grid softmax against a tile-by-tile replay of
 *                      the online algorithm.
 *   block sparsity  -- tile scores against the mean of the fp64 dequantized
 *                      score matrix; the kept sets against the properties
 *                      that define reading S3 (ranking prefix, mass reaches
 *                      tau, no redundant tile, nested in tau); masked exact
 *                      mode against a brute-force softmax over the kept keys.
 *
 * Build:  gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -fno-fast-math
 *             -fexcess-precision=standard -o liboracle.so sage_oracle.c -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <fenv.h>

#define ORACLE_Q_BLOCK 128 /* Q tokens per quantization block (reading C3) */
#define ORACLE_K_BLOCK 64  /* K tokens per quantization block (reading C3) */
#define ORACLE_E4M3_MAX 448.0
#define ORACLE_SEL_TILE 128 /* tokens per query / key tile of the block selection (reading S1) */

/* ------------------------------------------------------------------------ */
/* Number formats                                                           */
/* ------------------------------------------------------------------------ */

/* bf16 bit pattern -> value: the top 16 bits of an IEEE binary32. Exact. */
double oracle_bf16_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static float bf16_to_float(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a double to bf16, nearest-even (1 sign, 8 exponent, 7 fraction bits),
 * returned as the bit pattern.  The rounding is done once, directly on the
 * double, at the spacing of the target binade (no detour through binary32). */
uint16_t oracle_bf16_rne(double x)
{
    if (isnan(x)) return 0x7fc0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7f80;
    int e;
    frexp(a, &e);             /* a = f * 2^e with f in [0.5, 1) */
    /* bf16 keeps 8 significant bits; normals start at 2^-126. */
    int exp_unbiased = e - 1; /* a in [2^exp_unbiased, 2^(exp_unbiased+1)) */
    double q;                 /* significand in units of the last place */
    int lsb_exp;
    if (exp_unbiased < -126) lsb_exp = -126 - 7; /* subnormal spacing 2^-133 */
    else lsb_exp = exp_unbiased - 7;
    q = ldexp(a, -lsb_exp); /* exact: scaling by a power of two */
    double r = nearbyint(q); /* ties to even in the default rounding mode */
    double v = ldexp(r, lsb_exp);
    if (v > 0x1.fep127) return sign | 0x7f80; /* rounds past the largest finite -> inf */
    float vf = (float)v; /* exact: v has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &vf, sizeof u);
    return (uint16_t)(sign | ((u >> 16) & 0x7fff));
}

/* e4m3 ("fn" variant: no infinities, one NaN pattern S.1111.111).
 * Value of a code: exponent field E (4 bits, bias 7), mantissa M (3 bits);
 * E > 0: 2^(E-7) * (1 + M/8); E == 0: 2^-6 * (M/8).  Largest finite 448. */
double oracle_e4m3_decode(uint8_t code)
{
    int s = code >> 7, E = (code >> 3) & 0xf, M = code & 7;
    double v;
    if (E == 0xf && M == 7) return NAN;
    if (E == 0) v = ldexp((double)M / 8.0, -6);
    else v = ldexp(1.0 + (double)M / 8.0, E - 7);
    return s ? -v : v;
}

/* Round a finite double to e4m3, nearest-even, saturating to +-448
 * ("satfinite").  Returns the code. */
uint8_t oracle_e4m3_encode(double x)
{
    uint8_t s = signbit(x) ? 0x80 : 0;
    double a = fabs(x);
    if (isnan(x)) return 0x7f;
    if (a >= ORACLE_E4M3_MAX) return s | 0x7e; /* 448 = E 15, M 6 */
    if (a == 0.0) return s;
    int e;
    frexp(a, &e);
    int exp_unbiased = e - 1;   /* a in [2^exp, 2^(exp+1)) */
    int lsb_exp;
    if (exp_unbiased < -6) lsb_exp = -9; /* subnormal spacing 2^-9 */
    else lsb_exp = exp_unbiased - 3;
    double r = nearbyint(ldexp(a, -lsb_exp)); /* ties to even */
    double v = ldexp(r, lsb_exp);
    if (v > ORACLE_E4M3_MAX) v = ORACLE_E4M3_MAX; /* cannot happen below 448 */
    /* encode v exactly */
    if (v == 0.0) return s;
    int ev;
    frexp(v, &ev);
    int E = (ev - 1) + 7;
    uint8_t code;
    if (E <= 0) { /* subnormal: v = M * 2^-9 */
        code = (uint8_t)(int)ldexp(v, 9);
    } else {
        double frac = ldexp(v, -(ev - 1)) - 1.0; /* in [0,1) */
        int M = (int)(frac * 8.0);
        code = (uint8_t)((E << 3) | M);
    }
    return s | code;
}

double oracle_e4m3_round(double x) { return oracle_e4m3_decode(oracle_e4m3_encode(x)); }

/* ------------------------------------------------------------------------ */
/* Exact mode: the plain definition (dense formula of both pages)           */
/* ------------------------------------------------------------------------ */

/* out[r][c] = sum_j w_rj v_j[c],  w_rj = exp(s_rj - max_j s) / sum_j exp(...),
 * s_rj = sm_scale * sum_c q_r[c] k_j[c].  All fp64; inputs decoded exactly.
 * If weights != NULL, the softmax weights of each requested row are written
 * there ([nrows][N]). */
int oracle_attn_exact(const uint16_t *q, int64_t q_rs,
                      const uint16_t *k, int64_t k_rs,
                      const uint16_t *v, int64_t v_rs,
                      int N, int d, double sm_scale,
                      const int32_t *rows, int nrows,
                      double *out, double *weights)
{
    if (N <= 0 || d <= 0) return -1;
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    if (!s) return -2;
    for (int ri = 0; ri < nrows; ++ri) {
        int r = rows[ri];
        if (r < 0 || r >= N) { free(s); return -3; }
        double smax = -INFINITY;
        for (int j = 0; j < N; ++j) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += oracle_bf16_to_double(q[(int64_t)r * q_rs + c]) *
                       oracle_bf16_to_double(k[(int64_t)j * k_rs + c]);
            s[j] = acc * sm_scale;
            if (s[j] > smax) smax = s[j];
        }
        double l = 0.0;
        for (int j = 0; j < N; ++j) { s[j] = exp(s[j] - smax); l += s[j]; }
        for (int c = 0; c < d; ++c) out[(int64_t)ri * d + c] = 0.0;
        for (int j = 0; j < N; ++j) {
            double w = s[j] / l;
            if (weights) weights[(int64_t)ri * N + j] = w;
            for (int c = 0; c < d; ++c)
                out[(int64_t)ri * d + c] += w * oracle_bf16_to_double(v[(int64_t)j * v_rs + c]);
        }
    }
    free(s);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Quantization (smoothing, block INT8 for Q and K, per-channel e4m3 for V)  */
/* ------------------------------------------------------------------------ */

/* Symmetric INT8 code of one fp32 value given the fp32 reciprocal scale:
 * round half to even of the fp32 product, clamped to [-127, 127] (reading C2). */
static int8_t int8_code(float x, float inv)
{
    float y = x * inv;           /* one IEEE fp32 multiply */
    float r = nearbyintf(y);     /* ties to even */
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

/*
 * Quantize one (b,h) slab (all N tokens).
 *   k_mean[c]  = mean over the N tokens of K[:,c]            (reading C1; fp64,
 *                stored rounded to fp32)
 *   Q block b (128 tokens, reading C3):  amax = max |Q| over the block's valid
 *                tokens and all channels; q_scale = fp32(amax/127);
 *                code = rne(fp32(Q * fp32(127/amax)))          (reading C2)
 *   K block b (64 tokens): the same on fp32(K - k_mean32)     (readings C1-C3)
 *   V channel c: amax = max_n |V[n,c]|; v_scale = fp32(amax/448);
 *                code = e4m3_rn_satfinite(fp32(V * fp32(448/amax)))  (reading C7)
 * A zero amax gives scale 0 and all-zero codes.
 * smooth_k = 0 skips the mean subtraction (used by tests).
 * Output layouts (row-major, token-major, no padding):
 *   q_i8[N][d], q_scale[ceil(N/128)], k_i8[N][d], k_scale[ceil(N/64)],
 *   k_mean[d], v_e4m3[N][d], v_scale[d].
 */
int oracle_quantize(const uint16_t *q, int64_t q_rs,
                    const uint16_t *k, int64_t k_rs,
                    const uint16_t *v, int64_t v_rs,
                    int N, int d, int smooth_k,
                    int8_t *q_i8, float *q_scale,
                    int8_t *k_i8, float *k_scale, float *k_mean,
                    uint8_t *v_e4m3, float *v_scale)
{
    if (N <= 0 || d <= 0) return -1;
    /* smoothing statistic */
    for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int n = 0; n < N; ++n) acc += oracle_bf16_to_double(k[(int64_t)n * k_rs + c]);
        k_mean[c] = smooth_k ? (float)(acc / (double)N) : 0.0f;
    }
    /* Q blocks */
    int nqb = (N + ORACLE_Q_BLOCK - 1) / ORACLE_Q_BLOCK;
    for (int b = 0; b < nqb; ++b) {
        int n0 = b * ORACLE_Q_BLOCK, n1 = n0 + ORACLE_Q_BLOCK;
        if (n1 > N) n1 = N;
        float amax = 0.0f;
        for (int n = n0; n < n1; ++n)
            for (int c = 0; c < d; ++c) {
                float a = fabsf(bf16_to_float(q[(int64_t)n * q_rs + c]));
                if (a > amax) amax = a;
            }
        float inv = amax > 0.0f ? 127.0f / amax : 0.0f;
        q_scale[b] = amax > 0.0f ? amax / 127.0f : 0.0f;
        for (int n = n0; n < n1; ++n)
            for (int c = 0; c < d; ++c)
                q_i8[(int64_t)n * d + c] =
                    amax > 0.0f ? int8_code(bf16_to_float(q[(int64_t)n * q_rs + c]), inv) : 0;
    }
    /* K blocks on the smoothed keys */
    int nkb = (N + ORACLE_K_BLOCK - 1) / ORACLE_K_BLOCK;
    for (int b = 0; b < nkb; ++b) {
        int n0 = b * ORACLE_K_BLOCK, n1 = n0 + ORACLE_K_BLOCK;
        if (n1 > N) n1 = N;
        float amax = 0.0f;
        for (int n = n0; n < n1; ++n)
            for (int c = 0; c < d; ++c) {
                float ks = bf16_to_float(k[(int64_t)n * k_rs + c]) - k_mean[c];
                float a = fabsf(ks);
                if (a > amax) amax = a;
            }
        float inv = amax > 0.0f ? 127.0f / amax : 0.0f;
        k_scale[b] = amax > 0.0f ? amax / 127.0f : 0.0f;
        for (int n = n0; n < n1; ++n)
            for (int c = 0; c < d; ++c) {
                float ks = bf16_to_float(k[(int64_t)n * k_rs + c]) - k_mean[c];
                k_i8[(int64_t)n * d + c] = amax > 0.0f ? int8_code(ks, inv) : 0;
            }
    }
    /* V per channel */
    for (int c = 0; c < d; ++c) {
        float amax = 0.0f;
        for (int n = 0; n < N; ++n) {
            float a = fabsf(bf16_to_float(v[(int64_t)n * v_rs + c]));
            if (a > amax) amax = a;
        }
        float inv = amax > 0.0f ? 448.0f / amax : 0.0f;
        v_scale[c] = amax > 0.0f ? amax / 448.0f : 0.0f;
        for (int n = 0; n < N; ++n) {
            float x = bf16_to_float(v[(int64_t)n * v_rs + c]) * inv;
            v_e4m3[(int64_t)n * d + c] = amax > 0.0f ? oracle_e4m3_encode((double)x) : 0;
        }
    }
    return 0;
}

/*
 * K-residual quantization of K for one slab ("ComfyUI-sol-attn", 核心亮点
 * item 1: quantize only the residual of K inside each block, keep the mean
 * term at bf16 precision).  Readings where the page is silent: the blocks are
 * the 64-token K blocks of reading C3; the block mean is the fp64 mean over
 * the block's valid tokens, rounded to bf16 (RNE); the residual k - mean is
 * formed in fp32 (exact: both are bf16 values) and coded as in reading C2 with
 * the block's amax of the residual.
 *   k_bmean[nkb][d] (bf16 bit patterns), k_i8[N][d], k_scale[nkb].
 */
int oracle_quantize_kres(const uint16_t *k, int64_t k_rs, int N, int d,
                         int8_t *k_i8, float *k_scale, uint16_t *k_bmean)
{
    if (N <= 0 || d <= 0) return -1;
    int nkb = (N + ORACLE_K_BLOCK - 1) / ORACLE_K_BLOCK;
    for (int b = 0; b < nkb; ++b) {
        int n0 = b * ORACLE_K_BLOCK, n1 = n0 + ORACLE_K_BLOCK;
        if (n1 > N) n1 = N;
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int n = n0; n < n1; ++n) acc += oracle_bf16_to_double(k[(int64_t)n * k_rs + c]);
            k_bmean[(size_t)b * d + c] = oracle_bf16_rne(acc / (double)(n1 - n0));
        }
        float amax = 0.0f;
        for (int n = n0; n < n1; ++n)
            for (int c = 0; c < d; ++c) {
                float r = bf16_to_float(k[(int64_t)n * k_rs + c]) - bf16_to_float(k_bmean[(size_t)b * d + c]);
                float a = fabsf(r);
                if (a > amax) amax = a;
            }
        float inv = amax > 0.0f ? 127.0f / amax : 0.0f;
        k_scale[b] = amax > 0.0f ? amax / 127.0f : 0.0f;
        for (int n = n0; n < n1; ++n)
            for (int c = 0; c < d; ++c) {
                float r = bf16_to_float(k[(int64_t)n * k_rs + c]) - bf16_to_float(k_bmean[(size_t)b * d + c]);
                k_i8[(int64_t)n * d + c] = amax > 0.0f ? int8_code(r, inv) : 0;
            }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Quant-emulation attention                                                */
/* ------------------------------------------------------------------------ */

/* Switches for the error sources (all 1 = the scheme as specified). */
typedef struct {
    int int8_qk;    /* 0: scores from the exact smoothed product q.(k-mean)   */
    int fp8_p;      /* 0: P kept unrounded                                     */
    int fp8_v;      /* 0: V kept exact (no e4m3, no scale)                      */
    int round_bf16; /* 0: out_bf16 still written, but from the unrounded value */
    int smooth_k;   /* 0: no mean subtraction before K quantization            */
    int k_residual; /* 1: K-residual quantization (oracle_quantize_kres) instead
                       of the smoothing; the scores then add q.mean_block     */
} oracle_quant_flags;

/*
 * For each requested query row r of one slab:
 *   S_rj   = sum_c qcode[r,c] * kcode[j,c]                 (exact integer)
 *   c_rj   = fp32( fp32(q_scale[r/128] * s_l2) * k_scale[j/64] ),
 *            s_l2 = fp32(fp32(sm_scale) * fp32(log2 e))    (reading C4)
 *   x_rj   = S_rj * c_rj                                   (fp64; log2 units)
 *   m_r    = ceil(max_j x_rj)                              (reading C5)
 *   p_rj   = 2^(x_rj - m_r)            l_r = sum_j p_rj   (fp64, unrounded)
 *   P_rj   = e4m3_rn_satfinite(448 p_rj)                   (reading C6)
 *   O_rc   = sum_j P_rj * vcode_value[j,c]                 (fp64)
 *   out_rc = bf16_rne( O_rc * v_scale[c] / (448 l_r) )    (reading C8)
 * The dropped smoothing term q.mean is a per-row constant of the scores and
 * cancels in the softmax (reading C1).  With k_residual the K codes are those
 * of oracle_quantize_kres and x_rj gains e_rb = (q_r . mean_b) * sm_scale *
 * log2 e for the key's block b (fp64 from the bf16 values): that term varies
 * with the block, so it is kept, at the mean's bf16 precision.  Because m_r lies on the integer grid,
 * a tiled online evaluation that rescales by 2^(m_old - m_new) produces the
 * same P codes as this one-pass form wherever 448 p stays in e4m3's normal
 * range (reading C5); below it (448 p < 2^-6) the one-pass form is used.
 * out_f64 (may be NULL) receives the value before the bf16 rounding,
 * out_bf16 (may be NULL) the rounded bit pattern; both [nrows][d].
 */
int oracle_attn_quant_masked(const uint16_t *q, int64_t q_rs,
                             const uint16_t *k, int64_t k_rs,
                             const uint16_t *v, int64_t v_rs,
                             int N, int d, float sm_scale,
                             const oracle_quant_flags *flags,
                             const uint8_t *keep,
                             const int32_t *rows, int nrows,
                             double *out_f64, uint16_t *out_bf16)
{
    /* keep (may be NULL = every key): [nt][nt] with nt = ceil(N/128); key j
     * takes part in row r's softmax iff keep[(r/128)*nt + j/128] != 0.  A row
     * whose tile keeps no key tile has no softmax: its output is 0. */
    const int nt = (N + ORACLE_SEL_TILE - 1) / ORACLE_SEL_TILE;
    if (N <= 0 || d <= 0 || !flags) return -1;
    int nqb = (N + ORACLE_Q_BLOCK - 1) / ORACLE_Q_BLOCK;
    int nkb = (N + ORACLE_K_BLOCK - 1) / ORACLE_K_BLOCK;
    size_t nd = (size_t)N * (size_t)d;
    int8_t *qc = (int8_t *)malloc(nd), *kc = (int8_t *)malloc(nd);
    uint8_t *vc = (uint8_t *)malloc(nd);
    float *qs = (float *)malloc(sizeof(float) * nqb), *ks = (float *)malloc(sizeof(float) * nkb);
    float *km = (float *)malloc(sizeof(float) * d), *vs = (float *)malloc(sizeof(float) * d);
    double *x = (double *)malloc(sizeof(double) * (size_t)N);
    double *vval = (double *)malloc(sizeof(double) * nd);
    double *o = (double *)malloc(sizeof(double) * (size_t)d);
    uint16_t *kbm = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)nkb * d);
    double *e = (double *)malloc(sizeof(double) * (size_t)nkb);
    int rc = 0;
    if (!qc || !kc || !vc || !qs || !ks || !km || !vs || !x || !vval || !o || !kbm || !e) { rc = -2; goto done; }

    rc = oracle_quantize(q, q_rs, k, k_rs, v, v_rs, N, d, flags->k_residual ? 0 : flags->smooth_k,
                         qc, qs, kc, ks, km, vc, vs);
    if (!rc && flags->k_residual) rc = oracle_quantize_kres(k, k_rs, N, d, kc, ks, kbm);
    if (rc) goto done;

    /* value of V used in the P.V product, already multiplied by its scale */
    for (int n = 0; n < N; ++n)
        for (int c = 0; c < d; ++c)
            vval[(size_t)n * d + c] =
                flags->fp8_v ? oracle_e4m3_decode(vc[(size_t)n * d + c]) * (double)vs[c]
                             : oracle_bf16_to_double(v[(int64_t)n * v_rs + c]);

    const float log2e_f = (float)1.4426950408889634; /* log2(e) rounded to fp32 */
    const float s_l2 = sm_scale * log2e_f;           /* one fp32 multiply */

    for (int ri = 0; ri < nrows; ++ri) {
        int r = rows[ri];
        if (r < 0 || r >= N) { rc = -3; goto done; }
        float sq = qs[r / ORACLE_Q_BLOCK];
        float cq = sq * s_l2; /* fp32 */
        double xmax = -INFINITY;
        for (int b = 0; b < nkb; ++b) {
            double acc = 0.0;
            if (flags->k_residual)
                for (int c = 0; c < d; ++c)
                    acc += oracle_bf16_to_double(q[(int64_t)r * q_rs + c]) *
                           oracle_bf16_to_double(kbm[(size_t)b * d + c]);
            e[b] = acc * (double)sm_scale * 1.4426950408889634;
        }
        const uint8_t *krow = keep ? keep + (size_t)(r / ORACLE_SEL_TILE) * nt : NULL;
        for (int j = 0; j < N; ++j) {
            if (krow && !krow[j / ORACLE_SEL_TILE]) {
                x[j] = -INFINITY; /* skipped key tile */
                continue;
            }
            if (flags->int8_qk) {
                int64_t S = 0;
                for (int c = 0; c < d; ++c)
                    S += (int64_t)qc[(size_t)r * d + c] * (int64_t)kc[(size_t)j * d + c];
                float cj = cq * ks[j / ORACLE_K_BLOCK]; /* fp32 */
                x[j] = (double)S * (double)cj + e[j / ORACLE_K_BLOCK];
            } else {
                double acc = 0.0;
                for (int c = 0; c < d; ++c) {
                    const double kj = oracle_bf16_to_double(k[(int64_t)j * k_rs + c]);
                    const double sub = flags->k_residual
                                           ? oracle_bf16_to_double(kbm[(size_t)(j / ORACLE_K_BLOCK) * d + c])
                                           : (flags->smooth_k ? (double)km[c] : 0.0);
                    acc += oracle_bf16_to_double(q[(int64_t)r * q_rs + c]) * (kj - sub);
                }
                x[j] = acc * (double)sm_scale * 1.4426950408889634 + e[j / ORACLE_K_BLOCK];
            }
            if (x[j] > xmax) xmax = x[j];
        }
        if (xmax == -INFINITY) { /* no key kept */
            for (int c = 0; c < d; ++c) {
                if (out_f64) out_f64[(size_t)ri * d + c] = 0.0;
                if (out_bf16) out_bf16[(size_t)ri * d + c] = 0;
            }
            continue;
        }
        double m = ceil(xmax);
        double l = 0.0;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        for (int j = 0; j < N; ++j) {
            double p = exp2(x[j] - m);
            l += p;
            double P = flags->fp8_p ? oracle_e4m3_round(p * ORACLE_E4M3_MAX) : p * ORACLE_E4M3_MAX;
            if (P == 0.0) continue;
            for (int c = 0; c < d; ++c) o[c] += P * vval[(size_t)j * d + c];
        }
        for (int c = 0; c < d; ++c) {
            double y = o[c] / (ORACLE_E4M3_MAX * l);
            if (out_f64) out_f64[(size_t)ri * d + c] = y;
            if (out_bf16) out_bf16[(size_t)ri * d + c] = oracle_bf16_rne(y);
        }
    }
done:
    free(qc); free(kc); free(vc); free(qs); free(ks); free(km); free(vs);
    free(x); free(vval); free(o); free(kbm); free(e);
    return rc;
}

int oracle_attn_quant(const uint16_t *q, int64_t q_rs,
                      const uint16_t *k, int64_t k_rs,
                      const uint16_t *v, int64_t v_rs,
                      int N, int d, float sm_scale,
                      const oracle_quant_flags *flags,
                      const int32_t *rows, int nrows,
                      double *out_f64, uint16_t *out_bf16)
{
    return oracle_attn_quant_masked(q, q_rs, k, k_rs, v, v_rs, N, d, sm_scale, flags, NULL, rows, nrows,
                                    out_f64, out_bf16);
}

/* ------------------------------------------------------------------------ */
/* Block-sparse skipping ("ComfyUI-sol-attn", 核心亮点 item 4 and its node   */
/* table: a sparsity value tau that may ramp over the sampling steps, sparse */
/* early and dense late).  The page names the control only; the readings    */
/* S1-S4 below are this project's.                                          */
/* ------------------------------------------------------------------------ */

/* Reading S1/S2 -- tiles and their score.  Queries and keys are cut into
 * tiles of 128 tokens (the Q quantization block; two K blocks).  The score of
 * (query tile i, key tile j) is the mean of the dequantized scores x_rs over
 * the tile pair, in log2 units:
 *     sbar_ij = (sum_r q_r) . (sum_s k_s) * fp32(sm_scale*log2 e) / (n_i n_j)
 * with q_r = q_scale(r) * qcode_r, k_s = k_scale(s) * kcode_s.  It is
 * computed in IEEE fp32 in this exact order, one rounding per operation:
 *     qs_i[c] = q_scale[i] * float(sum of Q codes of tile i, channel c)
 *     ks_j[c] = k_scale[2j] * float(sum over K block 2j)
 *             + k_scale[2j+1] * float(sum over K block 2j+1)
 *     dot     = (((0 + qs[0] ks[0]) + qs[1] ks[1]) + ...)     (c ascending)
 *     sbar    = (dot * s_l2) / float(n_i * n_j)
 * (the code sums are exact integers, so everything before the first fp32
 * product is order-independent).  Padded tokens (n >= N) take no part.
 * sbar is [nt][nt] row-major; q_scale has ceil(N/128) and k_scale ceil(N/64)
 * entries. */
int oracle_block_scores(const int8_t *qc, const float *qs, const int8_t *kc, const float *ks,
                        int N, int d, float sm_scale, float *sbar)
{
    if (N <= 0 || d <= 0) return -1;
    const int nt = (N + ORACLE_SEL_TILE - 1) / ORACLE_SEL_TILE;
    const int nkb = (N + ORACLE_K_BLOCK - 1) / ORACLE_K_BLOCK;
    float *qv = (float *)malloc(sizeof(float) * (size_t)nt * d);
    float *kv = (float *)malloc(sizeof(float) * (size_t)nt * d);
    if (!qv || !kv) { free(qv); free(kv); return -2; }
    for (int i = 0; i < nt; ++i) {
        const int r0 = i * ORACLE_SEL_TILE;
        for (int c = 0; c < d; ++c) {
            int64_t sq = 0, sa = 0, sb = 0;
            for (int r = r0; r < r0 + ORACLE_SEL_TILE && r < N; ++r) {
                sq += qc[(size_t)r * d + c];
                if (r < r0 + ORACLE_K_BLOCK) sa += kc[(size_t)r * d + c];
                else sb += kc[(size_t)r * d + c];
            }
            qv[(size_t)i * d + c] = qs[i] * (float)sq;
            const float kb0 = ks[2 * i] * (float)sa;
            const float kb1 = (2 * i + 1 < nkb ? ks[2 * i + 1] : 0.f) * (float)sb;
            kv[(size_t)i * d + c] = kb0 + kb1;
        }
    }
    const float s_l2 = sm_scale * (float)1.4426950408889634;
    for (int i = 0; i < nt; ++i) {
        const int ni = (N - i * ORACLE_SEL_TILE) < ORACLE_SEL_TILE ? N - i * ORACLE_SEL_TILE : ORACLE_SEL_TILE;
        for (int j = 0; j < nt; ++j) {
            const int nj = (N - j * ORACLE_SEL_TILE) < ORACLE_SEL_TILE ? N - j * ORACLE_SEL_TILE : ORACLE_SEL_TILE;
            float dot = 0.f;
            for (int c = 0; c < d; ++c) {
                const float prod = qv[(size_t)i * d + c] * kv[(size_t)j * d + c];
                dot = dot + prod;
            }
            const float num = dot * s_l2;
            sbar[(size_t)i * nt + j] = num / (float)(ni * nj);
        }
    }
    free(qv);
    free(kv);
    return 0;
}

/* Reading S3 -- which key tiles a query tile keeps.  Everything is IEEE fp32
 * with one rounding per operation, in this order, so that any implementation
 * following it gets the same bits:
 *   rank     key tiles by sbar descending, ties by the lower index;
 *   top      = sbar at rank 0;
 *   w_t      = float(n_j) * e2(sbar_j - top)  for the tile j at rank t;
 *   total    = (((0 + w_0) + w_1) + ...)      in rank order;
 *   lim      = tau * total                    (tau rounded to fp32);
 *   rank t is kept iff before_t < lim, with before_0 = 0 and
 *   before_{t+1} = before_t + w_t.
 * So the kept set is the shortest prefix of the ranking whose mass reaches
 * tau of the total; rank 0 is always kept, and tau >= 1 keeps every tile.
 * e2(x) for x <= 0 is 2^x evaluated as: 0 if x < -64 (such a tile weighs
 * less than 2^-64 of the top one); else k = floor(x), f = x - k, p = the
 * Taylor polynomial of 2^f = e^(f ln 2) to degree 8 by Horner (coefficients
 * (ln 2)^i / i! rounded to fp32; p = p*f then p = p + c_i, separately
 * rounded), and e2 = p * 2^k (exact).  On [0, 1] the polynomial is within
 * 2e-7 of 2^f; the selection only needs the order of magnitude of each mass,
 * the fixed arithmetic is what makes it reproducible.  keep is [nt][nt]. */
static float s3_exp2(float x)
{
    if (!(x >= -64.0f)) return 0.0f;
    float c[9];
    double fact = 1.0;
    for (int i = 0; i <= 8; ++i) {
        if (i > 0) fact *= (double)i;
        c[i] = (float)(pow(0.69314718055994530942, (double)i) / fact);
    }
    const float k = floorf(x);
    const float f = x - k;
    float p = c[8];
    for (int i = 7; i >= 0; --i) {
        p = p * f;
        p = p + c[i];
    }
    return ldexpf(p, (int)k);
}

int oracle_block_select(const float *sbar, int N, double tau, uint8_t *keep)
{
    if (N <= 0 || !(tau > 0.0)) return -1;
    const float tau32 = (float)tau;
    const int nt = (N + ORACLE_SEL_TILE - 1) / ORACLE_SEL_TILE;
    int *order = (int *)malloc(sizeof(int) * (size_t)nt);
    float *w = (float *)malloc(sizeof(float) * (size_t)nt);
    if (!order || !w) { free(order); free(w); return -2; }
    for (int i = 0; i < nt; ++i) {
        const float *row = sbar + (size_t)i * nt;
        uint8_t *kr = keep + (size_t)i * nt;
        if (tau32 >= 1.0f) {
            for (int j = 0; j < nt; ++j) kr[j] = 1;
            continue;
        }
        /* insertion sort: sbar descending, index ascending on ties */
        for (int j = 0; j < nt; ++j) {
            int t = j;
            while (t > 0 && (row[order[t - 1]] < row[j] || (row[order[t - 1]] == row[j] && order[t - 1] > j))) {
                order[t] = order[t - 1];
                --t;
            }
            order[t] = j;
        }
        const float top = row[order[0]];
        float total = 0.0f;
        for (int t = 0; t < nt; ++t) {
            const int j = order[t];
            const int nj = (N - j * ORACLE_SEL_TILE) < ORACLE_SEL_TILE ? N - j * ORACLE_SEL_TILE : ORACLE_SEL_TILE;
            w[t] = (float)nj * s3_exp2(row[j] - top);
            total = total + w[t];
        }
        const float lim = tau32 * total;
        for (int j = 0; j < nt; ++j) kr[j] = 0;
        float before = 0.0f;
        for (int t = 0; t < nt && before < lim; ++t) {
            kr[order[t]] = 1;
            before = before + w[t];
        }
    }
    free(order);
    free(w);
    return 0;
}

/* Array form of the selection's exponential, for the tests. */
void oracle_s3_exp2_array(const float *x, int64_t n, float *y)
{
    for (int64_t i = 0; i < n; ++i) y[i] = s3_exp2(x[i]);
}

/* Integer score tile from given codes: s[i][j] = sum_c a[i][c] * b[j][c]
 * for i < m, j < n (row-major codes with row strides a_rs, b_rs).  This is
 * the definition of the INT8 product with int32 accumulation; |s| <= d*127^2
 * fits int32 for d <= 133000. */
int oracle_int8_gemm_nt(const int8_t *a, int64_t a_rs, const int8_t *b, int64_t b_rs,
                        int m, int n, int d, int32_t *s)
{
    for (int i = 0; i < m; ++i)
        for (int j = 0; j < n; ++j) {
            int64_t acc = 0;
            for (int c = 0; c < d; ++c)
                acc += (int64_t)a[(int64_t)i * a_rs + c] * (int64_t)b[(int64_t)j * b_rs + c];
            s[(int64_t)i * n + j] = (int32_t)acc;
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Array forms of the format helpers (for the tests)                        */
/* ------------------------------------------------------------------------ */

void oracle_e4m3_encode_array(const double *x, int64_t n, uint8_t *code)
{
    for (int64_t i = 0; i < n; ++i) code[i] = oracle_e4m3_encode(x[i]);
}

void oracle_e4m3_decode_array(const uint8_t *code, int64_t n, double *x)
{
    for (int64_t i = 0; i < n; ++i) x[i] = oracle_e4m3_decode(code[i]);
}

void oracle_bf16_rne_array(const double *x, int64_t n, uint16_t *h)
{
    for (int64_t i = 0; i < n; ++i) h[i] = oracle_bf16_rne(x[i]);
}
