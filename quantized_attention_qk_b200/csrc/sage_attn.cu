// sage_attn.cu -- fused quantized attention kernel for sm_100a.
//
// One CTA computes two 128-query tiles of one (batch, head) against all keys,
// 128 keys per step, never writing the score matrix out
// ("GitHub榜单静默期：Attention优化从架构转向推理加速", section 2.2).  Scores come
// from INT8 tensor-core products and P.V from FP8 (e4m3) products
// ("MiniMax H3 接入 SageAttention 实测加速", section 一).
//
// Warp roles (384 threads, three warpgroups):
//   warpgroup t (warps 4t..4t+3), t = 0, 1: softmax of Q tile t, one query row
//              per thread; the two warpgroups run independently of each other
//   warp 8     TMA producer: both Q tiles once, then a ring of (K, V) stages
//   warp 9     tensor-memory allocator and single-thread tcgen05.mma issuer
//   warps 10-11 idle
// After set-up the softmax warpgroups raise their register limit to 216 and
// warpgroup 2 lowers its own to 64 (setmaxnreg).
// V tiles are loaded token-major (key rows of d channels) and fed to the P.V MMA
// as an MN-major operand.
// Tensor memory (512 columns x 128 lanes): S0, S1 (int32, 128 columns each) at
// [0,256), O0, O1 (fp32, d columns each) from 256.
// P (e4m3) goes to shared memory, two buffers per tile, in the 128-byte-swizzled
// K-major layout the P.V MMA reads.  A warpgroup releases S(j) as soon as it
// holds it in registers, so the tensor core computes S(j+1) while the softmax
// of step j runs.  MMA order per step j:
//   S0(j+1), S1(j+1)   (each once its tile released S(j) and K(j+1) is loaded)
//   PV0(j), PV1(j)     (each once its tile posted P(j) and rescaled O)
// Barriers a waiter tracks by phase parity never get two phases ahead of it:
// "P ready" has one barrier per P buffer, and the epilogue waits on a barrier
// committed once after the tile's last PV.
// Block-sparse instantiation (SPARSE): each Q tile attends only to the key
// tiles its row of a bit mask selects.  Three warps turn the two mask rows into
// step lists in shared memory at the start (tile 0's key tiles, tile 1's, and
// their union with a flag per entry saying which tiles attend), so a step costs
// one shared load per role.  The producer streams the union through the ring;
// each tile's QK and PV MMAs, barriers and P buffers advance with the tile's
// own step count; a tile that keeps no key tile writes zeros.
// Prologue-quantized Q (FUSED_Q): the producer loads the bf16 rows of both
// tiles into the P buffers (idle until the first P is stored); each softmax
// warpgroup takes its tile's |max| (each thread its row, the four warps
// combined through shared memory) and codes the rows into the swizzled INT8
// Q tile with the quantize pass's arithmetic, so the codes are the same and
// the quantize pass codes K and V only.  No P is stored before S(0), which
// waits for all eight warps' codes.
// K-residual instantiation (KRES): K holds the codes of its residual inside
// each 64-token block, and every score gains that block's mean term
// e[row][b] = (q_row . mean_b) * sm_scale * log2 e; each 128-key step covers
// two blocks, so e folds into the two per-half offsets the exponent already
// takes (no work per score).  The CTA computes e for its 256 rows and every
// block in a prologue, while tensor memory and the ring / P buffers are still
// free: the producer loads the tiles' bf16 Q rows (into the ring's last two
// stages) and up to 256 block means at a time (into the P buffers; 128-byte
// swizzle) while the ring's first stage takes K/V tiles, the MMA warp
// multiplies them on the tensor cores (tcgen05 kind::f16, bf16 x bf16 ->
// fp32, M = 128, N <= 256, one accumulator per tile), and the softmax warps
// scale each row's values and keep them in a
// per-SM scratch slot [block][256 rows] (one CTA per SM at a time, so the
// slot of the SM the CTA runs on is its own), which the same threads read back
// one step ahead in the main loop.
// Numerics (readings C4-C8): x = S*(sq*sm_scale*log2e*sk) with one sk per
// 64-key block; running max m' = max(m, ceil(rowmax x)) so that the O / l
// rescale 2^(m-m') is an exact power of two; P = e4m3(2^(x-m') * 448) computed as
// 2^(x - m' + log2 448); l accumulates the unrounded values; the epilogue
// writes bf16(O * v_scale / l), staging each warp's rows in its tile's (then
// idle) P buffers so that every store instruction covers whole output rows.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {

__device__ unsigned g_device_error = 0;
static_assert(kErrTimeout == kErrTimeoutBit, "device and host disagree on the timeout bit");

namespace {

template <int D>
struct Cfg {
    static constexpr int BM = 128;                 // queries per tile
    static constexpr int BN = kKvTile;             // keys per step
    static constexpr int STAGES = 3;
    static constexpr int Q_BYTES = BM * D;
    static constexpr int K_BYTES = BN * D;
    static constexpr int V_BYTES = BN * D;          // V tile: BN key rows of d e4m3 channels
    static constexpr int P_BYTES = BM * BN;        // one P buffer (e4m3)
    static constexpr int TILE_BYTES = 2 * Q_BYTES + STAGES * (K_BYTES + V_BYTES) + 4 * P_BYTES;
    static constexpr uint32_t T_O = 256;           // O of tile t at 256 + d t
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int THREADS = 384;            // three warpgroups
    static constexpr int LAUNCH_REGS = 168;        // per thread, what 384 threads x 1 block allow
    static constexpr uint32_t SOFTMAX_REGS = 216;  // warpgroups 0 and 1 after setmaxnreg
    static constexpr uint32_t OTHER_REGS = 72;     // warpgroup 2 (TMA, MMA, two idle warps)
    static_assert(2 * 128 * SOFTMAX_REGS + 128 * OTHER_REGS <= LAUNCH_REGS * THREADS,
                  "register split exceeds the registers the block is launched with");
};

template <int D>
struct Ctl {
    uint64_t q_full;
    uint64_t kv_full[Cfg<D>::STAGES];
    uint64_t kv_empty[Cfg<D>::STAGES];
    uint64_t s_full[2];     // per tile: S(j) computed
    uint64_t s_free[2];     // per tile: the softmax holds S(j) in registers
    uint64_t p_ready[2][2]; // [tile][P buffer]: P(j) in shared memory and O rescaled
    uint64_t o_done[2];     // per tile: PV of a step completed
    uint64_t o_final[2];    // per tile: every PV of the tile completed (committed once)
    uint64_t drain;
    uint64_t qb_full;       // FUSED_Q: the bf16 Q rows landed
    uint64_t q_amax_bar[2]; // FUSED_Q, per tile: the four warps posted their |max|
    uint64_t mb_full[1];    // KRES prologue: a chunk of block means landed
    uint64_t e_full[1];     // KRES prologue: a chunk's mean-term products are in tensor memory
    uint64_t e_free[1];     // KRES prologue: the softmax warps took them out
    float q_amax[2][4];
    int steps[3];           // SPARSE: own steps of tile 0, of tile 1, union steps
    uint32_t tmem_base;
    AbortState abort;
    float v_scale[D];
};

// At least 120 KB so that a second CTA never shares the SM: each CTA takes
// all 512 tensor-memory columns.  (The tiles need more than that anyway.)
template <int D>
constexpr int smem_bytes(int extra = 0) {
    const int need = Cfg<D>::TILE_BYTES + static_cast<int>(sizeof(Ctl<D>)) + extra + 1024;
    return need > 120 * 1024 ? need : 120 * 1024;
}

struct AttnParams {
    const float *q_scale;  // [BH][nqb]
    const float *k_scale;  // [BH][nkb]
    const float *v_scale;  // [BH][D]
    uint16_t *out;         // bf16
    int64_t osb, osh, osn;
    int H, N, nqb, nkb;
    float s_l2;            // fp32(sm_scale * fp32(log2 e))
    unsigned *err;
    // debug export of one S tile (EXPORT_S instantiation only)
    int32_t *s_export;
    int bh0, q_tile0, kv_tile0;
    // SPARSE instantiation: [BH][nqb][mask_words], bit j of row (bh, i) set =
    // query tile i attends to key tile j
    const uint32_t *kv_mask;
    int mask_words;
    // KRES instantiation: per-SM scratch slots of the mean term, [n_slots][nkb][256]
    float *eslot;
    int n_slots;
    int q_swap;            // FUSED_Q, KRES: the bf16 Q map takes H before N
};

// Step lists of the SPARSE instantiation, built by one warp from mask rows r0
// (and r1, may be null) of `words` words, bits at or past n ignored: the
// indices of the set bits of r0 | r1 in ascending order go to list[], and, if
// flags is not null, flags[k] = (bit in r0) | (bit in r1) << 1.  Returns the
// count (every lane).
__device__ __forceinline__ int build_steps(const uint32_t *r0, const uint32_t *r1, int words, int n, uint16_t *list,
                                           uint8_t *flags) {
    const int lane = threadIdx.x & 31;
    int count = 0;
    for (int w0 = 0; w0 < words; w0 += 32) {
        const int w = w0 + lane;
        uint32_t a = 0u, b = 0u;
        if (w < words) {
            const uint32_t keep = (w == words - 1 && (n & 31)) ? (1u << (n & 31)) - 1u : ~0u;
            a = (r0 ? __ldg(r0 + w) : 0u) & keep;
            b = (r1 ? __ldg(r1 + w) : 0u) & keep;
        }
        uint32_t bits = a | b;
        const int c = __popc(bits);
        int incl = c;  // inclusive scan of the lanes' counts
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += o;
        }
        int pos = count + incl - c;
        while (bits) {
            const int bit = __ffs(bits) - 1;
            bits &= bits - 1u;
            list[pos] = static_cast<uint16_t>((w << 5) + bit);
            if (flags) flags[pos] = static_cast<uint8_t>(((a >> bit) & 1u) | (((b >> bit) & 1u) << 1));
            ++pos;
        }
        count += __shfl_sync(0xffffffffu, incl, 31);
    }
    return count;
}

// 2^k for an integer-valued k <= 0 (exact; 0 below the normal range).
__device__ __forceinline__ float exp2_int(float k) {
    const int e = 127 + static_cast<int>(k);
    return e > 0 ? __int_as_float(e << 23) : 0.f;
}

// Largest of the 64 scores in a/b (columns col0.. of the step; with MASK,
// columns at or past n_valid are left out; INT_MIN if none is valid).
template <bool MASK>
__device__ __forceinline__ int row_max64(const uint32_t (&a)[32], const uint32_t (&b)[32], int col0, int n_valid) {
    int m0 = INT_MIN, m1 = INT_MIN;  // two independent chains
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
        int a0 = static_cast<int>(a[i]), a1 = static_cast<int>(a[i + 1]);
        int b0 = static_cast<int>(b[i]), b1 = static_cast<int>(b[i + 1]);
        if (MASK) {
            if (col0 + i >= n_valid) a0 = INT_MIN;
            if (col0 + i + 1 >= n_valid) a1 = INT_MIN;
            if (col0 + 32 + i >= n_valid) b0 = INT_MIN;
            if (col0 + 32 + i + 1 >= n_valid) b1 = INT_MIN;
        }
        m0 = __vimax3_s32(m0, a0, a1);
        m1 = __vimax3_s32(m1, b0, b1);
    }
    return max(m0, m1);
}

// 2^y for two values on the FMA pipe instead of the MUFU unit (16 ex2 per
// clock per SM, the softmax's limit when both warpgroups exponentiate at once).
// y = j + f with j the nearest integer (rounded by adding and subtracting
// 1.5 * 2^23) and f in [-1/2, 1/2]; 2^f by a degree-4 polynomial (Horner),
// then j is added to the exponent field.  The coefficients minimise the
// relative error of 2^f on [-1/2, 1/2] (weighted least squares iterated to
// equal ripple); evaluated in fp32 the relative error stays below 3e-6.  y is
// clamped at -120 so the exponent cannot underflow (2^-120 is 0 in e4m3).
__device__ __forceinline__ void exp2_poly2(float y0, float y1, float &p0, float &p1) {
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    constexpr float c0 = 0.9999992847442627f, c1 = 0.6931218504905701f, c2 = 0.240247443318367f,
                    c3 = 0.05591757968068123f, c4 = 0.009569989517331123f;
    y0 = fmaxf(y0, -120.f);
    y1 = fmaxf(y1, -120.f);
    float t0, t1, j0, j1, f0, f1, q0, q1;
    fadd2(t0, t1, y0, y1, kRound, kRound);       // integer part in the low mantissa bits
    fadd2(j0, j1, t0, t1, -kRound, -kRound);     // j as a float
    ffma2(f0, f1, j0, j1, -1.f, -1.f, y0, y1);   // f = y - j, exact
    ffma2(q0, q1, c4, c4, f0, f1, c3, c3);
    ffma2(q0, q1, q0, q1, f0, f1, c2, c2);
    ffma2(q0, q1, q0, q1, f0, f1, c1, c1);
    ffma2(q0, q1, q0, q1, f0, f1, c0, c0);
    // the low bits of t hold j (two's complement); j << 23 lands in the exponent
    p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
    p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

// 448 * 2^(x - m) for 32 scores, x = S * c: y = float(S) * c + (log2 448 - m)
// (one FMA per pair), p = 2^y: the MUFU ex2 for six of every eight scores,
// the polynomial above for the other two.  Accumulates the unrounded p into acc
// and packs the e4m3 codes four per word into w[0..7] (word j holds keys
// 4j..4j+3, lowest key in the lowest byte).
template <bool MASK>
__device__ __forceinline__ void p_pack32(const uint32_t (&r)[32], float c, float nb, int col0, int n_valid,
                                         float (&acc)[4], uint32_t *w) {
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
        float y[4], pv[4];
        ffma2(y[0], y[1], static_cast<float>(static_cast<int>(r[i])), static_cast<float>(static_cast<int>(r[i + 1])),
              c, c, nb, nb);
        ffma2(y[2], y[3], static_cast<float>(static_cast<int>(r[i + 2])),
              static_cast<float>(static_cast<int>(r[i + 3])), c, c, nb, nb);
        pv[0] = ex2_approx(y[0]);
        pv[1] = ex2_approx(y[1]);
        if ((i & 4) == 0) {
            pv[2] = ex2_approx(y[2]);
            pv[3] = ex2_approx(y[3]);
        } else {
            exp2_poly2(y[2], y[3], pv[2], pv[3]);
        }
        if (MASK) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (col0 + i + e >= n_valid) pv[e] = 0.f;
        }
        fadd2(acc[0], acc[1], acc[0], acc[1], pv[0], pv[1]);
        fadd2(acc[2], acc[3], acc[2], acc[3], pv[2], pv[3]);
        w[i / 4] = cvt_e4m3x2(pv[0], pv[1]) | (cvt_e4m3x2(pv[2], pv[3]) << 16);
    }
}

// Row `row` of a 128-byte-swizzled K-major tile (8-row atoms of 1024 bytes):
// 16-byte chunk c of the row lives at row*128 + ((c ^ (row & 7)) * 16).
__device__ __forceinline__ void store_p_row(uint32_t tile, int row, const uint32_t (&w)[32]) {
    const uint32_t rbase = tile + row * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c)
        st_shared_v4(rbase + ((c ^ (row & 7)) << 4), w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

template <int D, bool EXPORT_S, bool SPARSE, bool KRES, bool FUSED_Q>
__global__ void __launch_bounds__(Cfg<D>::THREADS, 1)
    k_attn(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_qb,
           const __grid_constant__ CUtensorMap tm_mean, const AttnParams p) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = base;
    uint8_t *sK = base + 2 * C::Q_BYTES;
    uint8_t *sV = sK + C::STAGES * C::K_BYTES;
    uint8_t *sP = sV + C::STAGES * C::V_BYTES;  // [tile][buffer] P tiles
    Ctl<D> *ctl = reinterpret_cast<Ctl<D> *>(sP + 4 * C::P_BYTES);
    // SPARSE step lists: tile 0's and tile 1's key tiles, the union, its flags
    uint16_t *slist = reinterpret_cast<uint16_t *>(ctl + 1);
    uint16_t *ulist = slist + 2 * (SPARSE ? p.nqb : 0);
    uint8_t *uflag = reinterpret_cast<uint8_t *>(ulist + (SPARSE ? p.nqb : 0));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = EXPORT_S ? p.bh0 : static_cast<int>(blockIdx.y);
    const int qt0 = EXPORT_S ? p.q_tile0 : 2 * static_cast<int>(blockIdx.x);
    const int kv0 = EXPORT_S ? p.kv_tile0 : 0;
    const int nkv = EXPORT_S ? 1 : (p.N + C::BN - 1) / C::BN;

    if (threadIdx.x == 0) {
        mbar_init(&ctl->q_full, FUSED_Q ? 8 : 1);  // the softmax warps' codes, or the TMA
        mbar_init(&ctl->qb_full, 1);
        mbar_init(&ctl->q_amax_bar[0], 4);
        mbar_init(&ctl->q_amax_bar[1], 4);
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&ctl->kv_full[s], 1);
            mbar_init(&ctl->kv_empty[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&ctl->s_full[t], 1);
            mbar_init(&ctl->s_free[t], 4);      // one arrival per softmax warp
            mbar_init(&ctl->p_ready[t][0], 4);
            mbar_init(&ctl->p_ready[t][1], 4);
            mbar_init(&ctl->o_done[t], 1);
            mbar_init(&ctl->o_final[t], 1);
        }
        mbar_init(&ctl->drain, 1);
        mbar_init(&ctl->mb_full[0], 1);
        mbar_init(&ctl->e_full[0], 1);
        mbar_init(&ctl->e_free[0], 8);
        ctl->abort.flag = 0;
        fence_barrier_init();
    }
    if (warp == 8 && lane == 0) {
        tma_prefetch_desc(FUSED_Q ? &tm_qb : &tm_q);
        tma_prefetch_desc(&tm_k);
        if (!EXPORT_S) tma_prefetch_desc(&tm_v);
        if (KRES) {
            tma_prefetch_desc(&tm_qb);
            tma_prefetch_desc(&tm_mean);
        }
    }
    // KRES prologue: chunks of up to 256 K blocks (one MMA per tile and K step,
    // tile t's products at tensor-memory columns [256 t, 256 t + 256)); the
    // chunk's means sit in the P buffers ([channel half][256 blocks][64]), the
    // bf16 Q rows of tile t in the ring's stages 1 and 2 (its K slots for tile
    // 0, its V slots for tile 1: [channel half][128 rows][64]), so stage 0
    // takes the first K/V tiles meanwhile
    constexpr int kEChunk = 256;
    uint8_t *const sQb[2] = {sK + C::K_BYTES, sV + C::V_BYTES};
    static_assert(2 * C::K_BYTES == C::BM * D * 2 && kEChunk * D * 2 <= 4 * C::P_BYTES,
                  "the prologue's operands fit the ring's last stages and the P buffers");
    const int e_chunks = KRES ? (p.nkb + kEChunk - 1) / kEChunk : 0;
    // everything below reads what the previous kernel of the stream wrote
    grid_dep_wait();
    for (int i = threadIdx.x; i < D; i += blockDim.x) ctl->v_scale[i] = EXPORT_S ? 0.f : p.v_scale[bh * D + i];
    if constexpr (SPARSE) {
        // a tile past the last query tile keeps nothing
        if (warp < 3) {
            const uint32_t *r0 = p.kv_mask + ((size_t)bh * p.nqb + qt0) * p.mask_words;
            const uint32_t *r1 = qt0 + 1 < p.nqb ? r0 + p.mask_words : nullptr;
            const int n = warp < 2 ? build_steps(warp == 0 ? r0 : r1, nullptr, p.mask_words, nkv,
                                                 slist + warp * p.nqb, nullptr)
                                   : build_steps(r0, r1, p.mask_words, nkv, ulist, uflag);
            if (lane == 0) ctl->steps[warp] = n;
        }
    }
    if (warp == 9) {
        tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;

    if (warp >= 8) regs_decrease<C::OTHER_REGS>();
    if (warp == 8) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            if (FUSED_Q) {
                // bf16 rows of both tiles into the P buffers: [tile][d/64][128 rows][64]
                const int b = bh / p.H, h = bh % p.H;
                mbar_arrive_expect_tx(&ctl->qb_full, 2 * C::BM * D * 2);
                for (int t = 0; t < 2; ++t)
                    for (int half = 0; half < D / 64; ++half)
                        for (int r = 0; r < C::BM; r += 64) {
                            uint16_t *dst = reinterpret_cast<uint16_t *>(sP) + ((t * (D / 64) + half) * C::BM + r) * 64;
                            const int n = (qt0 + t) * C::BM + r;
                            if (p.q_swap)
                                tma_load_4d(dst, &tm_qb, &ctl->qb_full, half * 64, h, n, b);
                            else
                                tma_load_4d(dst, &tm_qb, &ctl->qb_full, half * 64, n, h, b);
                        }
            } else {
                mbar_arrive_expect_tx(&ctl->q_full, 2 * C::Q_BYTES);
                tma_load_3d(sQ, &tm_q, &ctl->q_full, 0, qt0 * C::BM, bh);
                tma_load_3d(sQ + C::Q_BYTES, &tm_q, &ctl->q_full, 0, (qt0 + 1) * C::BM, bh);
            }
            bool pro_ok = true;
            int m_issued = 0;  // KRES: means chunks issued
            int issued = 0;
            const int nsteps_all = SPARSE ? ctl->steps[2] : nkv;
            auto issue_kv = [&](int j) {  // K/V tiles of step j into stage j % STAGES
                const int kt = SPARSE ? ulist[j] : j;  // key tile of step j
                const int s = j % C::STAGES;
                mbar_arrive_expect_tx(&ctl->kv_full[s], EXPORT_S ? C::K_BYTES : C::K_BYTES + C::V_BYTES);
                tma_load_3d(sK + s * C::K_BYTES, &tm_k, &ctl->kv_full[s], 0, (kv0 + kt) * C::BN, bh);
                if (!EXPORT_S)
                    tma_load_3d(sV + s * C::V_BYTES, &tm_v, &ctl->kv_full[s], 0, (kv0 + kt) * C::BN, bh);
                issued = j + 1;
            };
            if (KRES) {
                // the ring's first stage takes its K/V tiles at once
                if (nsteps_all > 0) issue_kv(0);
                // bf16 Q rows of both tiles into the ring's (still idle) stages 1
                // and 2: tile t's [channel half][128 rows][64], 128-byte swizzle
                const int b = bh / p.H, h = bh % p.H;
                mbar_arrive_expect_tx(&ctl->qb_full, 2 * C::BM * D * 2);
                for (int t = 0; t < 2; ++t)
                    for (int half = 0; half < D / 64; ++half) {
                        uint8_t *dst = sQb[t] + half * C::BM * 128;
                        const int n = (qt0 + t) * C::BM;
                        if (p.q_swap)
                            tma_load_4d(dst, &tm_qb, &ctl->qb_full, half * 64, h, n, b);
                        else
                            tma_load_4d(dst, &tm_qb, &ctl->qb_full, half * 64, n, h, b);
                    }
                // the block means, a chunk at a time, into the (still idle) P
                // buffers, each once the tensor core finished with the last
                for (int c = 0; pro_ok && c < e_chunks; ++c) {
                    if (c >= 1 && !(pro_ok = wait_one(&ctl->e_full[0], (c - 1) & 1, p.err, &ctl->abort, false, 1)))
                        break;
                    mbar_arrive_expect_tx(&ctl->mb_full[0], kEChunk * D * 2);
                    for (int half = 0; half < D / 64; ++half)
                        tma_load_3d(sP + half * kEChunk * 128, &tm_mean, &ctl->mb_full[0], half * 64, c * kEChunk, bh);
                    m_issued = c + 1;
                }
                // the ring's stages 1 and 2 and the P buffers are free once the
                // last products are done (the MMAs complete in order)
                if (pro_ok && e_chunks > 0) pro_ok = wait_one(&ctl->e_full[0], (e_chunks - 1) & 1, p.err, &ctl->abort, false, 1);
            }
            const int nsteps = !pro_ok ? 0 : nsteps_all;
            for (int j = issued; j < nsteps; ++j) {
                if (j >= C::STAGES &&
                    !wait_one(&ctl->kv_empty[j % C::STAGES], ((j / C::STAGES) - 1) & 1, p.err, &ctl->abort, false, 1))
                    break;
                issue_kv(j);
            }
            // every copy started here lands before the CTA may exit
            wait_one(FUSED_Q ? &ctl->qb_full : &ctl->q_full, 0, p.err, &ctl->abort, true, 2);
            if (KRES) {
                wait_one(&ctl->qb_full, 0, p.err, &ctl->abort, true, 2);
                // each means chunk after the first went out after the previous one's
                // products were done, so only the last one issued can be in flight
                if (m_issued > 0) wait_one(&ctl->mb_full[0], (m_issued - 1) & 1, p.err, &ctl->abort, true, 2);
            }
            for (int j = issued > C::STAGES ? issued - C::STAGES : 0; j < issued; ++j)
                wait_one(&ctl->kv_full[j % C::STAGES], (j / C::STAGES) & 1, p.err, &ctl->abort, true, 3);
        }
    } else if (warp == 9) {
        // ----------------------------------------------------------- MMA issue
        // The whole warp runs this loop (waits are warp-uniform); the elected
        // lane issues the MMAs and commits.
        const bool me = elect_one();
        const uint32_t idesc_qk = idesc_i8_s32(128, C::BN);
        const uint32_t idesc_pv = idesc_e4m3_f32_bmn(128, D);
        // Descriptors are built once; within a tile the start address field
        // (address / 16 in the low bits, no carry for shared addresses) is
        // advanced by plain additions.
        const uint64_t dq = smem_desc_kmajor(smem_u32(sQ), D);
        const uint64_t dk = smem_desc_kmajor(smem_u32(sK), D);
        const uint64_t dv = smem_desc_mnmajor(smem_u32(sV), D);
        const uint64_t dp = smem_desc_kmajor(smem_u32(sP), C::BN);
        auto issue_qk = [&](int t, int s) {
            const uint64_t a = dq + (uint64_t)((t * C::Q_BYTES) >> 4);
            const uint64_t b = dk + (uint64_t)((s * C::K_BYTES) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk)
                mma_i8_ss_if(me, tmem + t * 128, a + 2 * kk, b + 2 * kk, idesc_qk, kk > 0 ? 1u : 0u);
            tc_commit_if(me, &ctl->s_full[t]);
        };
        // n: the tile's own step (P buffer n % 2; O accumulates after its first)
        auto issue_pv = [&](int t, int s, int n, bool last) {
            const uint64_t a = dp + (uint64_t)((((2 * t + (n & 1)) * C::P_BYTES)) >> 4);
            const uint64_t b = dv + (uint64_t)((s * C::V_BYTES) >> 4);
#pragma unroll
            for (int kk = 0; kk < C::BN / 32; ++kk)
                mma_f8_ss_if(me, tmem + C::T_O + t * D, a + 2 * kk, b + 2 * kk * D, idesc_pv,
                             (n > 0 || kk > 0) ? 1u : 0u);
            tc_commit_if(me, &ctl->o_done[t]);
            if (last) tc_commit_if(me, &ctl->o_final[t]);
        };
        if constexpr (SPARSE) {
            // union step u streams key tile kt; tile t runs its own steps
            // PVs go in union order; each tile's next QK goes out as soon as its
            // K tile is in the ring (within STAGES-1 union steps), its S buffer
            // is free and PV(n-2) of that tile is issued (so S(n) finishing still
            // proves P buffer n%2 free).  With every tile kept this is the dense
            // issue order.
            const int tot[2] = {ctl->steps[0], ctl->steps[1]}, nu = ctl->steps[2];
            int nq[2] = {0, 0}, np[2] = {0, 0};  // QK and PV MMAs issued per tile
            int cq[2];                           // union step of each tile's next QK
            auto next_of = [&](int t, int from) {
                while (from < nu && !((uflag[from] >> t) & 1u)) ++from;
                return from;
            };
            cq[0] = next_of(0, 0);
            cq[1] = next_of(1, 0);
            bool ok = wait_warp(&ctl->q_full, 0, p.err, &ctl->abort, 4);
            for (int t = 0; ok && t < 2; ++t) {
                const int v = cq[t];
                if (v >= nu || v > C::STAGES - 1) continue;
                if (!(ok = wait_warp(&ctl->kv_full[v % C::STAGES], (v / C::STAGES) & 1, p.err, &ctl->abort, 5)))
                    break;
                tc_fence_after();
                issue_qk(t, v % C::STAGES);
                nq[t] = 1;
                cq[t] = next_of(t, v + 1);
            }
            for (int u = 0; ok && u < nu; ++u) {
                const int s = u % C::STAGES;
                for (int t = 0; ok && t < 2; ++t) {
                    const int v = cq[t], n = nq[t];
                    if (v >= nu || v > u + C::STAGES - 1 || np[t] < n - 1) continue;
                    if (!(ok = wait_warp(&ctl->kv_full[v % C::STAGES], (v / C::STAGES) & 1, p.err, &ctl->abort, 6)))
                        break;
                    // the tile's softmax holds its previous S in registers already
                    if (n > 0 && !(ok = wait_warp(&ctl->s_free[t], (n - 1) & 1, p.err, &ctl->abort, 7))) break;
                    tc_fence_after();
                    issue_qk(t, v % C::STAGES);
                    nq[t] = n + 1;
                    cq[t] = next_of(t, v + 1);
                }
                const uint32_t fl = uflag[u];  // tiles attending union step u
                for (int t = 0; ok && t < 2; ++t) {
                    if (!((fl >> t) & 1u)) continue;
                    const int n = np[t];
                    if (!(ok = wait_warp(&ctl->p_ready[t][n & 1], (n >> 1) & 1, p.err, &ctl->abort, 8))) break;
                    tc_fence_after();
                    issue_pv(t, s, n, n == tot[t] - 1);
                    np[t] = n + 1;
                }
                if (ok) tc_commit_if(me, &ctl->kv_empty[s]);
            }
        } else {
        bool ok = true;
        if constexpr (KRES) {
            // mean-term products: tile t's accumulator at columns [256 t, 256 t + N)
            const uint64_t dqb[2] = {smem_desc_kmajor(smem_u32(sQb[0]), 128),   // [half][128][64] bf16
                                     smem_desc_kmajor(smem_u32(sQb[1]), 128)};
            const uint64_t dmb = smem_desc_kmajor(smem_u32(sP), 128);        // [half][256][64] bf16
            ok = wait_warp(&ctl->qb_full, 0, p.err, &ctl->abort, 4);
            for (int c = 0; ok && c < e_chunks; ++c) {
                const int nb = min(kEChunk, p.nkb - c * kEChunk);
                const uint32_t idesc = idesc_bf16_f32(128, (nb + 15) & ~15);
                if (!(ok = wait_warp(&ctl->mb_full[0], c & 1, p.err, &ctl->abort, 5))) break;
                // tensor memory held chunk c - 1: the softmax took it out
                if (c >= 1 && !(ok = wait_warp(&ctl->e_free[0], (c - 1) & 1, p.err, &ctl->abort, 7))) break;
                tc_fence_after();
#pragma unroll
                for (int t = 0; t < 2; ++t)
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        // K step kk: channels 16 kk.. = 32 bytes into the rows of half kk / 4
                        const uint64_t a = dqb[t] + (uint64_t)((((kk / 4) * C::BM * 128) + (kk % 4) * 32) >> 4);
                        const uint64_t bm = dmb + (uint64_t)((((kk / 4) * kEChunk * 128) + (kk % 4) * 32) >> 4);
                        mma_f16_ss_if(me, tmem + t * 256, a, bm, idesc, kk > 0 ? 1u : 0u);
                    }
                tc_commit_if(me, &ctl->e_full[0]);
            }
            // tensor memory is the softmax warps' again before the first QK
            if (ok && e_chunks > 0) ok = wait_warp(&ctl->e_free[0], (e_chunks - 1) & 1, p.err, &ctl->abort, 7);
        }
        ok = ok && wait_warp(&ctl->q_full, 0, p.err, &ctl->abort, 4) &&
             wait_warp(&ctl->kv_full[0], 0, p.err, &ctl->abort, 5);
        if (ok) {
            tc_fence_after();
            issue_qk(0, 0);
            issue_qk(1, 0);
        }
        for (int j = 0; ok && j < nkv; ++j) {
            const int s = j % C::STAGES;
            if (j + 1 < nkv) {
                const int s1 = (j + 1) % C::STAGES;
                if (!(ok = wait_warp(&ctl->kv_full[s1], ((j + 1) / C::STAGES) & 1, p.err, &ctl->abort, 6))) break;
                for (int t = 0; ok && t < 2; ++t) {
                    if (!(ok = wait_warp(&ctl->s_free[t], j & 1, p.err, &ctl->abort, 7))) break;
                    tc_fence_after();
                    issue_qk(t, s1);  // the tile's softmax holds S(j) in registers already
                }
            } else {
                for (int t = 0; ok && t < 2; ++t) ok = wait_warp(&ctl->s_free[t], j & 1, p.err, &ctl->abort, 7);
            }
            for (int t = 0; ok && t < 2; ++t) {
                if (!(ok = wait_warp(&ctl->p_ready[t][j & 1], (j >> 1) & 1, p.err, &ctl->abort, 8))) break;
                tc_fence_after();
                if (!EXPORT_S) issue_pv(t, s, j, j == nkv - 1);
            }
            if (ok) tc_commit_if(me, &ctl->kv_empty[s]);
        }
        }
        // all MMAs issued here finish before tensor memory is released
        tc_commit_if(me, &ctl->drain);
        if (me) wait_one(&ctl->drain, 0, p.err, &ctl->abort, true, 9);
        __syncwarp();
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax
        regs_increase<C::SOFTMAX_REGS>();
        const int t = warp >> 2;         // Q tile of this warpgroup
        const int wq = warp & 3;         // tensor-memory lane quarter
        const int row = wq * 32 + lane;  // query row within the tile
        const int qt = qt0 + t;
        const int grow = qt * C::BM + row;
        const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tmem + lane_off + t * 128;
        const uint32_t tO = tmem + lane_off + C::T_O + t * D;
        const uint32_t pbase = smem_u32(sP) + 2 * t * C::P_BYTES;
        bool ok = true;
        float sq;
        if constexpr (FUSED_Q) {
            // This tile's bf16 rows are in the P buffers; the tile's block scale is
            // its |max| / 127 and the codes rne(x * fp32(127 / |max|)).  Each warp
            // takes its own 32 rows four at a time: lane l holds the 8 channels
            // 8 (l mod 8).. of row 4i + l/8 in each 64-channel half, so a warp's
            // 16-byte loads cover four whole 128-byte rows (no bank conflicts).
            const uint16_t *qtile = reinterpret_cast<const uint16_t *>(sP) + t * (D / 64) * C::BM * 64;
            float amax = 0.f;
            if ((ok = wait_warp(&ctl->qb_full, 0, p.err, &ctl->abort, 14))) {
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int half = 0; half < D / 64; ++half) {
                        const int r = wq * 32 + i * 4 + (lane >> 3);
                        float f[8];
                        unpack8(*reinterpret_cast<const uint4 *>(qtile + (half * C::BM + r) * 64 + (lane & 7) * 8), f);
#pragma unroll
                        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
                    }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                if (lane == 0) ctl->q_amax[t][wq] = amax;
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->q_amax_bar[t]);
                ok = wait_warp(&ctl->q_amax_bar[t], 0, p.err, &ctl->abort, 14);
            }
            if (ok) {
                amax = fmaxf(fmaxf(ctl->q_amax[t][0], ctl->q_amax[t][1]), fmaxf(ctl->q_amax[t][2], ctl->q_amax[t][3]));
                const float inv = amax > 0.f ? __fdiv_rn(127.f, amax) : 0.f;
                // codes at their swizzled places in the K-major tile (128-byte
                // swizzle for d = 128, 64-byte for d = 64, as the TMA writes them):
                // 16-byte chunk c of row r sits at r*d + ((c ^ swz(r)) * 16)
                const uint32_t qdst = smem_u32(sQ + t * C::Q_BYTES);
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int half = 0; half < D / 64; ++half) {
                        const int r = wq * 32 + i * 4 + (lane >> 3);
                        const int ch = half * 64 + (lane & 7) * 8;  // first of this lane's 8 channels
                        float f[8];
                        unpack8(*reinterpret_cast<const uint4 *>(qtile + (half * C::BM + r) * 64 + (lane & 7) * 8), f);
                        const uint2 w = i8x8(f, inv);
                        const int swz = D == 128 ? (r & 7) : ((r >> 1) & 3);
                        st_shared_v2(qdst + r * D + (((ch >> 4) ^ swz) << 4) + ((ch >> 3) & 1) * 8, w.x, w.y);
                    }
                fence_proxy_async_smem();  // make the codes visible to the tensor core
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->q_full);
            }
            sq = amax > 0.f ? __fdiv_rn(amax, 127.f) : 0.f;
        } else {
            sq = qt < p.nqb ? p.q_scale[(int64_t)bh * p.nqb + qt] : 0.f;
        }
        float *eslot = nullptr;  // KRES: this CTA's scratch slot, [nkb][256 rows]
        if constexpr (KRES) {
            uint32_t smid;
            asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
            if (static_cast<int>(smid) >= p.n_slots) {
                // no slot for this SM: give up (reported like a timed-out wait, site 0)
                if (lane == 0) record_timeout(p.err, &ctl->abort, 0);
                ok = false;
            } else {
                eslot = p.eslot + (int64_t)smid * p.nkb * 256 + t * 128 + row;
            }
            for (int c = 0; ok && c < e_chunks; ++c) {
                if (!(ok = wait_warp(&ctl->e_full[0], c & 1, p.err, &ctl->abort, 14))) break;
                tc_fence_after();
                const int nb = min(kEChunk, p.nkb - c * kEChunk);
                for (int cc = 0; cc < nb; cc += 32) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tmem + lane_off + t * 256 + cc, v);
                    tmem_wait_ld_x32(v);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (cc + i < nb) eslot[(int64_t)(c * kEChunk + cc + i) * 256] = __uint_as_float(v[i]) * p.s_l2;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->e_free[0]);
            }
        }
        const float cq = sq * p.s_l2;
        const float kLog2_448 = 8.807354922057604f;
        const float *ksc = p.k_scale + (int64_t)bh * p.nkb + 2 * kv0;
        const uint16_t *mylist = slist + t * (SPARSE ? p.nqb : 0);
        const int steps = SPARSE ? ctl->steps[t] : nkv;  // this tile's own steps
        int kt_next = (SPARSE && steps > 0) ? mylist[0] : 0;  // key tile of the next step
        float m = -INFINITY, l = 0.f;
        float ks_next0 = (EXPORT_S || steps == 0) ? 0.f : __ldg(ksc + 2 * kt_next);
        float ks_next1 = (EXPORT_S || steps == 0) ? 0.f : __ldg(ksc + 2 * kt_next + 1);
        // KRES: this row's mean terms from the slot (written by this thread above)
        float e_next0 = (KRES && ok) ? eslot[(2 * kt_next) * 256] : 0.f;
        float e_next1 = (KRES && ok) ? eslot[(2 * kt_next + 1) * 256] : 0.f;
        for (int j = 0; ok && j < steps; ++j) {
            // this step's key tile and its two K-block scales were fetched one step ahead
            const int kt = kt_next;
            const float ks0 = ks_next0, ks1 = ks_next1;
            const float e0 = e_next0, e1 = e_next1;
            if (!EXPORT_S && j + 1 < steps) {
                kt_next = SPARSE ? mylist[j + 1] : j + 1;
                ks_next0 = __ldg(ksc + 2 * kt_next);
                ks_next1 = __ldg(ksc + 2 * kt_next + 1);
                if (KRES) {
                    e_next0 = eslot[(2 * kt_next) * 256];
                    e_next1 = eslot[(2 * kt_next + 1) * 256];
                }
            }
            if (!(ok = wait_warp(&ctl->s_full[t], j & 1, p.err, &ctl->abort, 10 + t))) break;
            tc_fence_after();
            uint32_t ra[32], rb[32], rc[32], rd[32];
            tmem_ld_32x32b_x32(tS + 0, ra);
            tmem_ld_32x32b_x32(tS + 32, rb);
            tmem_ld_32x32b_x32(tS + 64, rc);
            tmem_ld_32x32b_x32(tS + 96, rd);
            tmem_wait_ld_x32(ra);
            tmem_wait_ld_x32(rb);
            tmem_wait_ld_x32(rc);
            tmem_wait_ld_x32(rd);
            // S(j) is in registers: the tensor core may overwrite it with S(j+1)
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->s_free[t]);
            if (EXPORT_S) {
                if (t == 0) {
                    int32_t *dst = p.s_export + row * C::BN;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        dst[i] = static_cast<int32_t>(ra[i]);
                        dst[32 + i] = static_cast<int32_t>(rb[i]);
                        dst[64 + i] = static_cast<int32_t>(rc[i]);
                        dst[96 + i] = static_cast<int32_t>(rd[i]);
                    }
                }
            } else {
                const int n_valid = min(C::BN, p.N - (kv0 + kt) * C::BN);
                const float c0 = cq * ks0, c1 = cq * ks1;
                float x0, x1;
                if (n_valid == C::BN) {
                    x0 = static_cast<float>(row_max64<false>(ra, rb, 0, n_valid)) * c0;
                    x1 = static_cast<float>(row_max64<false>(rc, rd, 64, n_valid)) * c1;
                } else {
                    // ragged last step: keys at or past N take no part
                    const int mx0 = row_max64<true>(ra, rb, 0, n_valid);
                    const int mx1 = row_max64<true>(rc, rd, 64, n_valid);
                    x0 = mx0 == INT_MIN ? -INFINITY : static_cast<float>(mx0) * c0;
                    x1 = mx1 == INT_MIN ? -INFINITY : static_cast<float>(mx1) * c1;
                }
                if (KRES) x0 += e0, x1 += e1;
                const float m_new = fmaxf(m, ceilf(fmaxf(x0, x1)));
                const float alpha = (m == -INFINITY) ? 0.f : exp2_int(m - m_new);
                const float nb = kLog2_448 - m_new;
                const float nb0 = KRES ? nb + e0 : nb, nb1 = KRES ? nb + e1 : nb;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                uint32_t w[32];
                if (n_valid == C::BN) {
                    p_pack32<false>(ra, c0, nb0, 0, n_valid, acc, w + 0);
                    p_pack32<false>(rb, c0, nb0, 32, n_valid, acc, w + 8);
                    p_pack32<false>(rc, c1, nb1, 64, n_valid, acc, w + 16);
                    p_pack32<false>(rd, c1, nb1, 96, n_valid, acc, w + 24);
                } else {
                    p_pack32<true>(ra, c0, nb0, 0, n_valid, acc, w + 0);
                    p_pack32<true>(rb, c0, nb0, 32, n_valid, acc, w + 8);
                    p_pack32<true>(rc, c1, nb1, 64, n_valid, acc, w + 16);
                    p_pack32<true>(rd, c1, nb1, 96, n_valid, acc, w + 24);
                }
                l = l * alpha + ((acc[0] + acc[1]) + (acc[2] + acc[3]));
                // P buffer j%2 was last read by PV(j-2), which finished before S(j)
                // did (the MMAs run in order), so it can be overwritten now
                store_p_row(pbase + (j & 1) * C::P_BYTES, row, w);
                fence_proxy_async_smem();  // make the stores visible to the tensor core
                const bool need = (j > 0) && (m_new > m);
                m = m_new;
                if (__any_sync(0xffffffffu, need)) {
                    // O must hold step j-1's product before it is rescaled; S(j)
                    // arriving proves PV(j-2) finished, so this barrier is at most
                    // one phase behind
                    if (!(ok = wait_warp(&ctl->o_done[t], (j - 1) & 1, p.err, &ctl->abort, 12))) break;
                    tc_fence_after();
                    const float a = need ? alpha : 1.f;
                    // the S registers are free again: load all of O's row at once
                    tmem_ld_32x32b_x32(tO + 0, ra);
                    tmem_ld_32x32b_x32(tO + 32, rb);
                    if (D == 128) {
                        tmem_ld_32x32b_x32(tO + 64, rc);
                        tmem_ld_32x32b_x32(tO + 96, rd);
                    }
                    tmem_wait_ld_x32(ra);
                    tmem_wait_ld_x32(rb);
                    if (D == 128) {
                        tmem_wait_ld_x32(rc);
                        tmem_wait_ld_x32(rd);
                    }
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        float x0, x1;
                        fmul2(x0, x1, __uint_as_float(ra[i]), __uint_as_float(ra[i + 1]), a, a);
                        ra[i] = __float_as_uint(x0), ra[i + 1] = __float_as_uint(x1);
                        fmul2(x0, x1, __uint_as_float(rb[i]), __uint_as_float(rb[i + 1]), a, a);
                        rb[i] = __float_as_uint(x0), rb[i + 1] = __float_as_uint(x1);
                        if (D == 128) {
                            fmul2(x0, x1, __uint_as_float(rc[i]), __uint_as_float(rc[i + 1]), a, a);
                            rc[i] = __float_as_uint(x0), rc[i + 1] = __float_as_uint(x1);
                            fmul2(x0, x1, __uint_as_float(rd[i]), __uint_as_float(rd[i + 1]), a, a);
                            rd[i] = __float_as_uint(x0), rd[i + 1] = __float_as_uint(x1);
                        }
                    }
                    tmem_st_32x32b_x32(tO + 0, ra);
                    tmem_st_32x32b_x32(tO + 32, rb);
                    if (D == 128) {
                        tmem_st_32x32b_x32(tO + 64, rc);
                        tmem_st_32x32b_x32(tO + 96, rd);
                    }
                    tmem_wait_st();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->p_ready[t][j & 1]);
        }
        if (SPARSE && steps == 0) {
            // the tile keeps no key tile: its rows have no softmax and are 0
            if (grow < p.N) {
                uint4 *dst = reinterpret_cast<uint4 *>(p.out + (int64_t)(bh / p.H) * p.osb +
                                                       (int64_t)(bh % p.H) * p.osh + (int64_t)grow * p.osn);
#pragma unroll
                for (int i = 0; i < D / 8; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
            }
        } else if (ok && !EXPORT_S && wait_warp(&ctl->o_final[t], 0, p.err, &ctl->abort, 13)) {
            tc_fence_after();
            const float inv_l = 1.f / l;
            // The warp's 32 bf16 rows go through its share of the tile's P buffers
            // (free: every P.V has completed) so that the global stores cover
            // whole rows: 16-byte chunk c of row r is staged at r*2d +
            // ((c ^ (r mod CPR)) * 16), then each store instruction writes
            // 32 * 16 bytes = 512 / (2d) rows.
            constexpr int CPR = D / 8;  // 16-byte chunks per row
            const uint32_t stage = pbase + (row - lane) * D * 2;  // the warp's 32 rows of its tile's P buffers
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                tmem_ld_32x32b_x32(tO + cc * 32, o);
                tmem_wait_ld_x32(o);
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int cidx = cc * 32 + 2 * i;
                    w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * ctl->v_scale[cidx] * inv_l,
                                       __uint_as_float(o[2 * i + 1]) * ctl->v_scale[cidx + 1] * inv_l);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int c = cc * 4 + i;
                    st_shared_v4(stage + lane * D * 2 + ((c ^ (lane & (CPR - 1))) << 4), w[4 * i], w[4 * i + 1],
                                 w[4 * i + 2], w[4 * i + 3]);
                }
            }
            __syncwarp();
            constexpr int RPI = 32 / CPR;  // rows per store instruction
            const int c = lane % CPR;
            uint16_t *obase = p.out + (int64_t)(bh / p.H) * p.osb + (int64_t)(bh % p.H) * p.osh;
#pragma unroll 1
            for (int r0 = 0; r0 < 32; r0 += RPI) {
                const int r = r0 + lane / CPR;
                const uint4 val = ld_shared_v4(stage + r * D * 2 + ((c ^ (r & (CPR - 1))) << 4));
                const int gr = grow - lane + r;  // this warp's first row is grow - lane
                if (gr < p.N) *reinterpret_cast<uint4 *>(obase + (int64_t)gr * p.osn + c * 8) = val;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 3-D uint8 tensor map: dims (inner..outer), byte strides of dims 1 and 2,
// box (b0, b1, 1), zero fill outside the tensor.
cudaError_t make_map(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t st1,
                     uint64_t st2, uint32_t b0, uint32_t b1) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorSymbolNotFound;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {st1, st2};
    const cuuint32_t box[3] = {b0, b1, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapSwizzle sw = b0 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}


template <int D, bool EXPORT_S, bool SPARSE, bool KRES = false, bool FUSED_Q = false>
cudaError_t launch_attn_d(const Shape &s, const int8_t *q_i8, const int8_t *k_i8, const uint8_t *v_e4m3,
                          const AttnParams &p0, dim3 grid, cudaStream_t st, const Src *q_bf16 = nullptr,
                          const uint16_t *k_bmean = nullptr) {
    using C = Cfg<D>;
    const int n_pad = s.n_pad();
    CUtensorMap tq, tk, tv, tqb, tmean;
    AttnParams p = p0;
    cudaError_t e;
    if (FUSED_Q) {
        if (!q_bf16) return cudaErrorInvalidValue;
        if ((e = make_bf16_token_map(&tqb, *q_bf16, s, 64, &p.q_swap)) != cudaSuccess) return e;
        q_i8 = k_i8;  // the INT8 Q map is not read; any valid map will do
    }
    if (KRES) {
        // bf16 Q rows (128 per box, 128-byte swizzle) and the bf16 block means
        // [BH][nkb][d] (256 blocks per box, 128-byte swizzle) for the prologue
        if (!q_bf16 || !k_bmean) return cudaErrorInvalidValue;
        if ((e = make_bf16_token_map(&tqb, *q_bf16, s, C::BM, &p.q_swap, true)) != cudaSuccess) return e;
        if ((e = make_bf16_map3(&tmean, k_bmean, D, s.n_kblocks(), s.BH(), 256)) != cudaSuccess) return e;
    }
    if ((e = make_map(&tq, q_i8, D, n_pad, s.BH(), D, (uint64_t)n_pad * D, D, C::BM)) != cudaSuccess) return e;
    if ((e = make_map(&tk, k_i8, D, n_pad, s.BH(), D, (uint64_t)n_pad * D, D, C::BN)) != cudaSuccess) return e;
    if (EXPORT_S) {
        tv = tk;  // not read
    } else if ((e = make_map(&tv, v_e4m3, D, n_pad, s.BH(), D, (uint64_t)n_pad * D, D, C::BN)) != cudaSuccess) {
        return e;
    }
    if (!FUSED_Q && !KRES) tqb = tq;  // not read
    if (!KRES) tmean = tq;              // not read
    p.err = device_error_ptr();
    if (!p.err) return cudaErrorSymbolNotFound;
    const int smem = smem_bytes<D>(SPARSE ? 7 * p.nqb + 8 : 0);  // three uint16 lists and one uint8 list
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    auto kern = k_attn<D, EXPORT_S, SPARSE, KRES, FUSED_Q>;
    // The setmaxnreg split assumes the kernel is launched with LAUNCH_REGS per
    // thread; with fewer the increases could never be satisfied.
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return e;
    if (fa.numRegs != C::LAUNCH_REGS) return cudaErrorInvalidConfiguration;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess) return e;
    return launch_dependent(kern, grid, dim3(C::THREADS), smem, st, tq, tk, tv, tqb, tmean, p);
}

}  // namespace

unsigned *device_error_ptr() {
    static unsigned *ptrs[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!ptrs[dev]) {
        void *a = nullptr;
        if (cudaGetSymbolAddress(&a, g_device_error) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<unsigned *>(a);
    }
    return ptrs[dev];
}

cudaError_t make_bf16_token_map(CUtensorMap *m, const Src &src, const Shape &s, uint32_t rows, int *hn_swapped,
                                bool swizzle128) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorSymbolNotFound;
    // Dimensions after the channels: N and H in order of stride, then B.  A
    // dimension of extent 1 is never stepped, so it gets the packed stride.
    uint64_t st_n = (uint64_t)src.sn * 2, st_h = (uint64_t)src.sh * 2, st_b = (uint64_t)src.sb * 2;
    bool swap;
    if (s.H == 1) {
        swap = false;
        st_h = st_n * (uint64_t)s.N;
    } else if (s.N == 1) {
        swap = true;
        st_n = st_h * (uint64_t)s.H;
    } else {
        swap = st_h < st_n;
    }
    const uint64_t e1 = swap ? s.H : s.N, e2 = swap ? s.N : s.H;
    const uint64_t s1 = swap ? st_h : st_n, s2 = swap ? st_n : st_h;
    if (s.B == 1) st_b = s2 * e2;
    const cuuint64_t dims[4] = {(cuuint64_t)s.d, e1, e2, (cuuint64_t)s.B};
    const cuuint64_t strides[3] = {s1, s2, st_b};
    const cuuint32_t box[4] = {64, swap ? 1u : rows, swap ? rows : 1u, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint16_t *>(src.p), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    *hn_swapped = swap ? 1 : 0;
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 3-D map of a contiguous bf16 [d2][d1][d0] array (d0 = 64 or 128 channels):
// box 64 channels x `rows` x 1, 128-byte swizzle, zeros outside the array.
cudaError_t make_bf16_map3(CUtensorMap *m, const uint16_t *base, uint64_t d0, uint64_t d1, uint64_t d2,
                           uint32_t rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorSymbolNotFound;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    const cuuint32_t box[3] = {64, rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Parameters every attention launch shares: codes' scales, output view, shape
// and fp32(sm_scale * fp32(log2 e)).
AttnParams attn_params(const Shape &s, const Codes &c, const Dst &out, float sm_scale) {
    AttnParams p{};
    p.q_scale = c.q_scale;
    p.k_scale = c.k_scale;
    p.v_scale = c.v_scale;
    p.out = out.p;
    p.osb = out.sb;
    p.osh = out.sh;
    p.osn = out.sn;
    p.H = s.H;
    p.N = s.N;
    p.nqb = s.n_qblocks();
    p.nkb = s.n_kblocks();
    p.s_l2 = sm_scale * static_cast<float>(1.4426950408889634);
    return p;
}

cudaError_t launch_attention(const Shape &s, const Codes &c, const Dst &out, float sm_scale, cudaStream_t st) {
    AttnParams p = attn_params(s, c, out, sm_scale);
    dim3 grid((s.n_qblocks() + 1) / 2, s.BH());
    return s.d == 128 ? launch_attn_d<128, false, false>(s, c.q_i8, c.k_i8, c.v_e4m3, p, grid, st)
                      : launch_attn_d<64, false, false>(s, c.q_i8, c.k_i8, c.v_e4m3, p, grid, st);
}

cudaError_t launch_attention_fused_q(const Shape &s, const Codes &c, const Src &q_bf16, const Dst &out,
                                     float sm_scale, cudaStream_t st) {
    AttnParams p = attn_params(s, c, out, sm_scale);
    p.q_scale = nullptr;  // the kernel computes each tile's Q scale
    dim3 grid((s.n_qblocks() + 1) / 2, s.BH());
    return s.d == 128
               ? launch_attn_d<128, false, false, false, true>(s, nullptr, c.k_i8, c.v_e4m3, p, grid, st, &q_bf16)
               : launch_attn_d<64, false, false, false, true>(s, nullptr, c.k_i8, c.v_e4m3, p, grid, st, &q_bf16);
}

int kres_slots() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess)
        return 0;
    return sms;
}

cudaError_t launch_attention_kres(const Shape &s, const Codes &c, const Src &q_bf16, const uint16_t *k_bmean,
                                  const Dst &out, float sm_scale, float *eslot, int n_slots, cudaStream_t st) {
    AttnParams p = attn_params(s, c, out, sm_scale);
    p.eslot = eslot;
    p.n_slots = n_slots;
    dim3 grid((s.n_qblocks() + 1) / 2, s.BH());
    return s.d == 128
               ? launch_attn_d<128, false, false, true>(s, c.q_i8, c.k_i8, c.v_e4m3, p, grid, st, &q_bf16, k_bmean)
               : launch_attn_d<64, false, false, true>(s, c.q_i8, c.k_i8, c.v_e4m3, p, grid, st, &q_bf16, k_bmean);
}

cudaError_t launch_attention_sparse(const Shape &s, const Codes &c, const Dst &out, float sm_scale,
                                    const uint32_t *kv_mask, cudaStream_t st) {
    AttnParams p = attn_params(s, c, out, sm_scale);
    p.kv_mask = kv_mask;
    p.mask_words = s.mask_words();
    dim3 grid((s.n_qblocks() + 1) / 2, s.BH());
    return s.d == 128 ? launch_attn_d<128, false, true>(s, c.q_i8, c.k_i8, c.v_e4m3, p, grid, st)
                      : launch_attn_d<64, false, true>(s, c.q_i8, c.k_i8, c.v_e4m3, p, grid, st);
}

cudaError_t launch_debug_qk_tile(const Shape &s, const int8_t *q_i8, const int8_t *k_i8, int bh, int q_tile,
                                 int kv_tile, int32_t *s_out, cudaStream_t st) {
    AttnParams p{};
    p.H = s.H;
    p.N = s.N;
    p.nqb = s.n_qblocks();
    p.nkb = s.n_kblocks();
    p.s_export = s_out;
    p.bh0 = bh;
    p.q_tile0 = q_tile;
    p.kv_tile0 = kv_tile;
    return s.d == 128 ? launch_attn_d<128, true, false>(s, q_i8, k_i8, nullptr, p, dim3(1, 1), st)
                      : launch_attn_d<64, true, false>(s, q_i8, k_i8, nullptr, p, dim3(1, 1), st);
}

cudaError_t read_and_clear_device_error(unsigned *value, cudaStream_t st) {
    unsigned *ptr = device_error_ptr();
    if (!ptr) return cudaErrorSymbolNotFound;
    cudaError_t e = cudaMemcpyAsync(value, ptr, sizeof(unsigned), cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return e;
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return e;
    return cudaMemsetAsync(ptr, 0, sizeof(unsigned), st);
}

}  // namespace sage
