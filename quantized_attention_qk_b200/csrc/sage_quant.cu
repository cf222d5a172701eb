// sage_quant.cu -- the quantize pass of the quantized attention forward.
//
// Pages: "MiniMax H3 接入 SageAttention 实测加速", section 一 (outlier smoothing of
// QK^T, INT8 QK, FP8 PV).  Block sizes, rounding and scale conventions are the
// readings C1-C3 and C7 of the design notes:
//   scale = amax/127 (fp32 IEEE divide), code = rne(x * fp32(127/amax)) in
//   [-127,127]; V: code = e4m3_rn_satfinite(v * fp32(448/amax_c)).
//
// One HBM-bound streaming kernel, k_qpass (no tensor cores: there is no
// contraction), launched cooperatively so that all its CTAs are resident at
// once, in two phases:
//   A  statistics: CTA i takes the i-th of G equal parts of all (b,h, 64-token
//      sub-block)s; within each head its part covers, the warps stream the
//      K and V rows (direct 16-byte loads held in registers, kept in L2 for
//      phase B) and accumulate per channel the fp64 sum of K and the max |V|;
//      the warps' results are added in warp order into one partial per
//      (CTA, head), published with a release store of a flag.
//   B  codes: CTA i takes the i-th of G equal parts of the (b,h, 128-token
//      block)s -- the same part of the token range, last block first, so the
//      K and V rows read most recently in phase A are the first ones reused.
//      For each head it waits (acquire loads, bounded) for the flags of the
//      CTAs that covered the head in phase A, adds their partials in CTA
//      order (fp64) and finishes the statistics (the K mean and the 448/amax
//      factors of V).  Then each 128-token block is coded from registers by
//      a group of warps (16 rows each for d = 128, 32 for d = 64): Q block
//      -> INT8 (the group exchanges its warps' maxima through shared memory),
//      (K - mean) per 64-token block -> INT8, V -> e4m3 (token-major, like
//      the codes of Q and K; the attention kernel reads it as an MN-major
//      operand).
// Warps work on their own rows and exchange block maxima only within their
// group; the only CTA-wide barriers are at head boundaries.  The fp64 K sums
// are exact for bf16 inputs whenever a column's values span fewer than 53
// bits, so the mean does not depend on how the rows were split among CTAs and
// warps.
//
// K-residual mode ("ComfyUI-sol-attn", 核心亮点 item 1: quantize only the
// residual of K inside each block and keep the block-mean term at bf16
// precision).  Readings where the page is silent: the blocks are the 64-token
// K blocks; the block mean is the mean of the block's valid tokens (summed
// exactly in fp64), rounded to bf16 (RNE); the residual fp32(k) - fp32(mean)
// is coded like the other INT8 codes.  Phase A then sums no K; phase B writes
// the residual codes, the per-block scales and the bf16 block means (blocks
// past N: mean 0, codes 0).  The attention kernel adds the mean term.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <chrono>

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {
namespace {

constexpr int kPassWarps = 8;  // two CTAs per SM (128 registers a thread)
constexpr int kPassThreads = 32 * kPassWarps;

// Geometry of one warp's rows for head dim D: a warp load instruction covers
// RPI rows of VPR 16-byte vectors; a lane holds NB vectors of each of Q, K and
// V in phase B (RB rows per warp) and NA of K and of V in phase A (RA rows); a
// 128-token block takes a group of WU warps, a 64-token K block KW of them.
template <int D>
struct Geom {
    static constexpr int VPR = D / 8;
    static constexpr int RPI = 32 / VPR;
    static constexpr int NB = 8;
    static constexpr int RB = NB * RPI;
    static constexpr int WU = kQBlock / RB;
    static constexpr int KW = kKBlock / RB;
    static constexpr int GROUPS = kPassWarps / WU;
    static constexpr int NA = 8;
    static constexpr int RA = NA * RPI;
};
static_assert(Geom<128>::WU * Geom<128>::RB == kQBlock && Geom<64>::WU * Geom<64>::RB == kQBlock &&
                  Geom<128>::KW >= 1 && Geom<64>::KW >= 1 && kPassWarps % Geom<128>::WU == 0,
              "a warp group codes a 128-token block; a K block spans whole warps");
static_assert(kKBlock % Geom<128>::RA == 0 && kKBlock % Geom<64>::RA == 0, "phase-A batches tile a sub-block");
static_assert(Geom<64>::GROUPS < 16, "named barriers 1..GROUPS");

// 16 bytes of a read-only input, not kept in L1, with an L2 eviction policy.
// The memory clobber keeps a block's loads after the previous block's stores,
// so that no more than one block's rows are live in registers.
__device__ __forceinline__ uint4 ld_in(const uint16_t *p, uint64_t policy) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p), "l"(policy)
                 : "memory");
    return r;
}

// Per-half max of |x| over bf16 pairs: max of the accumulated magnitudes and
// the magnitudes of x (a NaN half is ignored, like fmaxf does).
__device__ __forceinline__ uint32_t bmax_abs(uint32_t m, uint32_t x) {
    uint32_t d;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(m), "r"(x & 0x7fff7fffu));
    return d;
}
__device__ __forceinline__ float bf_bits(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ void st_release_u64(unsigned long long *p, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
// Barrier of the `threads` threads of warp group `id` (ids from 1; 0 is
// __syncthreads').
__device__ __forceinline__ void group_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Two e4m3 codes (round to nearest even, saturating to +-448): lo in the low
// byte (cvt packs its first source in the high byte).
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tcvt.u32.u16 %0, t;\n\t}"
        : "=r"(r)
        : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float warp_fmax(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// x[i] = the 16 bytes at row row0 + i * RPI (stride sn elements from p), or
// zeros for rows >= limit.  Rows are stepped through with one pointer, and the
// common case of all rows valid takes no per-row test.
template <int NV, int RPI>
__device__ __forceinline__ void load_rows(uint4 (&x)[NV], const uint16_t *p, int64_t sn, int row0, int limit,
                                          uint64_t policy) {
    const uint16_t *r = p + (int64_t)row0 * sn;
    const int64_t step = (int64_t)RPI * sn;
    if (row0 + (NV - 1) * RPI < limit) {
#pragma unroll
        for (int i = 0; i < NV; ++i, r += step) x[i] = ld_in(r, policy);
    } else {
#pragma unroll
        for (int i = 0; i < NV; ++i, r += step)
            x[i] = row0 + i * RPI < limit ? ld_in(r, policy) : make_uint4(0u, 0u, 0u, 0u);
    }
}

// Tile pooling: add 8 int8 codes (channels 0..7 of this lane's vector) into
// four int16 pairs (channels 2j, 2j+1 in pair j), sign-extending each byte.
__device__ __forceinline__ uint32_t sext_pair(uint32_t w, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(w), "r"(sel));  // selector bit 3: replicate the byte's sign
    return r;
}
__device__ __forceinline__ void add_codes(uint32_t (&ps)[4], uint2 cw) {
    ps[0] = __vadd2(ps[0], sext_pair(cw.x, 0x9180u));
    ps[1] = __vadd2(ps[1], sext_pair(cw.x, 0xB3A2u));
    ps[2] = __vadd2(ps[2], sext_pair(cw.y, 0x9180u));
    ps[3] = __vadd2(ps[3], sext_pair(cw.y, 0xB3A2u));
}
// The warp's sums: lanes VPR apart hold the same channels; lanes < VPR store
// theirs into the warp's slot (D/2 int16 pairs).
template <int VPR>
__device__ __forceinline__ void pool_partial(uint32_t (&ps)[4], uint32_t *slot, int lane, int vec) {
#pragma unroll
    for (int o = VPR; o < 32; o <<= 1)
#pragma unroll
        for (int j = 0; j < 4; ++j) ps[j] = __vadd2(ps[j], __shfl_xor_sync(0xffffffffu, ps[j], o));
    if (lane < VPR) {
#pragma unroll
        for (int j = 0; j < 4; ++j) slot[vec * 4 + j] = ps[j];
    }
}

// A flag of phase A holds (stamp << 16) | readers: the call's 48-bit stamp
// and the number of phase-B CTAs that read the head (known from the split).
// Each reader takes one off after its wait and the last one clears the flag,
// so every flag is zero again when the kernel ends: a replay of the same
// launch (a captured graph: same stamp) never finds its own stamp left over,
// and a fresh workspace holds a given 48-bit stamp only by chance.
struct PassArgs {
    Src q, k, v;
    int H, BH, N, n_pad;
    double *ksum_part;          // [slots][D]: slot = CTA + head
    float *vmax_part;           // [slots][D]
    unsigned long long *flags;  // [slots]
    unsigned long long stamp;   // 48 bits, bit 47 set
    float *user_k_mean;         // optional copy of the K mean [BH][D]
    uint16_t *k_bmean;          // K-residual mode: bf16 block means [BH][N_pad/64][D]
    float *pool_qv, *pool_kvT;  // tile pooling: [BH][tiles][D] and [BH][D][tiles]
    Codes c;
    unsigned *err;
};

// RES: K is coded as the residual of its 64-token block mean (K-residual
// mode) instead of smoothing by the head's mean, so phase A sums no K.
// POOL: also the pooled tile vectors of the block selection (the code sums
// of each 128-token tile, times the scales), from the codes in registers.
template <int D, bool DO_Q, bool DO_K, bool DO_V, bool RES, bool POOL = false>
__global__ void __launch_bounds__(kPassThreads, 512 / kPassThreads) k_qpass(const PassArgs a) {
    using Gm = Geom<D>;
    constexpr int VPR = Gm::VPR, RPI = Gm::RPI, NB = Gm::NB, RB = Gm::RB, WU = Gm::WU, KW = Gm::KW, NA = Gm::NA,
                  RA = Gm::RA;
    constexpr int NW = kPassWarps;
    constexpr bool KSUM = DO_K && !RES;  // the head's K column sums (smoothing)
    constexpr bool STATS = KSUM || DO_V;
    __shared__ double red_s[NW][D];
    __shared__ float red_m[NW][D];
    __shared__ float mu[D], vinv[D];
    __shared__ float grp_max[Gm::GROUPS][2][2][WU];  // [group][unit parity][Q, K][warp]
    // K-residual mode: the warps' K block sums [group][warp][channel].  One
    // buffer is enough: between a block's reads and the next block's writes
    // every warp of the group passes the K-maximum barrier of the block.
    __shared__ double grp_sum[RES ? Gm::GROUPS : 1][RES ? WU : 1][RES ? D : 1];
    // tile pooling: the warps' code sums as int16 pairs [group][Q, K][warp][channel pair],
    // and the amax of the unit's two K blocks
    __shared__ uint32_t grp_pool[POOL ? Gm::GROUPS : 1][2][POOL ? WU : 1][POOL ? D / 2 : 1];
    __shared__ float grp_ka[POOL ? Gm::GROUPS : 1][2];
    __shared__ AbortState abort_st;
    __shared__ int bad;
    const int nqb = a.n_pad / kQBlock, nkb = a.n_pad / kKBlock, nsb = (a.N + kKBlock - 1) / kKBlock;
    const int G = gridDim.x;  // <= the 128-token blocks, so every CTA codes at least one
    const long long nA = (long long)a.BH * nsb, nB = (long long)a.BH * nqb;
    // the CTA whose part holds unit x, of n units split in G equal parts
    auto owner = [&](long long x, long long n) { return (int)(((x + 1) * G - 1) / n); };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int vec = lane % VPR, rl = lane / VPR;  // this lane's 8 channels and row within a load
    if (threadIdx.x == 0) {
        abort_st.flag = 0;
        bad = 0;
    }
    __syncthreads();
    grid_dep_launch();  // the attention kernel may take each SM this CTA leaves

    // ------------------------------------------------------------ phase A
    if constexpr (STATS) {
        const uint64_t keep = l2_policy_evict_last();  // phase B reads K and V again
        const long long a0 = nA * blockIdx.x / G, a1 = nA * (blockIdx.x + 1) / G;
        for (int h = (int)(a0 / nsb); h <= (int)((a1 - 1) / nsb); ++h) {
            const long long s0 = a0 > (long long)h * nsb ? a0 : (long long)h * nsb;
            const long long s1 = a1 < (long long)(h + 1) * nsb ? a1 : (long long)(h + 1) * nsb;
            const int r_begin = (int)(s0 - (long long)h * nsb) * kKBlock;
            const int r_end = min(a.N, (int)(s1 - (long long)h * nsb) * kKBlock);
            const int nbat = (r_end - r_begin + RA - 1) / RA;
            const int b = h / a.H, hh = h % a.H;
            const uint16_t *kp = a.k.p + b * a.k.sb + hh * a.k.sh + vec * 8;
            const uint16_t *vp = a.v.p + b * a.v.sb + hh * a.v.sh + vec * 8;
            double s8[8];
            uint32_t m4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int e = 0; e < 8; ++e) s8[e] = 0.0;
            for (int bt = warp; bt < nbat; bt += NW) {
                const int rb = r_begin + bt * RA + rl;
                uint4 kx[KSUM ? NA : 1], vx[DO_V ? NA : 1];
                if constexpr (KSUM) load_rows<NA, RPI>(kx, kp, a.k.sn, rb, r_end, keep);
                if constexpr (DO_V) load_rows<NA, RPI>(vx, vp, a.v.sn, rb, r_end, keep);
#pragma unroll
                for (int i = 0; i < NA; ++i) {
                    if constexpr (KSUM) {
                        float f[8];
                        unpack8(kx[i], f);
#pragma unroll
                        for (int e = 0; e < 8; ++e) s8[e] = __dadd_rn(s8[e], static_cast<double>(f[e]));
                    }
                    if (DO_V) {
                        m4[0] = bmax_abs(m4[0], vx[i].x);
                        m4[1] = bmax_abs(m4[1], vx[i].y);
                        m4[2] = bmax_abs(m4[2], vx[i].z);
                        m4[3] = bmax_abs(m4[3], vx[i].w);
                    }
                }
            }
            // the lanes VPR apart hold the same channels, then the warps in order
#pragma unroll
            for (int o = VPR; o < 32; o <<= 1) {
#pragma unroll
                for (int e = 0; e < 8; ++e) s8[e] = __dadd_rn(s8[e], __shfl_xor_sync(0xffffffffu, s8[e], o));
#pragma unroll
                for (int j = 0; j < 4; ++j) m4[j] = bmax_abs(m4[j], __shfl_xor_sync(0xffffffffu, m4[j], o));
            }
            if (lane < VPR) {
#pragma unroll
                for (int e = 0; e < 8; ++e) red_s[warp][vec * 8 + e] = s8[e];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    red_m[warp][vec * 8 + 2 * j] = bf_bits(m4[j] & 0xffffu);
                    red_m[warp][vec * 8 + 2 * j + 1] = bf_bits(m4[j] >> 16);
                }
            }
            __syncthreads();
            const int slot = blockIdx.x + h;
            for (int c = threadIdx.x; c < D; c += kPassThreads) {
                double ss = 0.0;
                float mm = 0.f;
#pragma unroll
                for (int w = 0; w < NW; ++w) {
                    ss = __dadd_rn(ss, red_s[w][c]);
                    mm = fmaxf(mm, red_m[w][c]);
                }
                if (KSUM) a.ksum_part[(int64_t)slot * D + c] = ss;
                if (DO_V) a.vmax_part[(int64_t)slot * D + c] = mm;
            }
            __syncthreads();  // every partial is written (and red_* free again)
            if (threadIdx.x == 0) {
                const long long x0 = (long long)h * nqb;
                const unsigned long long readers = owner(x0 + nqb - 1, nB) - owner(x0, nB) + 1;
                st_release_u64(a.flags + slot, (a.stamp << 16) | readers);
            }
        }
    }

    // ------------------------------------------------------------ phase B
    const uint64_t drop = l2_policy_evict_first();  // the last reads of Q, K and V
    const long long b0 = nB * blockIdx.x / G, b1 = nB * (blockIdx.x + 1) / G;
    const int grp = warp / WU, gw = warp % WU;  // warp group (one 128-token block at a time) and place in it
    int parity = 0;
    for (int h = (int)((b1 - 1) / nqb); h >= (int)(b0 / nqb); --h) {
        const int c0 = (int)((b0 > (long long)h * nqb ? b0 : (long long)h * nqb) - (long long)h * nqb);
        const int c1 = (int)((b1 < (long long)(h + 1) * nqb ? b1 : (long long)(h + 1) * nqb) - (long long)h * nqb);
        if constexpr (STATS) {
            __syncthreads();  // every warp is done with the previous head's statistics
            const int i0 = owner((long long)h * nsb, nA), i1 = owner((long long)h * nsb + nsb - 1, nA);
            for (int t = threadIdx.x; t <= i1 - i0; t += kPassThreads) {
                unsigned long long *f = a.flags + i0 + t + h;
                const long long t0 = clock64();
                bool ok = true;
                while ((ld_acquire_u64(f) >> 16) != a.stamp) {
                    if (*reinterpret_cast<volatile int *>(&abort_st.flag) || clock64() - t0 > kWaitLimitClocks) {
                        if (!*reinterpret_cast<volatile int *>(&abort_st.flag)) record_timeout(a.err, &abort_st, 10);
                        bad = 1;
                        ok = false;
                        break;
                    }
                    __nanosleep(64);
                }
                if (!ok) break;
                // one reader fewer; the last clears the flag (the partials are
                // written again only by a later launch)
                if ((atomicAdd(f, ~0ull) & 0xffffull) == 1ull) atomicExch(f, 0ull);
            }
            __syncthreads();
            if (bad) break;
            // the head's statistics: partials in CTA order (written by other
            // CTAs of this kernel: read through L2); mean = fp32(fp64 sum / N),
            // V factor 448 / amax
            for (int c = threadIdx.x; c < D; c += kPassThreads) {
                double sum = 0.0;
                float mx = 0.f;
                for (int i = i0; i <= i1; ++i) {
                    const int64_t o = (int64_t)(i + h) * D + c;
                    if (KSUM) sum = __dadd_rn(sum, __ldcg(a.ksum_part + o));
                    if (DO_V) mx = fmaxf(mx, __ldcg(a.vmax_part + o));
                }
                const float m = __double2float_rn(__ddiv_rn(sum, static_cast<double>(a.N)));
                mu[c] = m;
                vinv[c] = mx > 0.f ? 448.f / mx : 0.f;
                if (c0 == 0) {  // one CTA writes the per-head outputs
                    if (KSUM && a.user_k_mean) a.user_k_mean[(int64_t)h * D + c] = m;
                    if (DO_V) a.c.v_scale[(int64_t)h * D + c] = mx > 0.f ? mx / 448.f : 0.f;
                }
            }
            __syncthreads();
        }
        const int b = h / a.H, hh = h % a.H;
        for (int u = c1 - 1 - grp; u >= c0; u -= Gm::GROUPS) {
            const int rbase = u * kQBlock + gw * RB + rl;  // this lane's first row
            const int64_t obase = ((int64_t)h * a.n_pad + rbase) * D + vec * 8;
            float q_scale_unit = 0.f;  // POOL: the block's Q scale
            // all of the block's rows are requested at once: one memory latency per block
            uint4 xq[DO_Q ? NB : 1], xk[DO_K ? NB : 1], xv[DO_V ? NB : 1];
            if constexpr (DO_Q) load_rows<NB, RPI>(xq, a.q.p + b * a.q.sb + hh * a.q.sh + vec * 8, a.q.sn, rbase, a.N, drop);
            if constexpr (DO_K) load_rows<NB, RPI>(xk, a.k.p + b * a.k.sb + hh * a.k.sh + vec * 8, a.k.sn, rbase, a.N, drop);
            if constexpr (DO_V) load_rows<NB, RPI>(xv, a.v.p + b * a.v.sb + hh * a.v.sh + vec * 8, a.v.sn, rbase, a.N, drop);
            if constexpr (DO_Q) {
                const uint4 *x = xq;
                uint32_t am = 0u;
#pragma unroll
                for (int i = 0; i < NB; ++i)
                    am = bmax_abs(bmax_abs(bmax_abs(bmax_abs(am, x[i].x), x[i].y), x[i].z), x[i].w);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) am = bmax_abs(am, __shfl_xor_sync(0xffffffffu, am, o));
                float qa = fmaxf(bf_bits(am & 0xffffu), bf_bits(am >> 16));
                // the block's maximum over the group's warps
                if (lane == 0) grp_max[grp][parity][0][gw] = qa;
                group_sync(1 + grp, 32 * WU);
#pragma unroll
                for (int w = 0; w < WU; ++w) qa = fmaxf(qa, grp_max[grp][parity][0][w]);
                const float inv = qa > 0.f ? 127.f / qa : 0.f;
                uint32_t ps[4] = {0u, 0u, 0u, 0u};  // POOL: this lane's code sums per channel, int16 pairs
#pragma unroll
                for (int i = 0; i < NB; ++i) {
                    float f[8];
                    unpack8(x[i], f);
                    const uint2 cw = i8x8(f, inv);
                    *reinterpret_cast<uint2 *>(a.c.q_i8 + obase + (int64_t)i * RPI * D) = cw;
                    if constexpr (POOL) add_codes(ps, cw);
                }
                if constexpr (POOL) pool_partial<VPR>(ps, grp_pool[grp][0][gw], lane, vec);
                q_scale_unit = qa > 0.f ? qa / 127.f : 0.f;
                if (gw == 0 && lane == 0) a.c.q_scale[(int64_t)h * nqb + u] = q_scale_unit;
            }
            if constexpr (DO_K) {
                // the warp's rows lie in one 64-token K block, shared by KW warps
                const uint4 *x = xk;
                const int kb = (u * kQBlock + gw * RB) / kKBlock;
                float mu8[8];
                if constexpr (RES) {
                    // the block's mean: fp64 sum of its valid rows (exact for
                    // bf16 inputs), over the KW warps in order, one IEEE
                    // division, rounded to bf16
                    double s8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) s8[e] = 0.0;
#pragma unroll
                    for (int i = 0; i < NB; ++i) {
                        if (rbase + i * RPI < a.N) {
                            float f[8];
                            unpack8(x[i], f);
#pragma unroll
                            for (int e = 0; e < 8; ++e) s8[e] = __dadd_rn(s8[e], static_cast<double>(f[e]));
                        }
                    }
#pragma unroll
                    for (int o = VPR; o < 32; o <<= 1) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) s8[e] = __dadd_rn(s8[e], __shfl_xor_sync(0xffffffffu, s8[e], o));
                    }
                    if (KW > 1) {
                        if (lane < VPR) {
#pragma unroll
                            for (int e = 0; e < 8; ++e) grp_sum[grp][gw][vec * 8 + e] = s8[e];
                        }
                        group_sync(1 + grp, 32 * WU);
                        const int w0 = gw - gw % KW;
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            double t = 0.0;
#pragma unroll
                            for (int w = 0; w < KW; ++w) t = __dadd_rn(t, grp_sum[grp][w0 + w][vec * 8 + e]);
                            s8[e] = t;
                        }
                    }
                    const int nvalid = max(0, min(kKBlock, a.N - kb * kKBlock));
                    uint32_t mw[4];
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        const __nv_bfloat16 m0 =
                            __double2bfloat16(nvalid > 0 ? __ddiv_rn(s8[e], static_cast<double>(nvalid)) : 0.0);
                        const __nv_bfloat16 m1 =
                            __double2bfloat16(nvalid > 0 ? __ddiv_rn(s8[e + 1], static_cast<double>(nvalid)) : 0.0);
                        mu8[e] = __bfloat162float(m0);
                        mu8[e + 1] = __bfloat162float(m1);
                        mw[e / 2] = static_cast<uint32_t>(__bfloat16_as_ushort(m0)) |
                                    (static_cast<uint32_t>(__bfloat16_as_ushort(m1)) << 16);
                    }
                    if (gw % KW == 0 && lane < VPR)
                        *reinterpret_cast<uint4 *>(a.k_bmean + ((int64_t)h * nkb + kb) * D + vec * 8) =
                            make_uint4(mw[0], mw[1], mw[2], mw[3]);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) mu8[e] = mu[vec * 8 + e];
                }
                float ka = 0.f;
#pragma unroll
                for (int i = 0; i < NB; ++i) {
                    if (rbase + i * RPI < a.N) {  // rows past N stay zero (not -mean)
                        float f[8], d[8];
                        unpack8(x[i], f);
#pragma unroll
                        for (int e = 0; e < 8; e += 2) fsub2(d[e], d[e + 1], f[e], f[e + 1], mu8[e], mu8[e + 1]);
#pragma unroll
                        for (int e = 0; e < 8; ++e) ka = fmaxf(ka, fabsf(d[e]));
                    }
                }
                ka = warp_fmax(ka);
                if (KW > 1) {
                    if (lane == 0) grp_max[grp][parity][1][gw] = ka;
                    group_sync(1 + grp, 32 * WU);
                    const int w0 = gw - gw % KW;
#pragma unroll
                    for (int w = 0; w < KW; ++w) ka = fmaxf(ka, grp_max[grp][parity][1][w0 + w]);
                }
                const float inv = ka > 0.f ? 127.f / ka : 0.f;
                uint32_t ps[4] = {0u, 0u, 0u, 0u};  // POOL: this lane's code sums per channel, int16 pairs
#pragma unroll
                for (int i = 0; i < NB; ++i) {
                    float d[8];
                    if (rbase + i * RPI < a.N) {
                        float f[8];
                        unpack8(x[i], f);
#pragma unroll
                        for (int e = 0; e < 8; e += 2) fsub2(d[e], d[e + 1], f[e], f[e + 1], mu8[e], mu8[e + 1]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) d[e] = 0.f;
                    }
                    const uint2 cw = i8x8(d, inv);
                    *reinterpret_cast<uint2 *>(a.c.k_i8 + obase + (int64_t)i * RPI * D) = cw;
                    if constexpr (POOL) add_codes(ps, cw);
                }
                if (gw % KW == 0 && lane == 0) a.c.k_scale[(int64_t)h * nkb + kb] = ka > 0.f ? ka / 127.f : 0.f;
                if constexpr (POOL) {
                    pool_partial<VPR>(ps, grp_pool[grp][1][gw], lane, vec);
                    if (gw % KW == 0 && lane == 0) grp_ka[grp][gw / KW] = ka;
                    // the tile's pooled vectors (the code sums are exact in int16:
                    // at most 128 rows of |code| <= 127): qv = q_scale * sum of the Q
                    // codes, kvT = k_scale(2u) * sum of K block 2u + (the second block
                    // only if it holds a token) k_scale(2u+1) * its sum, one rounding
                    // per operation
                    group_sync(1 + grp, 32 * WU);
                    for (int t = gw * 32 + lane; t < D / 2; t += 32 * WU) {
                        uint32_t sq = 0u, s0 = 0u, s1 = 0u;
#pragma unroll
                        for (int w = 0; w < WU; ++w) {
                            sq = __vadd2(sq, grp_pool[grp][0][w][t]);
                            if (w < KW) s0 = __vadd2(s0, grp_pool[grp][1][w][t]);
                            else s1 = __vadd2(s1, grp_pool[grp][1][w][t]);
                        }
                        const float ks0 = grp_ka[grp][0] > 0.f ? grp_ka[grp][0] / 127.f : 0.f;
                        const float ks1 = grp_ka[grp][1] > 0.f ? grp_ka[grp][1] / 127.f : 0.f;
                        const bool second = (2 * u + 1) * kKBlock < a.N;
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            const int c = 2 * t + hf;
                            const float fq = static_cast<float>(static_cast<int16_t>(sq >> (16 * hf)));
                            const float f0 = static_cast<float>(static_cast<int16_t>(s0 >> (16 * hf)));
                            const float f1 = static_cast<float>(static_cast<int16_t>(s1 >> (16 * hf)));
                            a.pool_qv[((int64_t)h * nqb + u) * D + c] = __fmul_rn(q_scale_unit, fq);
                            const float k1 = second ? __fmul_rn(ks1, f1) : 0.f;
                            a.pool_kvT[((int64_t)h * D + c) * nqb + u] = __fadd_rn(__fmul_rn(ks0, f0), k1);
                        }
                    }
                }
            }
            if constexpr (DO_V) {
                const uint4 *x = xv;
                float vi8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) vi8[e] = vinv[vec * 8 + e];
#pragma unroll
                for (int i = 0; i < NB; ++i) {
                    float f[8];
                    unpack8(x[i], f);
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        // IEEE products (nothing is added); the conversion is
                        // volatile so that the vectors are coded one after
                        // another, not all unpacked at once
                        const float y0 = __fmul_rn(f[e], vi8[e]), y1 = __fmul_rn(f[e + 1], vi8[e + 1]);
                        w[e / 2] = e4m3x2(y0, y1);
                    }
                    *reinterpret_cast<uint2 *>(a.c.v_e4m3 + obase + (int64_t)i * RPI * D) =
                        make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
                }
            }
            parity ^= 1;
        }
    }
}

template <int D, bool DQ, bool DK, bool DV, bool RES = false, bool POOL = false>
cudaError_t launch_qpass_k(const Shape &s, const PassArgs &a, cudaStream_t st) {
    auto kern = k_qpass<D, DQ, DK, DV, RES, POOL>;
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t e;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kPassThreads, 0)) != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    // every CTA is resident at once (cooperative launch), so a CTA waiting on
    // another's phase-A partials never waits on one that has not started; no
    // more CTAs than 128-token blocks, nor than the statistics slots allow
    const long long grid = std::min<long long>(
        {(long long)sms * per_sm, (long long)s.BH() * s.n_qblocks(), (long long)kStatsMaxGrid});
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kPassThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

// A 48-bit stamp per call from a process-wide counter that starts at a
// clock-derived value; bit 47 is always set, so a zeroed flag never matches.
unsigned long long next_stamp() {
    static std::atomic<unsigned long long> counter{
        static_cast<unsigned long long>(std::chrono::steady_clock::now().time_since_epoch().count())};
    const unsigned long long v = counter.fetch_add(1, std::memory_order_relaxed) + 1;
    return (v & ((1ull << 48) - 1)) | (1ull << 47);
}

template <int D>
cudaError_t launch_qpass_d(const Shape &s, const Src *q, const Src *k, const Src *v, const StatsWs &ws,
                           float *user_k_mean, const Codes &c, uint16_t *k_bmean, float *pool_qv, float *pool_kvT,
                           cudaStream_t st) {
    PassArgs a{};
    const Src none{nullptr, 0, 0, 0};
    a.q = q ? *q : none;
    a.k = k ? *k : none;
    a.v = v ? *v : none;
    a.H = s.H;
    a.BH = s.BH();
    a.N = s.N;
    a.n_pad = s.n_pad();
    a.ksum_part = ws.ksum_part;
    a.vmax_part = ws.vmax_part;
    a.flags = ws.flags;
    a.stamp = next_stamp();
    a.user_k_mean = user_k_mean;
    a.k_bmean = k_bmean;
    a.pool_qv = pool_qv;
    a.pool_kvT = pool_kvT;
    a.c = c;
    if (!(a.err = device_error_ptr())) return cudaErrorSymbolNotFound;
    if (pool_qv || pool_kvT) {  // with the pooled tile vectors of the block selection
        if (q && k && v && !k_bmean && pool_qv && pool_kvT) return launch_qpass_k<D, true, true, true, false, true>(s, a, st);
        return cudaErrorInvalidValue;
    }
    if (k_bmean) {  // K-residual mode
        if (q && k && v) return launch_qpass_k<D, true, true, true, true>(s, a, st);
        if (!q && k && !v) return launch_qpass_k<D, false, true, false, true>(s, a, st);
        return cudaErrorInvalidValue;
    }
    if (q && k && v) return launch_qpass_k<D, true, true, true>(s, a, st);
    if (q && k && !v) return launch_qpass_k<D, true, true, false>(s, a, st);
    if (!q && k && v) return launch_qpass_k<D, false, true, true>(s, a, st);
    if (!q && !k && v) return launch_qpass_k<D, false, false, true>(s, a, st);
    if (q && !k && v) return launch_qpass_k<D, true, false, true>(s, a, st);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_qpass(const Shape &s, const Src *q, const Src *k, const Src *v, const StatsWs &ws,
                         float *user_k_mean, const Codes &c, cudaStream_t st, uint16_t *k_bmean, float *pool_qv,
                         float *pool_kvT) {
    return s.d == 128 ? launch_qpass_d<128>(s, q, k, v, ws, user_k_mean, c, k_bmean, pool_qv, pool_kvT, st)
                      : launch_qpass_d<64>(s, q, k, v, ws, user_k_mean, c, k_bmean, pool_qv, pool_kvT, st);
}

}  // namespace sage
