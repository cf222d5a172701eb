// sage_quant.cu -- the quantize pass of the quantized attention forward.
//
// Two HBM-bound streaming kernels (no tensor cores: there is no contraction):
//   k_stats  per (b,h, token chunk): sum of K (fp64, exact for bf16 inputs
//            whose values span fewer than 53 bits) and max |V| per channel
//            over the chunk, 64-token blocks staged through a 3-deep TMA ring
//   k_quant  per (b,h, 128-token block): finishes this (b,h)'s statistics from
//            the chunk partials (the K mean, the smoothing statistic, and the
//            448/amax factors of V) while TMA brings the block's Q, K and V
//            rows into shared memory, then Q block -> INT8, (K - mean) per
//            64-token block -> INT8, V -> e4m3 (token-major, like the codes of
//            Q and K; the attention kernel reads it as an MN-major operand).
// Pages: "MiniMax H3 接入 SageAttention 实测加速", section 一 (outlier smoothing of
// QK^T, INT8 QK, FP8 PV).  Block sizes, rounding and scale conventions are the
// readings C1-C3 and C7 of the design notes:
//   scale = amax/127 (fp32 IEEE divide), code = rne(x * fp32(127/amax)) in
//   [-127,127]; V: code = e4m3_rn_satfinite(v * fp32(448/amax_c)).
// Inputs are read through 4-D tensor maps over arbitrary (b,h,n) strides, so a
// fused-qkv view is read in place; codes are stored as 8-byte vectors.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

constexpr int kRowsPerLoad = 64;   // tokens per TMA box
constexpr int kStatsStages = 3;

// Shared-memory tile of `rows` tokens of one (b,h): [d/64][rows][64] bf16, as
// the 64-channel TMA boxes land.  Element (row, 8-channel vector cv) starts at:
__device__ __forceinline__ int tile_off(int rows, int row, int cv) {
    return ((cv >> 3) * rows + row) * 64 + (cv & 7) * 8;
}
__device__ __forceinline__ uint4 ld_tile(const uint16_t *tile, int off) {
    return *reinterpret_cast<const uint4 *>(tile + off);
}

// Issue the TMA loads of `rows` (a multiple of 64) tokens from token n of (b,h)
// into `tile` ([d/64][rows][64]), completing on `bar`.
// `policy` is the L2 eviction policy of the rows.
template <int D>
__device__ __forceinline__ void load_rows(uint16_t *tile, int rows, const CUtensorMap *map, int swap, uint64_t *bar,
                                          int n, int h, int b, uint64_t policy) {
#pragma unroll
    for (int half = 0; half < D / 64; ++half)
        for (int r = 0; r < rows; r += kRowsPerLoad) {
            uint16_t *dst = tile + (half * rows + r) * 64;
            if (swap)
                tma_load_4d_hint(dst, map, bar, half * 64, h, n + r, b, policy);
            else
                tma_load_4d_hint(dst, map, bar, half * 64, n + r, h, b, policy);
        }
}

// Max over the block of three values at once (all threads get the results).
// `sh` holds two slot sets [2][3][NT/32], used alternately (`set`): a set is
// written again only by the call after next, which every thread reaches after
// the next call's barrier, i.e. after all threads have read this call's slots;
// so one barrier per call suffices.
template <int NT>
__device__ __forceinline__ void block_max3_n(float &a, float &b, float &c, float *shs, int set) {
    constexpr int NW = NT / 32;
    float *sh = shs + set * 3 * NW;
    a = warp_max(a);
    b = warp_max(b);
    c = warp_max(c);
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) { sh[w] = a; sh[NW + w] = b; sh[2 * NW + w] = c; }
    __syncthreads();
    a = sh[0];
    b = sh[NW];
    c = sh[2 * NW];
#pragma unroll
    for (int i = 1; i < NW; ++i) { a = fmaxf(a, sh[i]); b = fmaxf(b, sh[NW + i]); c = fmaxf(c, sh[2 * NW + i]); }
}

// Persistent CTAs over the (b,h, token chunk) items, a contiguous range each,
// with a ring of kStatsStages 64-token stages kept full across item boundaries.
struct StatsArgs {
    int H, BH, N, nch, chunk, per;  // per: items per CTA
    int do_k, do_v, k_swap, v_swap;
    double *ksum_part;  // [BH][nch][D]
    float *vmax_part;   // [BH][nch][D]
    unsigned *err;
};

template <int D>
__global__ void __launch_bounds__(kThreads) k_stats(const __grid_constant__ CUtensorMap tk,
                                                    const __grid_constant__ CUtensorMap tv, const StatsArgs a) {
    constexpr int VPR = D / 8;              // 16-byte vectors per token row
    constexpr int RPI = kThreads / VPR;     // rows covered per pass of the block
    constexpr int TILE = kRowsPerLoad * D;  // elements of one tensor in one stage
    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint16_t *ring = reinterpret_cast<uint16_t *>(smem_raw);                    // [stage][K,V][TILE]
    double *red_s = reinterpret_cast<double *>(ring + kStatsStages * 2 * TILE);  // [warps][D]
    float *red_m = reinterpret_cast<float *>(red_s + (kThreads / 32) * D);      // [RPI][D]
    __shared__ uint64_t full[kStatsStages];
    __shared__ AbortState abort_st;
    __shared__ int bad;
    const int n_items = a.nch * a.BH;
    const int i0 = blockIdx.x * a.per, i1 = min(n_items, i0 + a.per);
    const int cv = threadIdx.x % VPR, r0 = threadIdx.x / VPR;
    const uint32_t bytes = (a.do_k + a.do_v) * TILE * 2;
    grid_dep_launch();  // the quantize kernel may take each SM this CTA leaves
    auto rows_of = [&](int item) {
        const int n0 = (item % a.nch) * a.chunk;
        return min(a.N, n0 + a.chunk) - n0;
    };
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStatsStages; ++i) mbar_init(&full[i], 1);
        abort_st.flag = 0;
        bad = 0;
        fence_barrier_init();
    }
    __syncthreads();
    // Stage sequence numbers count the CTA's 64-token loads in order.  Thread 0
    // keeps the producer state: the next sub-block to load, how many loads it
    // issued, how many the block consumed, and how many it saw complete.
    int p_item = i0, p_sb = 0, issued = 0, consumed = 0, waited = 0;
    // K and V are read again by the quantize pass right after: keep them in L2
    const uint64_t keep = l2_policy_evict_last();
    auto issue_more = [&]() {
        while (!bad && p_item < i1 && issued < consumed + kStatsStages) {
            const int st = issued % kStatsStages;
            uint16_t *base = ring + st * 2 * TILE;
            const int bh = p_item / a.nch, b = bh / a.H, h = bh % a.H;
            const int n = (p_item % a.nch) * a.chunk + p_sb * kRowsPerLoad;
            mbar_arrive_expect_tx(&full[st], bytes);
            if (a.do_k) load_rows<D>(base, kRowsPerLoad, &tk, a.k_swap, &full[st], n, h, b, keep);
            if (a.do_v) load_rows<D>(base + TILE, kRowsPerLoad, &tv, a.v_swap, &full[st], n, h, b, keep);
            ++issued;
            if (++p_sb * kRowsPerLoad >= rows_of(p_item)) {
                ++p_item;
                p_sb = 0;
            }
        }
    };
    if (threadIdx.x == 0) issue_more();
    int qbase = 0;  // sequence number of the item's first sub-block (every thread)
    for (int item = i0; item < i1; ++item) {
        const int rows = rows_of(item);
        const int nsub = (rows + kRowsPerLoad - 1) / kRowsPerLoad;
        double s[8];
        float m[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) { s[e] = 0.0; m[e] = 0.f; }
        for (int sb = 0; sb < nsub; ++sb) {
            const int q = qbase + sb;
            const int st = q % kStatsStages;
            if (threadIdx.x == 0 && !bad) {
                if (wait_one(&full[st], (q / kStatsStages) & 1, a.err, &abort_st, false, 0))
                    waited = q + 1;
                else
                    bad = 1;
            }
            __syncthreads();
            if (!bad) {
                const uint16_t *kt = ring + st * 2 * TILE, *vt = kt + TILE;
#pragma unroll
                for (int i = 0; i < kRowsPerLoad / RPI; ++i) {
                    const int row = r0 + i * RPI;
                    if (sb * kRowsPerLoad + row < rows) {  // the box may reach into the next chunk
                        float f[8];
                        if (a.do_k) {
                            unpack8(ld_tile(kt, tile_off(kRowsPerLoad, row, cv)), f);
#pragma unroll
                            for (int e = 0; e < 8; ++e) s[e] = __dadd_rn(s[e], static_cast<double>(f[e]));
                        }
                        if (a.do_v) {
                            unpack8(ld_tile(vt, tile_off(kRowsPerLoad, row, cv)), f);
#pragma unroll
                            for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(f[e]));
                        }
                    }
                }
            }
            __syncthreads();  // the stage is free again
            if (threadIdx.x == 0) {
                consumed = q + 1;
                issue_more();
            }
        }
        qbase += nsub;
        // the item's partials: the K sums of a warp's rows by shuffles (the
        // lanes VPR apart hold the same channels), then the warps in order;
        // the V maxima per row of the block, then per channel
#pragma unroll
        for (int e = 0; e < 8; ++e) {
#pragma unroll
            for (int o = VPR; o < 32; o <<= 1) s[e] = __dadd_rn(s[e], __shfl_xor_sync(0xffffffffu, s[e], o));
            red_m[r0 * D + cv * 8 + e] = m[e];
        }
        if ((threadIdx.x & 31) < VPR) {
#pragma unroll
            for (int e = 0; e < 8; ++e) red_s[(threadIdx.x >> 5) * D + cv * 8 + e] = s[e];
        }
        __syncthreads();
        for (int c = threadIdx.x; c < D; c += kThreads) {
            double ss = 0.0;
            float mm = 0.f;
            for (int w = 0; w < kThreads / 32; ++w) ss = __dadd_rn(ss, red_s[w * D + c]);
            for (int r = 0; r < RPI; ++r) mm = fmaxf(mm, red_m[r * D + c]);
            const int64_t o = (int64_t)item * D + c;  // item = bh * nch + chunk
            if (a.do_k) a.ksum_part[o] = ss;
            if (a.do_v) a.vmax_part[o] = mm;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        // every copy started here lands before the CTA exits
        for (int q = waited; q < issued; ++q)
            wait_one(&full[q % kStatsStages], (q / kStatsStages) & 1, a.err, &abort_st, true, 0);
    }
}

// Threads of a quantize CTA: 512 (one CTA per SM) for d = 128, 256 (two CTAs
// per SM, so two items are in flight per SM) for d = 64.
template <int D>
__host__ __device__ constexpr int quant_threads() { return D == 128 ? 512 : 256; }

// Persistent CTAs over the (b,h, 128-token block) items, a contiguous range
// each (so consecutive items share a (b,h) and its statistics), two buffers:
// the next item's Q, K and V rows land while the current one is coded.
struct QuantArgs {
    int H, BH, N, n_pad, nch, per;
    int q_swap, k_swap, v_swap;
    const double *ksum_part;  // [BH][nch][D]
    const float *vmax_part;   // [BH][nch][D]
    float *ws_k_mean, *ws_v_inv;         // [BH][D], written with the first block of each (b,h)
    float *user_k_mean;                  // optional copy of the K mean
    Codes c;
    unsigned *err;
};

template <int D, bool DO_Q, bool DO_K, bool DO_V>
__global__ void __launch_bounds__(quant_threads<D>(), 512 / quant_threads<D>()) k_quant(const __grid_constant__ CUtensorMap tq,
                                                        const __grid_constant__ CUtensorMap tk,
                                                        const __grid_constant__ CUtensorMap tv, const QuantArgs a) {
    constexpr int NTH = quant_threads<D>();
    constexpr int VPR = D / 8;
    constexpr int RPI = NTH / VPR;
    constexpr int NI = kQBlock / RPI;  // vectors per thread in one 128-token block
    constexpr int TILE = kQBlock * D;
    constexpr int NT = (DO_Q ? 1 : 0) + (DO_K ? 1 : 0) + (DO_V ? 1 : 0);
    constexpr int OQ = 0, OK = (DO_Q ? 1 : 0), OV = OK + (DO_K ? 1 : 0);  // tensor slots in a buffer
    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint16_t *bufs = reinterpret_cast<uint16_t *>(smem_raw);  // [2][NT][TILE]
    __shared__ uint64_t bar[2];
    __shared__ float mu[D], vinv[D], vmax[D];
    __shared__ float red[2 * 3 * (NTH / 32)];
    __shared__ AbortState abort_st;
    __shared__ int bad;
    const int nqb = a.n_pad / kQBlock, nkb = a.n_pad / kKBlock;
    const int n_items = nqb * a.BH;
    const int i0 = blockIdx.x * a.per, i1 = min(n_items, i0 + a.per);
    const int cv = threadIdx.x % VPR, r0 = threadIdx.x / VPR;

    if (threadIdx.x == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        abort_st.flag = 0;
        bad = 0;
        fence_barrier_init();
    }
    __syncthreads();
    // the last reads of Q, K and V: let them leave L2 first
    const uint64_t drop = l2_policy_evict_first();
    auto issue = [&](int item, int buf) {
        const int bh = item / nqb, blk = item % nqb, b = bh / a.H, h = bh % a.H;
        uint16_t *base = bufs + buf * NT * TILE;
        mbar_arrive_expect_tx(&bar[buf], NT * TILE * 2);
        if (DO_Q) load_rows<D>(base + OQ * TILE, kQBlock, &tq, a.q_swap, &bar[buf], blk * kQBlock, h, b, drop);
        if (DO_K) load_rows<D>(base + OK * TILE, kQBlock, &tk, a.k_swap, &bar[buf], blk * kQBlock, h, b, drop);
        if (DO_V) load_rows<D>(base + OV * TILE, kQBlock, &tv, a.v_swap, &bar[buf], blk * kQBlock, h, b, drop);
    };
    int issued = 0, waited = 0;  // thread 0: loads issued, and seen complete
    grid_dep_launch();  // the attention kernel may take each SM this CTA leaves
    // The rows are the caller's inputs, complete before the statistics kernel
    // started: the first item's loads go out before the wait for that kernel's
    // partials (and before anything here is written).
    if (threadIdx.x == 0 && i0 < i1) {
        issue(i0, 0);
        issued = 1;
    }
    grid_dep_wait();
    int cur_bh = -1;
    for (int item = i0, k = 0; item < i1; ++item, ++k) {
        const int buf = k & 1;
        const int bh = item / nqb, blk = item % nqb;
        if ((DO_K || DO_V) && bh != cur_bh) {
            // this (b,h)'s statistics from the chunk partials, in chunk order:
            // mean = fp32(fp64 sum / N) (IEEE divide, then one rounding to
            // fp32), V factor 448 / amax
            __syncthreads();  // every thread is done coding with the previous head's
            for (int c = threadIdx.x; c < D; c += NTH) {
                double sum = 0.0;
                float mx = 0.f;
#pragma unroll 8
                for (int ch = 0; ch < a.nch; ++ch) {
                    const int64_t o = ((int64_t)bh * a.nch + ch) * D + c;
                    if (DO_K) sum = __dadd_rn(sum, a.ksum_part[o]);
                    if (DO_V) mx = fmaxf(mx, a.vmax_part[o]);
                }
                mu[c] = __double2float_rn(__ddiv_rn(sum, static_cast<double>(a.N)));
                vmax[c] = mx;
                vinv[c] = mx > 0.f ? 448.f / mx : 0.f;
            }
            cur_bh = bh;
        }
        if (threadIdx.x == 0 && !bad) {
            if (wait_one(&bar[buf], (k >> 1) & 1, a.err, &abort_st, false, 0))
                waited = k + 1;
            else
                bad = 1;
        }
        // the rows and the statistics are ready, and every thread is done with
        // the previous item, so its buffer takes the next item's rows
        __syncthreads();
        if (threadIdx.x == 0 && !bad && item + 1 < i1) {
            issue(item + 1, buf ^ 1);
            ++issued;
        }
        if (blk == 0 && (DO_K || DO_V)) {
            for (int c = threadIdx.x; c < D; c += NTH) {
                if (DO_K) {
                    a.ws_k_mean[bh * D + c] = mu[c];
                    if (a.user_k_mean) a.user_k_mean[bh * D + c] = mu[c];
                }
                if (DO_V) {
                    a.ws_v_inv[bh * D + c] = vinv[c];
                    a.c.v_scale[bh * D + c] = vmax[c] > 0.f ? vmax[c] / 448.f : 0.f;
                }
            }
        }
        const int row0 = blk * kQBlock;
        const uint16_t *base = bufs + buf * NT * TILE;

        // Q and the smoothed K of this thread's rows stay in registers from the
        // maximum to the codes; one block reduction serves Q and both K blocks.
        float qv[DO_Q ? NI : 1][8], kv[DO_K ? NI : 1][8];
        float qa = 0.f, ka0 = 0.f, ka1 = 0.f;
        if (!bad) {
            if (DO_Q) {
#pragma unroll
                for (int i = 0; i < NI; ++i) {
                    unpack8(ld_tile(base + OQ * TILE, tile_off(kQBlock, r0 + i * RPI, cv)), qv[i]);
#pragma unroll
                    for (int e = 0; e < 8; ++e) qa = fmaxf(qa, fabsf(qv[i][e]));
                }
            }
            if (DO_K) {
                float m8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) m8[e] = mu[cv * 8 + e];
#pragma unroll
                for (int i = 0; i < NI; ++i) {
                    const int row = r0 + i * RPI;
                    if (row0 + row < a.N) {  // rows past N stay zero (not -mean)
                        float f[8];
                        unpack8(ld_tile(base + OK * TILE, tile_off(kQBlock, row, cv)), f);
#pragma unroll
                        for (int e = 0; e < 8; e += 2) fsub2(kv[i][e], kv[i][e + 1], f[e], f[e + 1], m8[e], m8[e + 1]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) kv[i][e] = 0.f;
                    }
                    float am = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) am = fmaxf(am, fabsf(kv[i][e]));
                    if (row < kKBlock) ka0 = fmaxf(ka0, am); else ka1 = fmaxf(ka1, am);
                }
            }
            block_max3_n<NTH>(qa, ka0, ka1, red, k & 1);
        }

        if (DO_Q && !bad) {
            const float inv = qa > 0.f ? 127.f / qa : 0.f;
            int8_t *dst = a.c.q_i8 + ((int64_t)bh * a.n_pad + row0) * D + cv * 8;
#pragma unroll
            for (int i = 0; i < NI; ++i)
                *reinterpret_cast<uint2 *>(dst + (int64_t)(r0 + i * RPI) * D) = i8x8(qv[i], inv);
            if (threadIdx.x == 0) a.c.q_scale[(int64_t)bh * nqb + blk] = qa > 0.f ? qa / 127.f : 0.f;
        }

        if (DO_K && !bad) {
            const float inv0 = ka0 > 0.f ? 127.f / ka0 : 0.f;
            const float inv1 = ka1 > 0.f ? 127.f / ka1 : 0.f;
            int8_t *dst = a.c.k_i8 + ((int64_t)bh * a.n_pad + row0) * D + cv * 8;
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                const int row = r0 + i * RPI;
                *reinterpret_cast<uint2 *>(dst + (int64_t)row * D) = i8x8(kv[i], row < kKBlock ? inv0 : inv1);
            }
            if (threadIdx.x == 0) {
                a.c.k_scale[(int64_t)bh * nkb + 2 * blk] = ka0 > 0.f ? ka0 / 127.f : 0.f;
                a.c.k_scale[(int64_t)bh * nkb + 2 * blk + 1] = ka1 > 0.f ? ka1 / 127.f : 0.f;
            }
        }

        if (DO_V && !bad) {
            const uint16_t *tile = base + OV * TILE;
            float inv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) inv[e] = vinv[cv * 8 + e];
            uint8_t *dst = a.c.v_e4m3 + ((int64_t)bh * a.n_pad + row0) * D + cv * 8;
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                float f[8];
                unpack8(ld_tile(tile, tile_off(kQBlock, r0 + i * RPI, cv)), f);
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    float y0, y1;
                    fmul2(y0, y1, f[e], f[e + 1], inv[e], inv[e + 1]);  // IEEE products; nothing is added
                    uint16_t pr;
                    // cvt packs its first source in the high byte: (hi=e+1, lo=e)
                    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pr) : "f"(y1), "f"(y0));
                    w[e / 2] = pr;
                }
                *reinterpret_cast<uint2 *>(dst + (int64_t)(r0 + i * RPI) * D) =
                    make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
            }
        }
    }
    if (threadIdx.x == 0) {
        // every copy started here lands before the CTA exits
        for (int k = waited; k < issued; ++k) wait_one(&bar[k & 1], (k >> 1) & 1, a.err, &abort_st, true, 0);
    }
}

// Raise a kernel's dynamic shared-memory limit on the current device once:
// the attribute belongs to the device, so `done` keeps one bit per device
// index (indices past 63 set it on every call).
template <typename K>
cudaError_t ensure_smem_limit(K kern, int smem, std::atomic<uint64_t> &done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev >= 0 && dev < 64 ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_relaxed) & bit)) return cudaSuccess;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess) return e;
    done.fetch_or(bit, std::memory_order_relaxed);
    return cudaSuccess;
}

// CTAs that fit at once on the device for a kernel and its dynamic shared memory.
template <typename K>
int resident_ctas(K kern, int threads, int smem) {
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) != cudaSuccess)
        return 0;
    return sms * per_sm;
}

template <int D>
cudaError_t launch_stats_d(const Shape &s, const Src *k, const Src *v, const StatsWs &ws, cudaStream_t st) {
    CUtensorMap tk, tv;
    StatsArgs a{};
    cudaError_t e;
    if (k && (e = make_bf16_token_map(&tk, *k, s, kRowsPerLoad, &a.k_swap)) != cudaSuccess) return e;
    if (v && (e = make_bf16_token_map(&tv, *v, s, kRowsPerLoad, &a.v_swap)) != cudaSuccess) return e;
    if (!k) tk = tv;
    if (!v) tv = tk;
    a.H = s.H;
    a.BH = s.BH();
    a.N = s.N;
    a.nch = s.n_chunks();
    a.chunk = s.chunk_rows();
    a.do_k = k != nullptr;
    a.do_v = v != nullptr;
    a.ksum_part = ws.ksum_part;
    a.vmax_part = ws.vmax_part;
    if (!(a.err = device_error_ptr())) return cudaErrorSymbolNotFound;
    constexpr int RPI = kThreads / (D / 8);
    const int smem = kStatsStages * 2 * kRowsPerLoad * D * 2 + (kThreads / 32) * D * 8 + RPI * D * 4;
    static std::atomic<uint64_t> limit_set{0};  // one per instantiation
    if ((e = ensure_smem_limit(k_stats<D>, smem, limit_set)) != cudaSuccess) return e;
    const int items = a.nch * s.BH();
    const int ctas = resident_ctas(k_stats<D>, kThreads, smem);
    if (ctas <= 0) return cudaErrorInvalidConfiguration;
    a.per = (items + ctas - 1) / ctas;
    k_stats<D><<<(items + a.per - 1) / a.per, kThreads, smem, st>>>(tk, tv, a);
    return cudaGetLastError();
}

template <int D, bool DQ, bool DK, bool DV>
cudaError_t launch_quant_k(const Shape &s, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                           QuantArgs a, cudaStream_t st) {
    constexpr int NT = (DQ ? 1 : 0) + (DK ? 1 : 0) + (DV ? 1 : 0);
    const int smem = 2 * NT * kQBlock * D * 2;
    auto kern = k_quant<D, DQ, DK, DV>;
    static std::atomic<uint64_t> limit_set{0};  // one per instantiation
    cudaError_t e;
    if ((e = ensure_smem_limit(kern, smem, limit_set)) != cudaSuccess) return e;
    const int items = s.n_qblocks() * s.BH();
    const int ctas = resident_ctas(kern, quant_threads<D>(), smem);
    if (ctas <= 0) return cudaErrorInvalidConfiguration;
    a.per = (items + ctas - 1) / ctas;
    return launch_dependent(kern, dim3((items + a.per - 1) / a.per), dim3(quant_threads<D>()), smem, st, tq, tk, tv,
                            a);
}

template <int D>
cudaError_t launch_quant_d(const Shape &s, const Src *q, const Src *k, const Src *v, const StatsWs &ws,
                           float *user_k_mean, const Codes &c, cudaStream_t st) {
    CUtensorMap tq, tk, tv;
    QuantArgs a{};
    cudaError_t e;
    if (q && (e = make_bf16_token_map(&tq, *q, s, kRowsPerLoad, &a.q_swap)) != cudaSuccess) return e;
    if (k && (e = make_bf16_token_map(&tk, *k, s, kRowsPerLoad, &a.k_swap)) != cudaSuccess) return e;
    if (v && (e = make_bf16_token_map(&tv, *v, s, kRowsPerLoad, &a.v_swap)) != cudaSuccess) return e;
    const CUtensorMap &any = q ? tq : (k ? tk : tv);
    if (!q) tq = any;
    if (!k) tk = any;
    if (!v) tv = any;
    a.H = s.H;
    a.BH = s.BH();
    a.N = s.N;
    a.n_pad = s.n_pad();
    a.nch = s.n_chunks();
    a.ksum_part = ws.ksum_part;
    a.vmax_part = ws.vmax_part;
    a.ws_k_mean = ws.k_mean;
    a.ws_v_inv = ws.v_inv;
    a.user_k_mean = user_k_mean;
    a.c = c;
    if (!(a.err = device_error_ptr())) return cudaErrorSymbolNotFound;
    if (q && k && v) return launch_quant_k<D, true, true, true>(s, tq, tk, tv, a, st);
    if (q && k && !v) return launch_quant_k<D, true, true, false>(s, tq, tk, tv, a, st);
    if (!q && k && v) return launch_quant_k<D, false, true, true>(s, tq, tk, tv, a, st);
    if (!q && !k && v) return launch_quant_k<D, false, false, true>(s, tq, tk, tv, a, st);
    if (q && !k && v) return launch_quant_k<D, true, false, true>(s, tq, tk, tv, a, st);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_stats(const Shape &s, const Src *k, const Src *v, const StatsWs &ws, cudaStream_t st) {
    return s.d == 128 ? launch_stats_d<128>(s, k, v, ws, st) : launch_stats_d<64>(s, k, v, ws, st);
}

cudaError_t launch_quant(const Shape &s, const Src *q, const Src *k, const Src *v, const StatsWs &ws,
                         float *user_k_mean, const Codes &c, cudaStream_t st) {
    return s.d == 128 ? launch_quant_d<128>(s, q, k, v, ws, user_k_mean, c, st)
                      : launch_quant_d<64>(s, q, k, v, ws, user_k_mean, c, st);
}

}  // namespace sage
