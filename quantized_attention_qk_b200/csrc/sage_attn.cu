// sage_attn.cu -- fused quantized attention kernel for sm_100a.
//
// One CTA computes two 128-query tiles (Q0, Q1) of one (batch, head) against
// all keys, 128 keys per step, never writing the score matrix out
// ("GitHub榜单静默期：Attention优化从架构转向推理加速", section 2.2).  Scores come
// from INT8 tensor-core products and P.V from FP8 (e4m3) products
// ("MiniMax H3 接入 SageAttention 实测加速", section 一).
//
// Warp roles (320 threads):
//   warps 0-3  softmax warpgroup of Q tile 0 (one query row per thread)
//   warps 4-7  softmax warpgroup of Q tile 1
//   warp  8    TMA producer: Q tiles once, then a ring of (K tile, V^T tile) stages
//   warp  9    tensor-memory allocator and single-thread tcgen05.mma issuer
// Tensor memory (512 columns x 128 lanes):
//   [0,128) S0 int32, [128,256) S1 int32, [256,256+d) O0 fp32, [256+d,256+2d) O1 fp32.
//   P_t (e4m3, 4 per column) overwrites columns [0,32) of S_t after softmax.
// Per KV step j the issue order is  PV0(j), S0(j+1), PV1(j), S1(j+1): while one
// warpgroup runs its softmax the tensor core works on the other tile.
// Numerics (readings C4-C8): x = S*(sq*sm_scale*log2e*sk) with one sk per
// 64-key block; running max m' = max(m, ceil(rowmax x)) so that the O / l
// rescale 2^(m-m') is an exact power of two; P = e4m3(2^(x-m') * 448) computed as
// 2^(x - m' + log2 448); l accumulates the unrounded values; the epilogue
// writes bf16(O * v_scale / l).
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
    static constexpr int STAGES = D == 128 ? 3 : 4;
    static constexpr int Q_BYTES = BM * D;
    static constexpr int K_BYTES = BN * D;
    static constexpr int V_BYTES = D * BN;
    static constexpr int TILE_BYTES = 2 * Q_BYTES + STAGES * (K_BYTES + V_BYTES);
    static constexpr uint32_t T_S0 = 0, T_S1 = 128, T_O0 = 256, T_O1 = 256 + D;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int THREADS = 320;
};

template <int D>
struct Ctl {
    uint64_t q_full;
    uint64_t kv_full[Cfg<D>::STAGES];
    uint64_t kv_empty[Cfg<D>::STAGES];
    uint64_t s_full[2];
    uint64_t p_ready[2];
    uint64_t o_done[2];
    uint64_t drain;
    uint32_t tmem_base;
    AbortState abort;
    float v_scale[D];
};

// At least 120 KB so that a second CTA never shares the SM: each CTA takes
// all 512 tensor-memory columns.
template <int D>
constexpr int smem_bytes() {
    constexpr int need = Cfg<D>::TILE_BYTES + static_cast<int>(sizeof(Ctl<D>)) + 1024;
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
};

// 2^k for an integer-valued k <= 0 (exact; 0 below the normal range).
__device__ __forceinline__ float exp2_int(float k) {
    const int e = 127 + static_cast<int>(k);
    return e > 0 ? __int_as_float(e << 23) : 0.f;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

template <int D, bool EXPORT_S>
__global__ void __launch_bounds__(Cfg<D>::THREADS, 1)
    k_attn(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
           const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = base;
    uint8_t *sK = base + 2 * C::Q_BYTES;
    uint8_t *sV = sK + C::STAGES * C::K_BYTES;
    Ctl<D> *ctl = reinterpret_cast<Ctl<D> *>(sV + C::STAGES * C::V_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = EXPORT_S ? p.bh0 : static_cast<int>(blockIdx.y);
    const int qt0 = EXPORT_S ? p.q_tile0 : 2 * static_cast<int>(blockIdx.x);
    const int kv0 = EXPORT_S ? p.kv_tile0 : 0;
    const int nkv = EXPORT_S ? 1 : (p.N + C::BN - 1) / C::BN;

    if (threadIdx.x == 0) {
        mbar_init(&ctl->q_full, 1);
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&ctl->kv_full[s], 1);
            mbar_init(&ctl->kv_empty[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&ctl->s_full[t], 1);
            mbar_init(&ctl->p_ready[t], 128);
            mbar_init(&ctl->o_done[t], 1);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort.flag = 0;
        fence_barrier_init();
    }
    if (warp == 8 && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        if (!EXPORT_S) tma_prefetch_desc(&tm_v);
    }
    for (int i = threadIdx.x; i < D; i += blockDim.x) ctl->v_scale[i] = EXPORT_S ? 0.f : p.v_scale[bh * D + i];
    if (warp == 9) {
        tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;

    if (warp == 8) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_arrive_expect_tx(&ctl->q_full, 2 * C::Q_BYTES);
            tma_load_3d(sQ, &tm_q, &ctl->q_full, 0, qt0 * C::BM, bh);
            tma_load_3d(sQ + C::Q_BYTES, &tm_q, &ctl->q_full, 0, (qt0 + 1) * C::BM, bh);
            int issued = 0;
            for (int j = 0; j < nkv; ++j) {
                const int s = j % C::STAGES;
                if (j >= C::STAGES &&
                    !wait_one(&ctl->kv_empty[s], ((j / C::STAGES) - 1) & 1, p.err, &ctl->abort))
                    break;
                mbar_arrive_expect_tx(&ctl->kv_full[s], EXPORT_S ? C::K_BYTES : C::K_BYTES + C::V_BYTES);
                tma_load_3d(sK + s * C::K_BYTES, &tm_k, &ctl->kv_full[s], 0, (kv0 + j) * C::BN, bh);
                if (!EXPORT_S)
                    tma_load_3d(sV + s * C::V_BYTES, &tm_v, &ctl->kv_full[s], (kv0 + j) * C::BN, 0, bh);
                issued = j + 1;
            }
            // every copy started here lands before the CTA may exit
            wait_one(&ctl->q_full, 0, p.err, &ctl->abort, true);
            for (int j = issued > C::STAGES ? issued - C::STAGES : 0; j < issued; ++j)
                wait_one(&ctl->kv_full[j % C::STAGES], (j / C::STAGES) & 1, p.err, &ctl->abort, true);
        }
    } else if (warp == 9) {
        // ----------------------------------------------------------- MMA issue
        if (lane == 0) {
            const uint32_t idesc_qk = idesc_i8_s32(128, C::BN);
            const uint32_t idesc_pv = idesc_e4m3_f32(128, D);
            const uint32_t q_addr[2] = {smem_u32(sQ), smem_u32(sQ) + C::Q_BYTES};
            auto issue_qk = [&](int t, int s) {
                const uint32_t kb = smem_u32(sK + s * C::K_BYTES);
                const uint32_t dt = tmem + (t ? C::T_S1 : C::T_S0);
#pragma unroll
                for (int kk = 0; kk < D / 32; ++kk)
                    mma_i8_ss(dt, smem_desc_kmajor(q_addr[t] + kk * 32, D), smem_desc_kmajor(kb + kk * 32, D),
                              idesc_qk, kk > 0 ? 1u : 0u);
                tc_commit(&ctl->s_full[t]);
            };
            auto issue_pv = [&](int t, int s, int j) {
                const uint32_t vb = smem_u32(sV + s * C::V_BYTES);
                const uint32_t dt = tmem + (t ? C::T_O1 : C::T_O0);
                const uint32_t at = tmem + (t ? C::T_S1 : C::T_S0);
#pragma unroll
                for (int kk = 0; kk < C::BN / 32; ++kk)
                    mma_f8_ts(dt, at + kk * 8, smem_desc_kmajor(vb + kk * 32, C::BN), idesc_pv,
                              (j > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&ctl->o_done[t]);
            };
            bool ok = wait_one(&ctl->q_full, 0, p.err, &ctl->abort) &&
                      wait_one(&ctl->kv_full[0], 0, p.err, &ctl->abort);
            if (ok) {
                tc_fence_after();
                issue_qk(0, 0);
                issue_qk(1, 0);
            }
            for (int j = 0; ok && j < nkv; ++j) {
                const int s = j % C::STAGES;
                if (!(ok = wait_one(&ctl->p_ready[0], j & 1, p.err, &ctl->abort))) break;
                tc_fence_after();
                if (!EXPORT_S) issue_pv(0, s, j);
                if (j + 1 < nkv) {
                    const int s2 = (j + 1) % C::STAGES;
                    if (!(ok = wait_one(&ctl->kv_full[s2], ((j + 1) / C::STAGES) & 1, p.err, &ctl->abort))) break;
                    tc_fence_after();
                    issue_qk(0, s2);
                }
                if (!(ok = wait_one(&ctl->p_ready[1], j & 1, p.err, &ctl->abort))) break;
                tc_fence_after();
                if (!EXPORT_S) issue_pv(1, s, j);
                tc_commit(&ctl->kv_empty[s]);
                if (j + 1 < nkv) issue_qk(1, (j + 1) % C::STAGES);
            }
            // all MMAs issued here finish before tensor memory is released
            tc_commit(&ctl->drain);
            wait_one(&ctl->drain, 0, p.err, &ctl->abort, true);
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int t = warp >> 2;         // Q tile of this warpgroup
        const int wq = warp & 3;         // tensor-memory lane quarter
        const int row_in_tile = wq * 32 + lane;
        const int qt = qt0 + t;
        const int row = qt * C::BM + row_in_tile;
        const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tmem + lane_off + (t ? C::T_S1 : C::T_S0);
        const uint32_t tO = tmem + lane_off + (t ? C::T_O1 : C::T_O0);
        const float sq = qt < p.nqb ? p.q_scale[(int64_t)bh * p.nqb + qt] : 0.f;
        const float cq = sq * p.s_l2;
        const float kLog2_448 = 8.807354922057604f;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nkv; ++j) {
            if (!(ok = wait_warp(&ctl->s_full[t], j & 1, p.err, &ctl->abort))) break;
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
            uint32_t pk[32];
            if (EXPORT_S) {
                if (t == 0) {
                    int32_t *dst = p.s_export + row_in_tile * C::BN;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        dst[i] = static_cast<int32_t>(ra[i]);
                        dst[32 + i] = static_cast<int32_t>(rb[i]);
                        dst[64 + i] = static_cast<int32_t>(rc[i]);
                        dst[96 + i] = static_cast<int32_t>(rd[i]);
                    }
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) pk[i] = 0;
            } else {
                const int kvt = kv0 + j;
                const int kv_valid = min(C::BN, p.N - kvt * C::BN);
                const float c0 = cq * p.k_scale[(int64_t)bh * p.nkb + 2 * kvt];
                const float c1 = cq * p.k_scale[(int64_t)bh * p.nkb + 2 * kvt + 1];
                if (kv_valid < C::BN) {
                    // ragged last step: keys at or past N take no part
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        if (i >= kv_valid) ra[i] = static_cast<uint32_t>(INT_MIN);
                        if (32 + i >= kv_valid) rb[i] = static_cast<uint32_t>(INT_MIN);
                        if (64 + i >= kv_valid) rc[i] = static_cast<uint32_t>(INT_MIN);
                        if (96 + i >= kv_valid) rd[i] = static_cast<uint32_t>(INT_MIN);
                    }
                }
                int mx0 = INT_MIN, mx1 = INT_MIN;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    mx0 = max(mx0, max(static_cast<int>(ra[i]), static_cast<int>(rb[i])));
                    mx1 = max(mx1, max(static_cast<int>(rc[i]), static_cast<int>(rd[i])));
                }
                const float x0 = mx0 == INT_MIN ? -INFINITY : static_cast<float>(mx0) * c0;
                const float x1 = mx1 == INT_MIN ? -INFINITY : static_cast<float>(mx1) * c1;
                const float m_new = fmaxf(m, ceilf(fmaxf(x0, x1)));
                const float alpha = (m == -INFINITY) ? 0.f : exp2_int(m - m_new);
                const float nb = kLog2_448 - m_new;
                float sum = 0.f;
                auto emit = [&](const uint32_t (&r)[32], float cc, int col0, uint32_t *dst) {
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        float pv[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int sv = static_cast<int>(r[i + e]);
                            float pe = ex2_approx(fmaf(static_cast<float>(sv), cc, nb));
                            if (col0 + i + e >= kv_valid) pe = 0.f;
                            pv[e] = pe;
                        }
                        sum += (pv[0] + pv[1]) + (pv[2] + pv[3]);
                        dst[i / 4] = cvt_e4m3x2(pv[0], pv[1]) | (cvt_e4m3x2(pv[2], pv[3]) << 16);
                    }
                };
                emit(ra, c0, 0, pk + 0);
                emit(rb, c0, 32, pk + 8);
                emit(rc, c1, 64, pk + 16);
                emit(rd, c1, 96, pk + 24);
                l = l * alpha + sum;
                const bool need = (j > 0) && (m_new > m);
                m = m_new;
                tmem_st_32x32b_x32(tS + 0, pk);
                tmem_wait_st();
                if (__any_sync(0xffffffffu, need)) {
                    // O must hold step j-1's product before it is rescaled
                    if (!(ok = wait_warp(&ctl->o_done[t], (j - 1) & 1, p.err, &ctl->abort))) break;
                    tc_fence_after();
                    const float a = need ? alpha : 1.f;
#pragma unroll 1
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t o[32];
                        tmem_ld_32x32b_x32(tO + cc * 32, o);
                        tmem_wait_ld_x32(o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * a);
                        tmem_st_32x32b_x32(tO + cc * 32, o);
                    }
                    tmem_wait_st();
                }
            }
            if (EXPORT_S) {
                tmem_st_32x32b_x32(tS + 0, pk);
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(&ctl->p_ready[t]);
        }
        if (ok && !EXPORT_S) {
            if (wait_warp(&ctl->o_done[t], (nkv - 1) & 1, p.err, &ctl->abort)) {
                tc_fence_after();
                const float inv_l = 1.f / l;
                uint16_t *orow = p.out + (int64_t)(bh / p.H) * p.osb + (int64_t)(bh % p.H) * p.osh +
                                 (int64_t)row * p.osn;
#pragma unroll 1
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t o[32];
                    tmem_ld_32x32b_x32(tO + cc * 32, o);
                    tmem_wait_ld_x32(o);
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int c = cc * 32 + 2 * i;
                        w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * ctl->v_scale[c] * inv_l,
                                           __uint_as_float(o[2 * i + 1]) * ctl->v_scale[c + 1] * inv_l);
                    }
                    if (row < p.N) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + cc * 32);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                    }
                }
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

template <int D, bool EXPORT_S>
cudaError_t launch_attn_d(const Shape &s, const int8_t *q_i8, const int8_t *k_i8, const uint8_t *v_t8,
                          const AttnParams &p0, dim3 grid, cudaStream_t st) {
    using C = Cfg<D>;
    const int n_pad = s.n_pad();
    CUtensorMap tq, tk, tv;
    cudaError_t e;
    if ((e = make_map(&tq, q_i8, D, n_pad, s.BH(), D, (uint64_t)n_pad * D, D, C::BM)) != cudaSuccess) return e;
    if ((e = make_map(&tk, k_i8, D, n_pad, s.BH(), D, (uint64_t)n_pad * D, D, C::BN)) != cudaSuccess) return e;
    if (EXPORT_S) {
        tv = tk;
    } else if ((e = make_map(&tv, v_t8, n_pad, D, s.BH(), n_pad, (uint64_t)n_pad * D, C::BN, D)) != cudaSuccess) {
        return e;
    }
    AttnParams p = p0;
    p.err = device_error_ptr();
    if (!p.err) return cudaErrorSymbolNotFound;
    const int smem = smem_bytes<D>();
    auto kern = k_attn<D, EXPORT_S>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess) return e;
    kern<<<grid, C::THREADS, smem, st>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const Shape &s, const Codes &c, const Dst &out, float sm_scale, cudaStream_t st) {
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
    dim3 grid((s.n_qblocks() + 1) / 2, s.BH());
    return s.d == 128 ? launch_attn_d<128, false>(s, c.q_i8, c.k_i8, c.v_t8, p, grid, st)
                      : launch_attn_d<64, false>(s, c.q_i8, c.k_i8, c.v_t8, p, grid, st);
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
    return s.d == 128 ? launch_attn_d<128, true>(s, q_i8, k_i8, nullptr, p, dim3(1, 1), st)
                      : launch_attn_d<64, true>(s, q_i8, k_i8, nullptr, p, dim3(1, 1), st);
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
