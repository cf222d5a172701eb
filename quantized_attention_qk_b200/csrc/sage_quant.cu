// sage_quant.cu -- the quantize pass of the quantized attention forward.
//
// Three HBM-bound streaming kernels (no tensor cores: there is no contraction):
//   k_stats_partial  per (b,h, token chunk): sum of K and max |V| per channel
//   k_stats_final    per (b,h): K mean (the smoothing statistic) and 448/amax of V
//   k_quant          per (b,h, 128-token block): Q block -> INT8, (K - mean) per
//                    64-token block -> INT8, V -> e4m3 (token-major, like the codes
//                    of Q and K; the attention kernel reads it as an MN-major operand).
// Pages: "MiniMax H3 接入 SageAttention 实测加速", section 一 (outlier smoothing of
// QK^T, INT8 QK, FP8 PV).  Block sizes, rounding and scale conventions are the
// readings C1-C3 and C7 of the design notes:
//   scale = amax/127 (fp32 IEEE divide), code = rne(x * fp32(127/amax)) in
//   [-127,127]; V: code = e4m3_rn_satfinite(v * fp32(448/amax_c)).
// Loads are 16-byte vectors from arbitrary (b,h,n) strides, so a fused-qkv
// view is read in place; codes are stored as 8-byte vectors.
#include <cuda_runtime.h>

#include "sage_internal.h"

namespace sage {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint4 ld_vec(const uint16_t *p) {
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// bf16 pair packed in a 32-bit word -> two floats (element 2i in the low half).
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
    f[0] = bf_lo(u.x); f[1] = bf_hi(u.x);
    f[2] = bf_lo(u.y); f[3] = bf_hi(u.y);
    f[4] = bf_lo(u.z); f[5] = bf_hi(u.z);
    f[6] = bf_lo(u.w); f[7] = bf_hi(u.w);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Max over the block of two values at once (all threads get the results).
__device__ __forceinline__ void block_max2(float &a, float &b, float *sh /*[2][8]*/) {
    a = warp_max(a);
    b = warp_max(b);
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) { sh[w] = a; sh[8 + w] = b; }
    __syncthreads();
    a = sh[0]; b = sh[8];
#pragma unroll
    for (int i = 1; i < kThreads / 32; ++i) { a = fmaxf(a, sh[i]); b = fmaxf(b, sh[8 + i]); }
    __syncthreads();
}

// Symmetric int8 code: rne(x * inv) clamped to [-127, 127]; the multiply is a
// single IEEE fp32 rounding (no contraction).
__device__ __forceinline__ uint32_t i8code(float x, float inv) {
    float r = rintf(__fmul_rn(x, inv));
    r = fminf(fmaxf(r, -127.f), 127.f);
    return static_cast<uint32_t>(static_cast<int>(r)) & 0xffu;
}

template <int D>
__global__ void __launch_bounds__(kThreads) k_stats_partial(Src k, Src v, int H, int N, int nch, int chunk,
                                                            int do_k, int do_v, float *ksum_part, float *vmax_part) {
    constexpr int VPR = D / 8;             // 16-byte vectors per token row
    constexpr int RPI = kThreads / VPR;    // rows covered per iteration
    __shared__ float red_s[RPI][D];
    __shared__ float red_m[RPI][D];
    const int bh = blockIdx.y, ch = blockIdx.x;
    const int b = bh / H, h = bh % H;
    const int cv = threadIdx.x % VPR, r0 = threadIdx.x / VPR;
    const int n0 = ch * chunk;
    const int n1 = min(N, n0 + chunk);
    float s[8], m[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) { s[e] = 0.f; m[e] = 0.f; }
    const uint16_t *kp = do_k ? k.p + b * k.sb + h * k.sh + cv * 8 : nullptr;
    const uint16_t *vp = do_v ? v.p + b * v.sb + h * v.sh + cv * 8 : nullptr;
    constexpr int U = 4;  // rows in flight per thread and tensor
    for (int n = n0 + r0; n < n1; n += U * RPI) {
        uint4 xk[U], xv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int nn = n + u * RPI;
            xk[u] = (do_k && nn < n1) ? ld_vec(kp + (int64_t)nn * k.sn) : make_uint4(0, 0, 0, 0);
            xv[u] = (do_v && nn < n1) ? ld_vec(vp + (int64_t)nn * v.sn) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float f[8];
            unpack8(xk[u], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) s[e] += f[e];
            unpack8(xv[u], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(f[e]));
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) { red_s[r0][cv * 8 + e] = s[e]; red_m[r0][cv * 8 + e] = m[e]; }
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += kThreads) {
        float ss = 0.f, mm = 0.f;
        for (int r = 0; r < RPI; ++r) { ss += red_s[r][c]; mm = fmaxf(mm, red_m[r][c]); }
        const int64_t o = ((int64_t)bh * nch + ch) * D + c;
        if (do_k) ksum_part[o] = ss;
        if (do_v) vmax_part[o] = mm;
    }
}

template <int D>
__global__ void k_stats_final(int N, int nch, int do_k, int do_v, const float *ksum_part, const float *vmax_part,
                              float *k_mean, float *user_k_mean, float *v_inv, float *v_scale) {
    const int bh = blockIdx.x, c = threadIdx.x;
    if (c >= D) return;
    float s = 0.f, m = 0.f;
    for (int ch = 0; ch < nch; ++ch) {
        const int64_t o = ((int64_t)bh * nch + ch) * D + c;
        if (do_k) s += ksum_part[o];
        if (do_v) m = fmaxf(m, vmax_part[o]);
    }
    if (do_k) {
        const float mu = s / static_cast<float>(N);
        k_mean[bh * D + c] = mu;
        if (user_k_mean) user_k_mean[bh * D + c] = mu;
    }
    if (do_v) {
        v_inv[bh * D + c] = m > 0.f ? 448.f / m : 0.f;
        v_scale[bh * D + c] = m > 0.f ? m / 448.f : 0.f;
    }
}

template <int D, bool DO_Q, bool DO_K, bool DO_V>
__global__ void __launch_bounds__(kThreads) k_quant(Src q, Src k, Src v, int H, int N, int n_pad,
                                                    const float *__restrict__ k_mean,
                                                    const float *__restrict__ v_inv, Codes c) {
    constexpr int VPR = D / 8;
    constexpr int RPI = kThreads / VPR;
    constexpr int NI = kQBlock / RPI;    // vectors per thread in one 128-token block
    __shared__ float red[16];
    const int blk = blockIdx.x, bh = blockIdx.y;
    const int b = bh / H, h = bh % H;
    const int cv = threadIdx.x % VPR, r0 = threadIdx.x / VPR;
    const int row0 = blk * kQBlock;
    const int nqb = n_pad / kQBlock, nkb = n_pad / kKBlock;

    if (DO_Q) {
        const uint16_t *qp = q.p + b * q.sb + h * q.sh + cv * 8;
        uint4 x[NI];
        float amax = 0.f, dummy = 0.f;
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            const int n = row0 + r0 + i * RPI;
            x[i] = n < N ? ld_vec(qp + (int64_t)n * q.sn) : make_uint4(0, 0, 0, 0);
            float f[8];
            unpack8(x[i], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
        }
        block_max2(amax, dummy, red);
        const float inv = amax > 0.f ? 127.f / amax : 0.f;
        int8_t *dst = c.q_i8 + ((int64_t)bh * n_pad + row0) * D + cv * 8;
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            float f[8];
            unpack8(x[i], f);
            uint2 w;
            w.x = i8code(f[0], inv) | (i8code(f[1], inv) << 8) | (i8code(f[2], inv) << 16) | (i8code(f[3], inv) << 24);
            w.y = i8code(f[4], inv) | (i8code(f[5], inv) << 8) | (i8code(f[6], inv) << 16) | (i8code(f[7], inv) << 24);
            *reinterpret_cast<uint2 *>(dst + (int64_t)(r0 + i * RPI) * D) = w;
        }
        if (threadIdx.x == 0) c.q_scale[(int64_t)bh * nqb + blk] = amax > 0.f ? amax / 127.f : 0.f;
    }

    if (DO_K) {
        const uint16_t *kp = k.p + b * k.sb + h * k.sh + cv * 8;
        float mu[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mu[e] = k_mean[bh * D + cv * 8 + e];
        float ks[NI][8];
        float a0 = 0.f, a1 = 0.f;  // amax of the two 64-token blocks
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            const int n = row0 + r0 + i * RPI;
            if (n < N) {
                float f[8];
                unpack8(ld_vec(kp + (int64_t)n * k.sn), f);
#pragma unroll
                for (int e = 0; e < 8; ++e) ks[i][e] = __fsub_rn(f[e], mu[e]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) ks[i][e] = 0.f;
            }
            float am = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) am = fmaxf(am, fabsf(ks[i][e]));
            if (i < NI / 2) a0 = fmaxf(a0, am); else a1 = fmaxf(a1, am);
        }
        block_max2(a0, a1, red);
        const float inv0 = a0 > 0.f ? 127.f / a0 : 0.f;
        const float inv1 = a1 > 0.f ? 127.f / a1 : 0.f;
        int8_t *dst = c.k_i8 + ((int64_t)bh * n_pad + row0) * D + cv * 8;
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            const float inv = i < NI / 2 ? inv0 : inv1;
            uint2 w;
            w.x = i8code(ks[i][0], inv) | (i8code(ks[i][1], inv) << 8) | (i8code(ks[i][2], inv) << 16) |
                  (i8code(ks[i][3], inv) << 24);
            w.y = i8code(ks[i][4], inv) | (i8code(ks[i][5], inv) << 8) | (i8code(ks[i][6], inv) << 16) |
                  (i8code(ks[i][7], inv) << 24);
            *reinterpret_cast<uint2 *>(dst + (int64_t)(r0 + i * RPI) * D) = w;
        }
        if (threadIdx.x == 0) {
            c.k_scale[(int64_t)bh * nkb + 2 * blk] = a0 > 0.f ? a0 / 127.f : 0.f;
            c.k_scale[(int64_t)bh * nkb + 2 * blk + 1] = a1 > 0.f ? a1 / 127.f : 0.f;
        }
    }

    if (DO_V) {
        const uint16_t *vp = v.p + b * v.sb + h * v.sh + cv * 8;
        float inv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) inv[e] = v_inv[bh * D + cv * 8 + e];
        uint4 x[NI];
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            const int n = row0 + r0 + i * RPI;
            x[i] = n < N ? ld_vec(vp + (int64_t)n * v.sn) : make_uint4(0, 0, 0, 0);
        }
        uint8_t *dst = c.v_e4m3 + ((int64_t)bh * n_pad + row0) * D + cv * 8;
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            float f[8];
            unpack8(x[i], f);
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                uint16_t pr;
                // cvt packs its first source in the high byte: (hi=e+1, lo=e)
                asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
                    : "=h"(pr)
                    : "f"(__fmul_rn(f[e + 1], inv[e + 1])), "f"(__fmul_rn(f[e], inv[e])));
                w[e / 2] = pr;
            }
            uint2 o;
            o.x = w[0] | (w[1] << 16);
            o.y = w[2] | (w[3] << 16);
            *reinterpret_cast<uint2 *>(dst + (int64_t)(r0 + i * RPI) * D) = o;
        }
    }
}

template <int D>
cudaError_t launch_stats_d(const Shape &s, const Src *k, const Src *v, const StatsWs &ws, float *user_k_mean,
                           float *v_scale, cudaStream_t st) {
    const int nch = s.n_chunks();
    Src z{nullptr, 0, 0, 0};
    dim3 g1(nch, s.BH());
    k_stats_partial<D><<<g1, kThreads, 0, st>>>(k ? *k : z, v ? *v : z, s.H, s.N, nch, s.chunk_rows(),
                                                k != nullptr, v != nullptr, ws.ksum_part, ws.vmax_part);
    k_stats_final<D><<<s.BH(), D, 0, st>>>(s.N, nch, k != nullptr, v != nullptr, ws.ksum_part, ws.vmax_part,
                                          ws.k_mean, user_k_mean, ws.v_inv, v_scale);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_quant_d(const Shape &s, const Src *q, const Src *k, const Src *v, const StatsWs &ws,
                           const Codes &c, cudaStream_t st) {
    Src z{nullptr, 0, 0, 0};
    dim3 g(s.n_qblocks(), s.BH());
    const Src qq = q ? *q : z, kk = k ? *k : z, vv = v ? *v : z;
    if (q && k && v)
        k_quant<D, true, true, true><<<g, kThreads, 0, st>>>(qq, kk, vv, s.H, s.N, s.n_pad(), ws.k_mean, ws.v_inv, c);
    else if (q && k && !v)
        k_quant<D, true, true, false><<<g, kThreads, 0, st>>>(qq, kk, vv, s.H, s.N, s.n_pad(), ws.k_mean, ws.v_inv, c);
    else if (!q && !k && v)
        k_quant<D, false, false, true><<<g, kThreads, 0, st>>>(qq, kk, vv, s.H, s.N, s.n_pad(), ws.k_mean, ws.v_inv, c);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_stats(const Shape &s, const Src *k, const Src *v, const StatsWs &ws, float *user_k_mean,
                         float *v_scale, cudaStream_t st) {
    return s.d == 128 ? launch_stats_d<128>(s, k, v, ws, user_k_mean, v_scale, st)
                      : launch_stats_d<64>(s, k, v, ws, user_k_mean, v_scale, st);
}

cudaError_t launch_quant(const Shape &s, const Src *q, const Src *k, const Src *v, const StatsWs &ws,
                         const Codes &c, cudaStream_t st) {
    return s.d == 128 ? launch_quant_d<128>(s, q, k, v, ws, c, st) : launch_quant_d<64>(s, q, k, v, ws, c, st);
}

}  // namespace sage
