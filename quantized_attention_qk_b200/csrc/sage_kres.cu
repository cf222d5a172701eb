// sage_kres.cu -- K-residual quantization ("ComfyUI-sol-attn", 核心亮点 item 1:
// quantize only the residual of K inside each block and keep the block-mean
// term at bf16 precision).  Readings where the page is silent:
//   * the blocks are the 64-token K blocks; the block mean is the mean of the
//     block's valid tokens (summed exactly in fp64), rounded to bf16 (RNE);
//   * the residual fp32(k) - fp32(mean) is coded like the other INT8 codes
//     (scale amax/127 per block, codes rne(fp32(r * fp32(127/amax))));
//   * the mean term of a score, e[r][b] = (q_r . mean_b) * fp32(sm_scale *
//     log2 e), comes from the bf16 inputs with fp32 accumulation and is added
//     to every score of row r against keys of block b (it varies with the
//     block, so softmax does not cancel it).
// k_kres writes the residual codes, scales and bf16 block means; the
// attention kernel's K-residual instantiation computes e on the tensor cores
// (tcgen05 kind::f16, fp32 accumulation) in its prologue -- an auxiliary
// product of 2 * N * (N/64) * d flops per head, next to the 4 * N^2 * d of the
// attention.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {
namespace {

constexpr int kKresThreads = 256;

template <int D>
__global__ void __launch_bounds__(kKresThreads)
    k_kres(const uint16_t *__restrict__ k, int64_t sb, int64_t sh, int64_t sn, int H, int N, int n_pad, int nkb,
           int8_t *__restrict__ k_i8, float *__restrict__ k_scale, uint16_t *__restrict__ k_bmean) {
    constexpr int CH = D / 8;                  // 16-byte chunks (8 channels) per row
    constexpr int RPP = kKresThreads / CH;     // rows per pass
    constexpr int PASSES = kKBlock / RPP;
    __shared__ double sums[RPP][D];
    __shared__ float mu[D];
    __shared__ float wmax[kKresThreads / 32];
    const int blk = blockIdx.x, bh = blockIdx.y;
    const int chunk = threadIdx.x % CH, rsub = threadIdx.x / CH;
    const int n0 = blk * kKBlock;
    const int nvalid = max(0, min(kKBlock, N - n0));
    const uint16_t *kb = k + (int64_t)(bh / H) * sb + (int64_t)(bh % H) * sh + chunk * 8;
    float x[PASSES][8];
    double part[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) part[e] = 0.0;
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const int row = n0 + rsub + p * RPP;
        if (row < N) {
            unpack8(*reinterpret_cast<const uint4 *>(kb + (int64_t)row * sn), x[p]);
#pragma unroll
            for (int e = 0; e < 8; ++e) part[e] += static_cast<double>(x[p][e]);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) x[p][e] = 0.f;
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) sums[rsub][chunk * 8 + e] = part[e];
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += kKresThreads) {
        double s = 0.0;
        for (int r = 0; r < RPP; ++r) s += sums[r][c];  // bf16 values: the fp64 sum is exact
        const __nv_bfloat16 m = __double2bfloat16(nvalid > 0 ? __ddiv_rn(s, static_cast<double>(nvalid)) : 0.0);
        mu[c] = __bfloat162float(m);
        k_bmean[((size_t)bh * nkb + blk) * D + c] = *reinterpret_cast<const uint16_t *>(&m);
    }
    __syncthreads();
    float amax = 0.f;
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const bool valid = n0 + rsub + p * RPP < N;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            x[p][e] = valid ? __fsub_rn(x[p][e], mu[chunk * 8 + e]) : 0.f;
            amax = fmaxf(amax, fabsf(x[p][e]));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = 0.f;
#pragma unroll
    for (int w = 0; w < kKresThreads / 32; ++w) amax = fmaxf(amax, wmax[w]);
    const float inv = amax > 0.f ? __fdiv_rn(127.f, amax) : 0.f;
    if (threadIdx.x == 0) k_scale[(size_t)bh * nkb + blk] = amax > 0.f ? __fdiv_rn(amax, 127.f) : 0.f;
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const int row = n0 + rsub + p * RPP;  // < n_pad: the grid covers n_pad / 64 blocks
        const uint2 codes = (row < N && amax > 0.f) ? i8x8(x[p], inv) : make_uint2(0u, 0u);
        *reinterpret_cast<uint2 *>(k_i8 + ((size_t)bh * n_pad + row) * D + chunk * 8) = codes;
    }
}

}  // namespace

cudaError_t launch_kres(const Shape &s, const Src &k, int8_t *k_i8, float *k_scale, uint16_t *k_bmean,
                        cudaStream_t st) {
    const dim3 grid(s.n_kblocks(), s.BH());
    if (s.d == 128)
        k_kres<128><<<grid, kKresThreads, 0, st>>>(k.p, k.sb, k.sh, k.sn, s.H, s.N, s.n_pad(), s.n_kblocks(), k_i8,
                                                  k_scale, k_bmean);
    else
        k_kres<64><<<grid, kKresThreads, 0, st>>>(k.p, k.sb, k.sh, k.sn, s.H, s.N, s.n_pad(), s.n_kblocks(), k_i8,
                                                 k_scale, k_bmean);
    return cudaGetLastError();
}

}  // namespace sage
