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
// k_kres writes the residual codes, scales and bf16 block means; k_ebias
// computes e for every (query row, K block) with bf16 tensor-core products
// (mma.sync m16n8k16, fp32 accumulation) -- an auxiliary product of
// 2 * N * (N/64) * d flops per head, next to the 4 * N^2 * d of the attention.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sage_device.cuh"
#include "sage_internal.h"

namespace sage {
namespace {

constexpr int kKresThreads = 256;
constexpr int kEbTile = 64;          // k_ebias: 64 query rows x 64 K blocks per CTA
constexpr int kEbThreads = 256;

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

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// e[bh][b][r] = fp32(sum_c q[r][c] * mean_b[c]) * s_l2 for query rows r < n_pad
// (rows at or past N read as 0) and K blocks b < nkb.  Both operands are
// K-major (channels contiguous), the A = Q tile row-major and B = the block
// means' tile "col" for the m16n8k16 product; shared rows are padded by 16
// bytes so that ldmatrix reads are conflict-free.  Warp w covers rows
// 32 (w % 2) .. +32 and blocks 16 (w / 2) .. +16 of the CTA's 64 x 64 tile.
template <int D>
__global__ void __launch_bounds__(kEbThreads)
    k_ebias(const uint16_t *__restrict__ q, int64_t sb, int64_t sh, int64_t sn, int H, int N, int n_pad, int nkb,
            const uint16_t *__restrict__ k_bmean, float s_l2, float *__restrict__ ebias) {
    constexpr int LD = D + 8;  // bf16 elements per shared row
    __shared__ __align__(16) uint16_t sq[kEbTile * LD];
    __shared__ __align__(16) uint16_t sm[kEbTile * LD];
    const int r0 = blockIdx.x * kEbTile, b0 = blockIdx.y * kEbTile, bh = blockIdx.z;
    const uint16_t *qb = q + (int64_t)(bh / H) * sb + (int64_t)(bh % H) * sh;
    constexpr int CH = D / 8;
    for (int x = threadIdx.x; x < kEbTile * CH; x += kEbThreads) {
        const int r = x / CH, c = (x - r * CH) * 8;
        const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4 *>(sq + r * LD + c) =
            r0 + r < N ? *reinterpret_cast<const uint4 *>(qb + (int64_t)(r0 + r) * sn + c) : zero;
        *reinterpret_cast<uint4 *>(sm + r * LD + c) =
            b0 + r < nkb ? *reinterpret_cast<const uint4 *>(k_bmean + ((size_t)bh * nkb + b0 + r) * D + c) : zero;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wr = (warp & 1) * 32, wb = (warp >> 1) * 16;
    float acc[2][2][4] = {};
    const uint32_t sq_base = smem_u32(sq), sm_base = smem_u32(sm);
#pragma unroll
    for (int k0 = 0; k0 < D; k0 += 16) {
        uint32_t a[2][4], b[2][2];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            const int row = wr + mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int col = k0 + (lane >> 4) * 8;
            ldsm_x4(sq_base + (row * LD + col) * 2, a[mt][0], a[mt][1], a[mt][2], a[mt][3]);
        }
        {
            const int row = wb + (lane & 7) + (lane >> 4) * 8;
            const int col = k0 + ((lane >> 3) & 1) * 8;
            ldsm_x4(sm_base + (row * LD + col) * 2, b[0][0], b[0][1], b[1][0], b[1][1]);
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) mma_bf16_16816(acc[mt][nt], a[mt], b[nt][0], b[nt][1]);
    }
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = r0 + wr + mt * 16 + g + (e >> 1) * 8;
                const int b = b0 + wb + nt * 8 + t4 * 2 + (e & 1);
                if (r < n_pad && b < nkb) ebias[((size_t)bh * nkb + b) * n_pad + r] = acc[mt][nt][e] * s_l2;
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

cudaError_t launch_ebias(const Shape &s, const Src &q, const uint16_t *k_bmean, float sm_scale, float *ebias,
                         cudaStream_t st) {
    const int nkb = s.n_kblocks();
    const dim3 grid(s.n_pad() / kEbTile, (nkb + kEbTile - 1) / kEbTile, s.BH());
    const float s_l2 = sm_scale * static_cast<float>(1.4426950408889634);
    if (s.d == 128)
        k_ebias<128><<<grid, kEbThreads, 0, st>>>(q.p, q.sb, q.sh, q.sn, s.H, s.N, s.n_pad(), nkb, k_bmean, s_l2,
                                                 ebias);
    else
        k_ebias<64><<<grid, kEbThreads, 0, st>>>(q.p, q.sb, q.sh, q.sn, s.H, s.N, s.n_pad(), nkb, k_bmean, s_l2,
                                                ebias);
    return cudaGetLastError();
}

}  // namespace sage
