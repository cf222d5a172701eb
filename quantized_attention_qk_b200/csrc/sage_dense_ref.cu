// sage_dense_ref.cu -- plain dense attention in fp32 on the CUDA cores, for A/B
// checks of the quantized path: out = softmax(Q K^T * sm_scale) V
// ("SDPA稠密注意力模式：大模型推理加速的优化方案", section 三.1 数学基础;
//  "MiniMax H3 接入 SageAttention 实测加速", section 一).
// No quantization and no tensor cores.  A CTA owns 64 query rows of one
// (b,h); keys stream through shared memory 32 at a time with an exact
// running-max softmax (expf), so nothing of size N x N is stored.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sage_internal.h"

namespace sage {
namespace {

constexpr int kRows = 64;
constexpr int kKeys = 32;
constexpr int kThreads = 256;  // 4 threads per query row

__device__ __forceinline__ float bf(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }

template <int D>
__global__ void __launch_bounds__(kThreads) k_dense_ref(Src q, Src k, Src v, Dst out, int H, int N, float sm_scale) {
    extern __shared__ float dyn[];
    float (*sq)[D + 1] = reinterpret_cast<float (*)[D + 1]>(dyn);
    float (*sk)[D + 1] = reinterpret_cast<float (*)[D + 1]>(dyn + kRows * (D + 1));
    float (*sv)[D + 1] = reinterpret_cast<float (*)[D + 1]>(dyn + (kRows + kKeys) * (D + 1));
    float (*sp)[kKeys + 1] = reinterpret_cast<float (*)[kKeys + 1]>(dyn + (kRows + 2 * kKeys) * (D + 1));
    const int bh = blockIdx.y, b = bh / H, h = bh % H;
    const int r0 = blockIdx.x * kRows;
    const int tid = threadIdx.x;
    const int my_row = tid / 4, part = tid % 4;   // 4 threads share a row
    constexpr int CPT = D / 4;                    // output channels per thread

    const uint16_t *qb = q.p + b * q.sb + h * q.sh;
    const uint16_t *kb = k.p + b * k.sb + h * k.sh;
    const uint16_t *vb = v.p + b * v.sb + h * v.sh;
    for (int i = tid; i < kRows * D; i += kThreads) {
        const int r = i / D, c = i % D;
        sq[r][c] = (r0 + r < N) ? bf(qb[(int64_t)(r0 + r) * q.sn + c]) : 0.f;
    }
    float o[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) o[c] = 0.f;
    float m = -INFINITY, l = 0.f;

    for (int j0 = 0; j0 < N; j0 += kKeys) {
        __syncthreads();
        for (int i = tid; i < kKeys * D; i += kThreads) {
            const int r = i / D, c = i % D;
            const bool in = j0 + r < N;
            sk[r][c] = in ? bf(kb[(int64_t)(j0 + r) * k.sn + c]) : 0.f;
            sv[r][c] = in ? bf(vb[(int64_t)(j0 + r) * v.sn + c]) : 0.f;
        }
        __syncthreads();
        // scores of my row against my 8 keys
        float s[kKeys / 4];
        float tmax = -INFINITY;
#pragma unroll
        for (int e = 0; e < kKeys / 4; ++e) {
            const int key = part * (kKeys / 4) + e;
            float acc = 0.f;
            for (int c = 0; c < D; ++c) acc = fmaf(sq[my_row][c], sk[key][c], acc);
            s[e] = (j0 + key < N) ? acc * sm_scale : -INFINITY;
            tmax = fmaxf(tmax, s[e]);
        }
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
        const float m_new = fmaxf(m, tmax);
        const float scale = (m == -INFINITY) ? 0.f : expf(m - m_new);
        float psum = 0.f;
#pragma unroll
        for (int e = 0; e < kKeys / 4; ++e) {
            const float pe = (s[e] == -INFINITY) ? 0.f : expf(s[e] - m_new);
            sp[my_row][part * (kKeys / 4) + e] = pe;
            psum += pe;
        }
        psum += __shfl_xor_sync(0xffffffffu, psum, 1);
        psum += __shfl_xor_sync(0xffffffffu, psum, 2);
        l = l * scale + psum;
        m = m_new;
        __syncwarp();
#pragma unroll
        for (int c = 0; c < CPT; ++c) o[c] *= scale;
        for (int key = 0; key < kKeys; ++key) {
            const float pe = sp[my_row][key];
#pragma unroll
            for (int c = 0; c < CPT; ++c) o[c] = fmaf(pe, sv[key][part * CPT + c], o[c]);
        }
    }
    const int row = r0 + my_row;
    if (row < N) {
        uint16_t *dst = out.p + b * out.sb + h * out.sh + (int64_t)row * out.sn + part * CPT;
        const float inv = 1.f / l;
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            __nv_bfloat16 x = __float2bfloat16_rn(o[c] * inv);
            dst[c] = *reinterpret_cast<uint16_t *>(&x);
        }
    }
}

template <int D>
constexpr int smem_floats() {
    return (kRows + 2 * kKeys) * (D + 1) + kRows * (kKeys + 1);
}

}  // namespace

cudaError_t launch_dense_ref(const Shape &s, const Src &q, const Src &k, const Src &v, const Dst &out,
                             float sm_scale, cudaStream_t st) {
    dim3 grid((s.N + kRows - 1) / kRows, s.BH());
    cudaError_t e;
    if (s.d == 128) {
        const int smem = smem_floats<128>() * 4;
        if ((e = cudaFuncSetAttribute(k_dense_ref<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)))
            return e;
        k_dense_ref<128><<<grid, kThreads, smem, st>>>(q, k, v, out, s.H, s.N, sm_scale);
    } else {
        const int smem = smem_floats<64>() * 4;
        if ((e = cudaFuncSetAttribute(k_dense_ref<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)))
            return e;
        k_dense_ref<64><<<grid, kThreads, smem, st>>>(q, k, v, out, s.H, s.N, sm_scale);
    }
    return cudaGetLastError();
}

}  // namespace sage
