// sage_sparse.cu -- block-sparse skipping: tile-pair scores and the tau
// selection of key tiles ("ComfyUI-sol-attn", 核心亮点 item 4: a sparsity value
// tau that may ramp over the sampling steps, sparse early and dense late).
// The page names only the control; the steps are this library's readings:
//   S1  queries and keys are cut into tiles of 128 tokens (the Q quantization
//       block and the attention kernel's key step);
//   S2  the score of (query tile i, key tile j) is the mean dequantized score
//       of the tile pair in log2 units, (sum q).(sum k) * s_l2 / (n_i n_j),
//       evaluated in fp32 in a fixed order from exact integer code sums;
//   S3  query tile i keeps the shortest prefix of its key tiles ranked by
//       score (ties: lower index first) whose estimated mass
//       n_j 2^(score - max score) reaches tau of the total (tau >= 1: all),
//       in fp32 with one rounding per operation in a fixed order (masses by
//       a fixed Taylor polynomial, sums in rank order), so that the kept set
//       is reproducible bit for bit;
//   S4  tau(step) moves linearly from tau_start to tau_end over the steps.
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <type_traits>

#include "sage.h"
#include "sage_internal.h"

namespace sage {
namespace {

constexpr int kPoolThreads = 256;  // 8 warps, each over every 8th row of a tile
constexpr int kScoreTile = 16;     // k_score: 16 query tiles x 16 key tiles per CTA
constexpr int kScoreThreads = 256; // one (query tile, key tile) pair per thread
constexpr int kSelThreads = 256;

// Per (b,h, tile i): qv[i][c] = q_scale[i] * float(sum of the tile's Q codes
// in channel c); kvT[c][i] = k_scale[2i] * float(sum over K block 2i) +
// k_scale[2i+1] * float(sum over K block 2i+1), channel-major so that the
// scoring kernel reads it coalesced.  Rows at or past N take no part.  All 16
// rows of a warp are loaded before any is summed (the loads overlap).
template <int D>
__global__ void __launch_bounds__(kPoolThreads)
    k_pool(const int8_t *__restrict__ q_i8, const float *__restrict__ q_scale, const int8_t *__restrict__ k_i8,
           const float *__restrict__ k_scale, int N, int n_pad, int nqb, int nkb, int nt, float *__restrict__ qv,
           float *__restrict__ kvT) {
    constexpr int CPL = D / 32;                   // channels per lane
    constexpr int RPW = kKvTile / (kPoolThreads / 32);  // rows per warp (16)
    using Vec = typename std::conditional<CPL == 4, uint32_t, uint16_t>::type;
    __shared__ int red[3][kPoolThreads / 32][D];
    const int i = blockIdx.x, bh = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = i * kKvTile;
    const size_t base = ((size_t)bh * n_pad + r0) * D + lane * CPL;
    Vec qw[RPW], kw[RPW];
#pragma unroll
    for (int x = 0; x < RPW; ++x) {
        const int r = warp + x * (kPoolThreads / 32);
        const bool in = r0 + r < N;
        qw[x] = in ? *reinterpret_cast<const Vec *>(q_i8 + base + (size_t)r * D) : Vec(0);
        kw[x] = in ? *reinterpret_cast<const Vec *>(k_i8 + base + (size_t)r * D) : Vec(0);
    }
    int aq[CPL], a0[CPL], a1[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) aq[c] = a0[c] = a1[c] = 0;
#pragma unroll
    for (int x = 0; x < RPW; ++x) {
        const int r = warp + x * (kPoolThreads / 32);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            const int qb = static_cast<int8_t>((qw[x] >> (8 * c)) & 0xff);
            const int kb = static_cast<int8_t>((kw[x] >> (8 * c)) & 0xff);
            aq[c] += qb;
            if (r < kKBlock) a0[c] += kb;
            else a1[c] += kb;
        }
    }
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        red[0][warp][lane * CPL + c] = aq[c];
        red[1][warp][lane * CPL + c] = a0[c];
        red[2][warp][lane * CPL + c] = a1[c];
    }
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += kPoolThreads) {
        int sq = 0, s0 = 0, s1 = 0;
        for (int w = 0; w < kPoolThreads / 32; ++w) sq += red[0][w][c], s0 += red[1][w][c], s1 += red[2][w][c];
        qv[((size_t)bh * nt + i) * D + c] = __fmul_rn(q_scale[(size_t)bh * nqb + i], static_cast<float>(sq));
        const float k0 = __fmul_rn(k_scale[(size_t)bh * nkb + 2 * i], static_cast<float>(s0));
        // the second K block of the tile exists only if it holds a token
        const float k1 = (2 * i + 1) * kKBlock < N
                             ? __fmul_rn(k_scale[(size_t)bh * nkb + 2 * i + 1], static_cast<float>(s1))
                             : 0.f;
        kvT[((size_t)bh * D + c) * nt + i] = __fadd_rn(k0, k1);
    }
}

// Tile-pair scores (reading S2) for a 16 x 16 block of (query tile, key tile)
// pairs of one (b,h): both pooled operands staged in shared memory, each dot
// product accumulated over the channels in ascending order, one fp32 rounding
// per multiply and per add (no contraction), then * s_l2 / (n_i n_j).
template <int D>
__global__ void __launch_bounds__(kScoreThreads)
    k_score(const float *__restrict__ qv, const float *__restrict__ kvT, int N, int nt, float s_l2,
            float *__restrict__ sbar) {
    __shared__ float sq[kScoreTile][D + 1];   // [query tile][channel]
    __shared__ float sk[D][kScoreTile];       // [channel][key tile]
    const int i0 = blockIdx.x * kScoreTile, j0 = blockIdx.y * kScoreTile, bh = blockIdx.z;
    static_assert(kScoreTile * D % kScoreThreads == 0, "staging loop has a fixed trip count");
#pragma unroll
    for (int x = threadIdx.x; x < kScoreTile * D; x += kScoreThreads) {  // all loads in flight at once
        const int r = x / D, c = x - r * D;
        sq[r][c] = i0 + r < nt ? qv[((size_t)bh * nt + i0 + r) * D + c] : 0.f;
        const int cc = x / kScoreTile, jj = x - cc * kScoreTile;
        sk[cc][jj] = j0 + jj < nt ? kvT[((size_t)bh * D + cc) * nt + j0 + jj] : 0.f;
    }
    __syncthreads();
    const int il = threadIdx.x / kScoreTile, jl = threadIdx.x % kScoreTile;
    float acc = 0.f;
#pragma unroll 16
    for (int c = 0; c < D; ++c) acc = __fadd_rn(acc, __fmul_rn(sq[il][c], sk[c][jl]));
    const int i = i0 + il, j = j0 + jl;
    if (i >= nt || j >= nt) return;
    const int ni = min(kKvTile, N - i * kKvTile), nj = min(kKvTile, N - j * kKvTile);
    sbar[((size_t)bh * nt + i) * nt + j] = __fdiv_rn(__fmul_rn(acc, s_l2), static_cast<float>(ni * nj));
}

// 2^x for x <= 0 as reading S3 fixes it: 0 below -64; else k = floor(x),
// f = x - k, the degree-8 Taylor polynomial of 2^f = e^(f ln 2) by Horner with
// the coefficients (ln 2)^i / i! rounded to fp32 (each multiply and add rounded
// on its own), times 2^k (exact: the result stays a normal number).
__device__ __forceinline__ float s3_exp2(float x) {
    if (!(x >= -64.f)) return 0.f;
    const float c[9] = {0x1p+0f,          0x1.62e43p-1f,    0x1.ebfbep-3f,  0x1.c6b08ep-5f, 0x1.3b2ab6p-7f,
                        0x1.5d87fep-10f,  0x1.430912p-13f,  0x1.ffcbfcp-17f, 0x1.62c022p-20f};
    const float k = floorf(x);
    const float f = __fsub_rn(x, k);
    float p = c[8];
#pragma unroll
    for (int i = 7; i >= 0; --i) p = __fadd_rn(__fmul_rn(p, f), c[i]);
    return __fmul_rn(p, __int_as_float((127 + static_cast<int>(k)) << 23));
}

// One CTA per (b,h, query tile i): ranks the row's key tiles (bitonic sort of
// P >= nt entries in shared memory: higher score first, then lower index),
// computes their masses n_j 2^(score - top) in parallel, then one thread takes
// the total and the kept prefix in rank order (reading S3's fixed fp32
// order: rank t is kept while the mass ranked before it is below tau of the
// total).  Writes the row's mask words.
__global__ void __launch_bounds__(kSelThreads)
    k_select(const float *__restrict__ sbar, int N, int nt, int P, int words, float tau, uint32_t *__restrict__ mask) {
    extern __shared__ float sm[];
    float *key = sm;                                       // [P] score, then mass
    int *idx = reinterpret_cast<int *>(key + P);           // [P] key tile
    uint32_t *mw = reinterpret_cast<uint32_t *>(idx + P);  // [words]
    __shared__ int s_cut;
    const int i = blockIdx.x, bh = blockIdx.y;
    const float *row = sbar + ((size_t)bh * nt + i) * nt;
    for (int w = threadIdx.x; w < words; w += kSelThreads) mw[w] = 0u;
    for (int j = threadIdx.x; j < P; j += kSelThreads) {
        key[j] = j < nt ? row[j] : -INFINITY;  // padding ranks last
        idx[j] = j;
    }
    __syncthreads();
    if (tau >= 1.f) {
        for (int j = threadIdx.x; j < nt; j += kSelThreads) atomicOr(&mw[j >> 5], 1u << (j & 31));
    } else {
        for (int k = 2; k <= P; k <<= 1) {
            for (int h = k >> 1; h > 0; h >>= 1) {
                for (int x = threadIdx.x; x < P; x += kSelThreads) {
                    const int y = x ^ h;
                    if (y > x) {
                        const float kx = key[x], ky = key[y];
                        const int ix = idx[x], iy = idx[y];
                        const bool y_first = ky > kx || (ky == kx && iy < ix);
                        if (y_first == ((x & k) == 0)) {
                            key[x] = ky, key[y] = kx;
                            idx[x] = iy, idx[y] = ix;
                        }
                    }
                }
                __syncthreads();
            }
        }
        const float top = key[0];
        __syncthreads();
        for (int r = threadIdx.x; r < nt; r += kSelThreads) {
            const int j = idx[r];
            key[r] = __fmul_rn(static_cast<float>(min(kKvTile, N - j * kKvTile)), s3_exp2(__fsub_rn(key[r], top)));
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            float total = 0.f;
#pragma unroll 8
            for (int r = 0; r < nt; ++r) total = __fadd_rn(total, key[r]);
            const float lim = __fmul_rn(tau, total);
            float before = 0.f;
            int cut = 0;
            while (cut < nt && before < lim) before = __fadd_rn(before, key[cut++]);
            s_cut = cut;
        }
        __syncthreads();
        for (int r = threadIdx.x; r < s_cut; r += kSelThreads) atomicOr(&mw[idx[r] >> 5], 1u << (idx[r] & 31));
    }
    __syncthreads();
    for (int w = threadIdx.x; w < words; w += kSelThreads) mask[((size_t)bh * nt + i) * words + w] = mw[w];
}

int pow2_at_least(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

constexpr size_t kAlign = 1024;
size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

}  // namespace

size_t select_ws_bytes(const Shape &s) {
    return 2 * up((size_t)s.BH() * s.n_tiles() * s.d * sizeof(float)) +
           up((size_t)s.BH() * s.n_tiles() * s.n_tiles() * sizeof(float));
}

size_t mask_bytes(const Shape &s) { return (size_t)s.BH() * s.n_tiles() * s.mask_words() * sizeof(uint32_t); }

void select_pool_ptrs(void *ws, const Shape &s, float **qv, float **kvT) {
    char *w = static_cast<char *>(ws);
    const size_t vec = up((size_t)s.BH() * s.n_tiles() * s.d * sizeof(float));
    *qv = reinterpret_cast<float *>(w);
    *kvT = reinterpret_cast<float *>(w + vec);
}

cudaError_t launch_select(const Shape &s, const int8_t *q_i8, const float *q_scale, const int8_t *k_i8,
                          const float *k_scale, float sm_scale, float tau, void *ws, uint32_t *mask, float *sbar_out,
                          cudaStream_t st, bool pooled) {
    const int nt = s.n_tiles();
    if (nt > kMaxSelectTiles) return cudaErrorInvalidValue;
    char *w = static_cast<char *>(ws);
    const size_t vec = up((size_t)s.BH() * nt * s.d * sizeof(float));
    float *qv = nullptr, *kvT = nullptr;
    select_pool_ptrs(ws, s, &qv, &kvT);
    float *sbar = sbar_out ? sbar_out : reinterpret_cast<float *>(w + 2 * vec);
    const float s_l2 = sm_scale * static_cast<float>(1.4426950408889634);
    const int P = pow2_at_least(nt), words = s.mask_words();
    const dim3 g1(nt, s.BH()), g2((nt + kScoreTile - 1) / kScoreTile, (nt + kScoreTile - 1) / kScoreTile, s.BH());
    const size_t smem = (size_t)(2 * P + words) * 4;
    if (s.d == 128) {
        if (!pooled)
            k_pool<128><<<g1, kPoolThreads, 0, st>>>(q_i8, q_scale, k_i8, k_scale, s.N, s.n_pad(), s.n_qblocks(),
                                                     s.n_kblocks(), nt, qv, kvT);
        k_score<128><<<g2, kScoreThreads, 0, st>>>(qv, kvT, s.N, nt, s_l2, sbar);
    } else {
        if (!pooled)
            k_pool<64><<<g1, kPoolThreads, 0, st>>>(q_i8, q_scale, k_i8, k_scale, s.N, s.n_pad(), s.n_qblocks(),
                                                    s.n_kblocks(), nt, qv, kvT);
        k_score<64><<<g2, kScoreThreads, 0, st>>>(qv, kvT, s.N, nt, s_l2, sbar);
    }
    k_select<<<g1, kSelThreads, smem, st>>>(sbar, s.N, nt, P, words, tau, mask);
    return cudaGetLastError();
}

}  // namespace sage

extern "C" float sage_tau_schedule(int step, int n_steps, float tau_start, float tau_end) {
    if (n_steps <= 1) return tau_end;
    const int s = step < 0 ? 0 : (step > n_steps - 1 ? n_steps - 1 : step);
    const double t = static_cast<double>(s) / static_cast<double>(n_steps - 1);
    return static_cast<float>(static_cast<double>(tau_start) +
                              (static_cast<double>(tau_end) - static_cast<double>(tau_start)) * t);
}
