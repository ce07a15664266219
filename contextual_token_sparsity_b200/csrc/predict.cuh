// predict.cuh - predicted token-block scores from low-rank ReLU predictors
// (step a8; Jenga summary section 4.2.2, Eq. 3 and the overhead analysis).
//
//   xbar_g   = mean of the rows of token block g of X                  (pool)
//   Qhat     = relu(xbar W1q) W2q,  Khat = relu(xbar W1k) W2k           (GEMMs)
//   P[n][m]  = (1/H) sum_h max(Qhat_n^h . Khat_m^h, 0),  n >= m          (block products)
//   score[m] = sum_{n >= m} P[n][m]                                      (column sum)
//
// Everything is fp32 on the CUDA cores: the predictor does O(s h^2) work on
// one representative per block plus O(s^2 / b^2) block products (a few
// GFLOP at 32K tokens), far below what would pay for tensor-core tiles, and
// fp32 keeps the predicted scores within 1e-5 of an exact evaluation.
// Split-K partial sums are reduced in a fixed order: results are the same
// bits on every run.
#pragma once

#include "common.cuh"

namespace lemo {
namespace predict {

__device__ __forceinline__ float bf16f(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }

// ---------------------------------------------------------------------------
// Block means of X (fp32).  CTA (g, c): token block g, columns [c*2048, +2048);
// each thread owns 8 consecutive columns (one 16-byte load per row).
// ---------------------------------------------------------------------------
constexpr int kPoolThreads = 256;
constexpr int kPoolCols = kPoolThreads * 8;

__global__ void __launch_bounds__(kPoolThreads)
    pool_kernel(const uint16_t* __restrict__ x, int64_t ld_x, int d, const int32_t* __restrict__ cu,
                int batch, int block, const char* __restrict__ ws, WsLayout lay,
                float* __restrict__ xbar) {
    const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(ws + lay.hdr);
    if (!hdr->valid) return;
    const int32_t* blk_prefix = reinterpret_cast<const int32_t*>(ws + lay.blk_prefix);
    const int g = blockIdx.x;
    if (g >= hdr->total_blocks) return;
    const int s = last_le(blk_prefix, batch + 1, g);
    const int m = g - blk_prefix[s];
    const int64_t r0 = (int64_t)cu[s] + (int64_t)m * block;
    const int64_t r1 = min((int64_t)cu[s + 1], r0 + block);
    const int c = blockIdx.y * kPoolCols + threadIdx.x * 8;
    if (c >= d) return;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int64_t r = r0; r < r1; ++r) {
        const uint4 v = *reinterpret_cast<const uint4*>(x + r * ld_x + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc[2 * i] += __uint_as_float(w[i] << 16);
            acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    const float inv = 1.f / (float)(r1 - r0);
    float4* out = reinterpret_cast<float4*>(xbar + (int64_t)g * d + c);
    out[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    out[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
}

// ---------------------------------------------------------------------------
// C_part[z] = A[:, kz] * B[kz, :] for the K slice kz of split z.
// A fp32 [M, K] row-major (lda), B bf16 [K, N] row-major (ldb).  64 x 64
// output tile per CTA, 256 threads x (4 x 4) outputs, K steps of 16 staged
// in shared memory.  M = number of token blocks is read on the device.
// ---------------------------------------------------------------------------
constexpr int GT = 64, GK = 16;

__global__ void __launch_bounds__(256)
    gemm_kernel(const float* __restrict__ A, int lda, const uint16_t* __restrict__ B, int ldb,
                float* __restrict__ Cpart, const PlanHeader* __restrict__ hdr, int N, int K,
                int kchunk) {
    const int M = hdr->total_blocks;
    const int m0 = blockIdx.y * GT, n0 = blockIdx.x * GT;
    if (!hdr->valid || m0 >= M) return;
    __shared__ float As[GK][GT + 4];
    __shared__ float Bs[GK][GT];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int kb = blockIdx.z * kchunk, ke = min(K, kb + kchunk);
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int k = kb; k < ke; k += GK) {
        for (int i = threadIdx.x; i < GT * GK; i += 256) {
            const int mm = i / GK, kk = i % GK;
            As[kk][mm] = (m0 + mm < M && k + kk < ke) ? A[(int64_t)(m0 + mm) * lda + k + kk] : 0.f;
        }
        for (int i = threadIdx.x; i < GT * GK; i += 256) {
            const int kk = i / GT, nn = i % GT;
            Bs[kk][nn] = (k + kk < ke && n0 + nn < N) ? bf16f(B[(int64_t)(k + kk) * ldb + n0 + nn]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < GK; ++kk) {
            float av[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
    float* C = Cpart + (int64_t)blockIdx.z * M * N;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int mm = m0 + ty * 4 + i;
        if (mm >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int nn = n0 + tx * 4 + j;
            if (nn < N) C[(int64_t)mm * N + nn] = acc[i][j];
        }
    }
}

// C[m][n] = act(sum_z Cpart[z][m][n]), z in increasing order (deterministic).
__global__ void __launch_bounds__(256)
    reduce_kernel(const float* __restrict__ Cpart, int splits, const PlanHeader* __restrict__ hdr,
                  int N, bool relu, float* __restrict__ C) {
    if (!hdr->valid) return;
    const int64_t total = (int64_t)hdr->total_blocks * N;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        float v = 0.f;
        for (int z = 0; z < splits; ++z) v += Cpart[(int64_t)z * total + i];
        C[i] = relu ? fmaxf(v, 0.f) : v;
    }
}

// ---------------------------------------------------------------------------
// Block products: P[n][m] = (1/H) sum_h max(Qhat_n^h . Khat_m^h, 0) for the
// 16 x 16 global block pairs of one CTA; pairs in different sequences or with
// n < m are skipped.  Qhat, Khat fp32 [TB, H*dh].  P uses the per-sequence
// [N_b, N_b] layout of the block-score matrices.
// ---------------------------------------------------------------------------
constexpr int PT = 16;

__global__ void __launch_bounds__(PT * PT)
    products_kernel(const float* __restrict__ qh, const float* __restrict__ kh, int H, int dh,
                    int batch, const char* __restrict__ ws, WsLayout lay, float inv_h,
                    float* __restrict__ P) {
    const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(ws + lay.hdr);
    if (!hdr->valid) return;
    const int32_t* blk_prefix = reinterpret_cast<const int32_t*>(ws + lay.blk_prefix);
    const int64_t* m_prefix = reinterpret_cast<const int64_t*>(ws + lay.m_prefix);
    const int TB = hdr->total_blocks;
    const int n0 = blockIdx.y * PT, mb0 = blockIdx.x * PT;
    if (n0 >= TB || mb0 >= TB || mb0 > n0 + PT - 1) return;  // tile strictly above the diagonal
    extern __shared__ float sh[];
    float* qs = sh;            // [PT][dh + 1]
    float* ks = sh + PT * (dh + 1);
    const int tn = threadIdx.x / PT, tm = threadIdx.x % PT;
    const int n = n0 + tn, m = mb0 + tm;
    const int HD = H * dh;
    float acc = 0.f;
    for (int h = 0; h < H; ++h) {
        for (int i = threadIdx.x; i < PT * dh; i += PT * PT) {
            const int r = i / dh, c = i % dh;
            qs[r * (dh + 1) + c] = (n0 + r < TB) ? qh[(int64_t)(n0 + r) * HD + h * dh + c] : 0.f;
            ks[r * (dh + 1) + c] = (mb0 + r < TB) ? kh[(int64_t)(mb0 + r) * HD + h * dh + c] : 0.f;
        }
        __syncthreads();
        float dot = 0.f;
        for (int c = 0; c < dh; ++c) dot = fmaf(qs[tn * (dh + 1) + c], ks[tm * (dh + 1) + c], dot);
        acc += fmaxf(dot, 0.f);
        __syncthreads();
    }
    if (n >= TB || m >= TB) return;
    const int s = last_le(blk_prefix, batch + 1, n);
    if (m < blk_prefix[s] || m > n) return;  // other sequence, or above the diagonal
    const int nb = blk_prefix[s + 1] - blk_prefix[s];
    P[m_prefix[s] + (int64_t)(n - blk_prefix[s]) * nb + (m - blk_prefix[s])] = acc * inv_h;
}

}  // namespace predict
}  // namespace lemo
