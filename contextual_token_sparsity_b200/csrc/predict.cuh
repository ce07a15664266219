// predict.cuh - predicted token-block scores from low-rank ReLU predictors
// (step a8; Jenga summary section 4.2.2, Eq. 3 and the overhead analysis).
//
//   xbar_g   = mean of the rows of token block g of X                  (pool)
//   Qhat     = relu(xbar W1q) W2q,  Khat = relu(xbar W1k) W2k           (GEMMs)
//   P[n][m]  = (1/H) sum_h max(Qhat_n^h . Khat_m^h, 0),  n >= m          (block products)
//   score[m] = sum_{n >= m} P[n][m]                                      (column sum)
//
// The pooling pass streams X once and is bound by HBM bandwidth.  The
// predictor GEMMs and the block products are small (about 2 GFLOP at 32K
// tokens, one representative per block) and bound by latency, so they run
// as register-tiled warp-level tensor-core MMAs (m16n8k16, bf16 operands,
// fp32 accumulation) rather than as TMEM tiles sized for large problems.
// fp32 operands are split into two bf16 parts, v = hi + lo with
// hi = bf16(v) and lo = bf16(v - hi); a product a.b is taken as
// a_hi b_hi + a_hi b_lo + a_lo b_hi (the weights are bf16 already, so for
// the GEMMs only a_hi b + a_lo b is needed).  The dropped terms are below
// 2^-16 of the product, so the predicted scores stay at fp32 accuracy.
// Split-K partial sums and per-head-group partial products are reduced in a
// fixed order: results are the same bits on every run.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace lemo {
namespace predict {

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
    pdl_entry();
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
// Warp-level tensor-core tiles.  A CTA of 4 warps computes a 64 x 64 tile of
// C = A B^T from fp32 A [M][K] and B given either as bf16 [K][N] (predictor
// weights, row-major) or as fp32 [N][K] (the key-side embeddings of the
// block products).  K advances in stages of 32, double-buffered in shared
// memory: the next stage's global loads are in flight while the current one
// is multiplied.  Each warp owns a 32 x 32 sub-tile (2 x 4 MMAs of 16 x 8).
// Shared rows are 40 bf16 (80 bytes) apart, which makes every fragment load
// of a warp hit 32 distinct banks.
// ---------------------------------------------------------------------------
constexpr int TM = 64, TN = 64, TK = 32, SROW = 40;
constexpr int kMmaThreads = 128;
constexpr int kStageElems = TM * SROW;  // one bf16 plane of one operand

__device__ __forceinline__ void split2(float v, uint16_t& hi, uint16_t& lo) {
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
    hi = *reinterpret_cast<const uint16_t*>(&h);
    lo = *reinterpret_cast<const uint16_t*>(&l);
}

__device__ __forceinline__ uint32_t lds32(const uint16_t* p) {
    return *reinterpret_cast<const uint32_t*>(p);
}

__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, const uint32_t* b) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// 64 x 32 fp32 tile (rows r0.., columns k0..) -> 16 values per thread.
// Rows at or past `rows` and columns at or past `kend` read as 0.
__device__ __forceinline__ void load_f32_tile(const float* __restrict__ src, int64_t ld,
                                              int r0, int rows, int k0, int kend, float* v) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int e = threadIdx.x + kMmaThreads * i;
        const int r = r0 + (e >> 5), c = k0 + (e & 31);
        v[i] = (r < rows && c < kend) ? src[(int64_t)r * ld + c] : 0.f;
    }
}

__device__ __forceinline__ void store_f32_tile(const float* v, uint16_t* hi, uint16_t* lo) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int e = threadIdx.x + kMmaThreads * i;
        const int o = (e >> 5) * SROW + (e & 31);
        split2(v[i], hi[o], lo[o]);
    }
}

// 32 x 64 bf16 tile of a [K][N] row-major matrix (k0.., columns n0..),
// stored transposed as [n][k] in shared memory.
__device__ __forceinline__ void load_kn_tile(const uint16_t* __restrict__ src, int64_t ld,
                                             int k0, int kend, int n0, int ncols, uint16_t* v) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int e = threadIdx.x + kMmaThreads * i;
        const int k = k0 + (e >> 6), n = n0 + (e & 63);
        v[i] = (k < kend && n < ncols) ? src[(int64_t)k * ld + n] : (uint16_t)0;
    }
}

__device__ __forceinline__ void store_kn_tile(const uint16_t* v, uint16_t* bt) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int e = threadIdx.x + kMmaThreads * i;
        bt[(e & 63) * SROW + (e >> 6)] = v[i];
    }
}

// One stage (TK = 32) of the warp's 32 x 32 sub-tile.  B_LO: the B operand
// has a low part too (fp32 B); otherwise B is exact in bf16.
template <bool B_LO>
__device__ __forceinline__ void mma_stage(const uint16_t* ahi, const uint16_t* alo,
                                          const uint16_t* bhi, const uint16_t* blo,
                                          float (*acc)[4][4]) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int wm = (warp >> 1) * 32, wn = (warp & 1) * 32;
#pragma unroll
    for (int ks = 0; ks < TK; ks += 16) {
        uint32_t ah[2][4], al[2][4];
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
            const int r = (wm + mi * 16 + g) * SROW + ks + 2 * t;
            ah[mi][0] = lds32(ahi + r);
            ah[mi][1] = lds32(ahi + r + 8 * SROW);
            ah[mi][2] = lds32(ahi + r + 8);
            ah[mi][3] = lds32(ahi + r + 8 * SROW + 8);
            al[mi][0] = lds32(alo + r);
            al[mi][1] = lds32(alo + r + 8 * SROW);
            al[mi][2] = lds32(alo + r + 8);
            al[mi][3] = lds32(alo + r + 8 * SROW + 8);
        }
#pragma unroll
        for (int ni = 0; ni < 4; ++ni) {
            const int c = (wn + ni * 8 + g) * SROW + ks + 2 * t;
            const uint32_t bh[2] = {lds32(bhi + c), lds32(bhi + c + 8)};
#pragma unroll
            for (int mi = 0; mi < 2; ++mi) {
                mma16816(acc[mi][ni], ah[mi], bh);
                mma16816(acc[mi][ni], al[mi], bh);
            }
            if (B_LO) {
                const uint32_t bl[2] = {lds32(blo + c), lds32(blo + c + 8)};
#pragma unroll
                for (int mi = 0; mi < 2; ++mi) mma16816(acc[mi][ni], ah[mi], bl);
            }
        }
    }
}

__device__ __forceinline__ void zero_acc(float (*acc)[4][4]) {
#pragma unroll
    for (int mi = 0; mi < 2; ++mi)
#pragma unroll
        for (int ni = 0; ni < 4; ++ni)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[mi][ni][i] = 0.f;
}

// Visit the accumulator elements with their tile coordinates (row, column).
template <typename F>
__device__ __forceinline__ void for_acc(const float (*acc)[4][4], F f) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int wm = (warp >> 1) * 32, wn = (warp & 1) * 32;
#pragma unroll
    for (int mi = 0; mi < 2; ++mi)
#pragma unroll
        for (int ni = 0; ni < 4; ++ni)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                f(wm + mi * 16 + g + (i >> 1) * 8, wn + ni * 8 + 2 * t + (i & 1), acc[mi][ni][i]);
}

// ---------------------------------------------------------------------------
// Predictor GEMM, both predictors in one launch: for side s (0 = query,
// 1 = key) and K split z (blockIdx.z = s * splits + z),
//   C[s] (+ z * c_split)[m][n] = sum_{k in split z} A[s][m][k] W[s][k][n]
// with A fp32 [M][K] (M = number of token blocks, read on the device) and W
// bf16 [K][N] row-major.
// ---------------------------------------------------------------------------
struct GemmArgs {
    const float* a[2];
    int64_t lda;
    const uint16_t* w[2];
    int64_t ldw;
    float* c[2];
    int64_t ldc;
    int64_t c_split;   // elements between the split-K partial planes
    const PlanHeader* hdr;
    int N, K;
    int k_chunk;       // K range of one split (a multiple of TK)
    int splits;
};

__global__ void __launch_bounds__(kMmaThreads) gemm_kernel(const GemmArgs p) {
    pdl_entry();
    const int M = p.hdr->total_blocks;
    const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
    if (!p.hdr->valid || m0 >= M) return;
    const int side = blockIdx.z / p.splits, z = blockIdx.z % p.splits;
    const int kb = z * p.k_chunk, ke = min(p.K, kb + p.k_chunk);
    if (kb >= ke) return;
    __shared__ __align__(16) uint16_t sm[2][3][kStageElems];  // [buffer][A hi, A lo, B]
    const float* A = side ? p.a[1] : p.a[0];  // (a select: no local copy of the array)
    const uint16_t* W = side ? p.w[1] : p.w[0];
    float acc[2][4][4];
    zero_acc(acc);
    float av[16];
    uint16_t bv[16];
    const int nst = (ke - kb + TK - 1) / TK;
    load_f32_tile(A, p.lda, m0, M, kb, ke, av);
    load_kn_tile(W, p.ldw, kb, ke, n0, p.N, bv);
    store_f32_tile(av, sm[0][0], sm[0][1]);
    store_kn_tile(bv, sm[0][2]);
    __syncthreads();
    for (int s = 0; s < nst; ++s) {
        const int buf = s & 1;
        if (s + 1 < nst) {
            load_f32_tile(A, p.lda, m0, M, kb + (s + 1) * TK, ke, av);
            load_kn_tile(W, p.ldw, kb + (s + 1) * TK, ke, n0, p.N, bv);
        }
        mma_stage<false>(sm[buf][0], sm[buf][1], sm[buf][2], nullptr, acc);
        if (s + 1 < nst) {
            store_f32_tile(av, sm[buf ^ 1][0], sm[buf ^ 1][1]);
            store_kn_tile(bv, sm[buf ^ 1][2]);
        }
        __syncthreads();
    }
    float* C = (side ? p.c[1] : p.c[0]) + (int64_t)z * p.c_split;
    for_acc(acc, [&](int r, int c, float v) {
        if (m0 + r < M && n0 + c < p.N) C[(int64_t)(m0 + r) * p.ldc + n0 + c] = v;
    });
}

// hid[s][m][n] = relu(sum_z part[s][z][m][n]), z in increasing order, for
// both sides (blockIdx.y = side).  Partial planes are `plane` elements
// apart, rows N apart.
__global__ void __launch_bounds__(256)
    reduce_kernel(const float* __restrict__ part, int64_t side_stride, int64_t plane, int splits,
                  const PlanHeader* __restrict__ hdr, int N, float* __restrict__ hid,
                  int64_t hid_side_stride) {
    pdl_entry();
    if (!hdr->valid) return;
    const int64_t total = (int64_t)hdr->total_blocks * N;
    const float* src = part + blockIdx.y * side_stride;
    float* dst = hid + blockIdx.y * hid_side_stride;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        // loads in batches of 8 (in flight together), added in z order
        float v = 0.f;
        int z = 0;
        for (; z + 8 <= splits; z += 8) {
            float t[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) t[u] = src[(int64_t)(z + u) * plane + i];
#pragma unroll
            for (int u = 0; u < 8; ++u) v += t[u];
        }
        for (; z < splits; ++z) v += src[(int64_t)z * plane + i];
        dst[i] = fmaxf(v, 0.f);
    }
}

// ---------------------------------------------------------------------------
// Block products.  CTA (tile, head group): the 64 x 64 tile of block pairs
// (n, m) number `tile` of the lower triangle (tile rows tn >= tile columns
// tm), heads [g * hpg, (g + 1) * hpg).  For each head the tile's dot
// products Qhat_n^h . Khat_m^h are accumulated over dh, then their positive
// parts are added up.  With one head group the CTA writes
// P[n][m] = inv_h * sum directly (per-sequence [N_b, N_b] layout, pairs of
// one sequence with n >= m only); otherwise it writes its partial sums to
// plane g of `part` ([groups][tb_cap][tb_cap]) for products_reduce_kernel.
// ---------------------------------------------------------------------------
struct ProductsArgs {
    const float* qh;   // [TB][H * dh]
    const float* kh;
    int H, dh, hpg, groups, batch;
    int64_t tb_cap;    // row stride of the partial planes
    float inv_h;
    float* part;       // [groups][tb_cap][tb_cap] (groups > 1)
    float* P;          // per-sequence block-product matrices
};

__device__ __forceinline__ void store_pair(const ProductsArgs& a, const int32_t* blk_prefix,
                                           const int64_t* m_prefix, int s, int n, int m,
                                           float v) {
    const int b0 = blk_prefix[s];
    if (m < b0 || m > n) return;  // other sequence, or above the diagonal
    const int nb = blk_prefix[s + 1] - b0;
    a.P[m_prefix[s] + (int64_t)(n - b0) * nb + (m - b0)] = v * a.inv_h;
}

__global__ void __launch_bounds__(kMmaThreads)
    products_kernel(const ProductsArgs a, const char* __restrict__ ws, WsLayout lay) {
    pdl_entry();
    const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(ws + lay.hdr);
    if (!hdr->valid) return;
    const int32_t* blk_prefix = reinterpret_cast<const int32_t*>(ws + lay.blk_prefix);
    const int64_t* m_prefix = reinterpret_cast<const int64_t*>(ws + lay.m_prefix);
    const int TB = hdr->total_blocks;
    // lower-triangular tile number -> (tn, tm), tm <= tn
    const int idx = blockIdx.x;
    int tn = (int)((sqrtf(8.f * (float)idx + 1.f) - 1.f) * 0.5f);
    while ((tn + 1) * (tn + 2) / 2 <= idx) ++tn;
    while (tn * (tn + 1) / 2 > idx) --tn;
    const int tm = idx - tn * (tn + 1) / 2;
    const int n0 = tn * TM, mb0 = tm * TN;
    if (n0 >= TB) return;
    const int HD = a.H * a.dh;
    __shared__ __align__(16) uint16_t sm[2][4][kStageElems];  // [buffer][A hi, A lo, B hi, B lo]
    float acc[2][4][4], tot[2][4][4];
    zero_acc(tot);
    float av[16], bv[16];
    const int h0 = blockIdx.y * a.hpg, h1 = min(a.H, h0 + a.hpg);
    const int per_head = (a.dh + TK - 1) / TK;
    const int nst = (h1 - h0) * per_head;
    auto kpos = [&](int s, int& k0, int& ke) {
        const int h = h0 + s / per_head;
        k0 = h * a.dh + (s % per_head) * TK;
        ke = (h + 1) * a.dh;
    };
    int k0, ke;
    kpos(0, k0, ke);
    load_f32_tile(a.qh, HD, n0, TB, k0, ke, av);
    load_f32_tile(a.kh, HD, mb0, TB, k0, ke, bv);
    store_f32_tile(av, sm[0][0], sm[0][1]);
    store_f32_tile(bv, sm[0][2], sm[0][3]);
    __syncthreads();
    zero_acc(acc);
    for (int s = 0; s < nst; ++s) {
        const int buf = s & 1;
        if (s + 1 < nst) {
            kpos(s + 1, k0, ke);
            load_f32_tile(a.qh, HD, n0, TB, k0, ke, av);
            load_f32_tile(a.kh, HD, mb0, TB, k0, ke, bv);
        }
        mma_stage<true>(sm[buf][0], sm[buf][1], sm[buf][2], sm[buf][3], acc);
        if ((s + 1) % per_head == 0) {  // head complete: keep its positive part
#pragma unroll
            for (int mi = 0; mi < 2; ++mi)
#pragma unroll
                for (int ni = 0; ni < 4; ++ni)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        tot[mi][ni][i] += fmaxf(acc[mi][ni][i], 0.f);
                        acc[mi][ni][i] = 0.f;
                    }
        }
        if (s + 1 < nst) {
            store_f32_tile(av, sm[buf ^ 1][0], sm[buf ^ 1][1]);
            store_f32_tile(bv, sm[buf ^ 1][2], sm[buf ^ 1][3]);
        }
        __syncthreads();
    }
    if (a.groups == 1) {
        for_acc(tot, [&](int r, int c, float v) {
            const int n = n0 + r, m = mb0 + c;
            if (n >= TB || m >= TB) return;
            store_pair(a, blk_prefix, m_prefix, last_le(blk_prefix, a.batch + 1, n), n, m, v);
        });
    } else {
        float* plane = a.part + (int64_t)blockIdx.y * a.tb_cap * a.tb_cap;
        for_acc(tot, [&](int r, int c, float v) {
            const int n = n0 + r, m = mb0 + c;
            if (n < TB && m < TB && m <= n) plane[(int64_t)n * a.tb_cap + m] = v;
        });
    }
}

// P[n][m] = inv_h * sum_g part[g][n][m], g in increasing order, for the
// pairs of one sequence with n >= m (head groups > 1).  Threads run along
// m, so the partial planes are read with coalesced loads.
__global__ void __launch_bounds__(256)
    products_reduce_kernel(const ProductsArgs a, const char* __restrict__ ws, WsLayout lay) {
    pdl_entry();
    const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(ws + lay.hdr);
    if (!hdr->valid) return;
    const int32_t* blk_prefix = reinterpret_cast<const int32_t*>(ws + lay.blk_prefix);
    const int64_t* m_prefix = reinterpret_cast<const int64_t*>(ws + lay.m_prefix);
    const int TB = hdr->total_blocks;
    const int64_t total = (int64_t)TB * TB;
    const int64_t plane = a.tb_cap * a.tb_cap;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int n = (int)(i / TB), m = (int)(i % TB);
        if (m > n) continue;
        const int s = last_le(blk_prefix, a.batch + 1, n);
        if (m < blk_prefix[s]) continue;
        const int64_t o = (int64_t)n * a.tb_cap + m;
        // loads in batches of 8 (in flight together), added in g order
        float v = 0.f;
        int g = 0;
        for (; g + 8 <= a.groups; g += 8) {
            float t[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) t[u] = a.part[(g + u) * plane + o];
#pragma unroll
            for (int u = 0; u < 8; ++u) v += t[u];
        }
        for (; g < a.groups; ++g) v += a.part[g * plane + o];
        store_pair(a, blk_prefix, m_prefix, s, n, m, v);
    }
}

}  // namespace predict
}  // namespace lemo
