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
// fp32 values are split into two bf16 parts, v = hi + lo with
// hi = bf16(v) and lo = bf16(v - hi); a product a.b is taken as
// a_hi b_hi + a_lo b_hi + a_hi b_lo (the weights are bf16 already, so for
// the GEMMs only a_hi b + a_lo b is needed).  The dropped term is below
// 2^-16 of each product, so a score's error is about 2^-16 of the sum of
// the magnitudes of its products: near fp32 accuracy, except where a block
// pair's dot products cancel (then it stays small against the scores'
// scale, not against that one score).
//
// Every fp32 intermediate (block means, hidden activations, Qhat, Khat) is
// split once, by the kernel that produces it, and stored as two bf16 planes
// whose rows are padded to a multiple of 8 elements.  Every operand of every
// MMA kernel is read with cp.async (16-byte chunks; 4-byte ones for weight
// rows that are only 4-byte aligned; weights with odd row lengths are first
// copied into padded planes) through a shared-memory pipeline, zero-filled
// outside the matrix, and taken into registers with ldmatrix.  Split-K partial sums and
// per-head-group partial products are reduced in a fixed order: results
// are the same bits on every run.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace lemo {
namespace predict {

__device__ __forceinline__ void split2(float v, uint16_t& hi, uint16_t& lo) {
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
    hi = *reinterpret_cast<const uint16_t*>(&h);
    lo = *reinterpret_cast<const uint16_t*>(&l);
}

// Split 8 fp32 values and store them as 8 bf16 in each plane (16 bytes).
__device__ __forceinline__ void store_split8(const float* v, uint16_t* hi, uint16_t* lo) {
    uint16_t h[8], l[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) split2(v[i], h[i], l[i]);
    uint4 a, b;
    a.x = h[0] | ((uint32_t)h[1] << 16);  b.x = l[0] | ((uint32_t)l[1] << 16);
    a.y = h[2] | ((uint32_t)h[3] << 16);  b.y = l[2] | ((uint32_t)l[3] << 16);
    a.z = h[4] | ((uint32_t)h[5] << 16);  b.z = l[4] | ((uint32_t)l[5] << 16);
    a.w = h[6] | ((uint32_t)h[7] << 16);  b.w = l[6] | ((uint32_t)l[7] << 16);
    *reinterpret_cast<uint4*>(hi) = a;
    *reinterpret_cast<uint4*>(lo) = b;
}

// ---------------------------------------------------------------------------
// Weight planes.  pad_kernel copies a bf16 matrix [rows][cols] (any
// alignment) into a plane [rows_out][ld] whose rows are 16-byte aligned:
// columns are grouped in runs of `run` (the head dimension of W2, or all
// columns of W1), each run padded to `run_ld` (a multiple of 8); padding and
// rows >= rows are zero.  blockIdx.y selects one of up to four matrices;
// CTA x copies rows [8 x, 8 x + 8), 32 threads per row.
// ---------------------------------------------------------------------------
struct PadArgs {
    const uint16_t* src[4];
    uint16_t* dst[4];
    int rows, rows_out, cols, run, run_ld;
    int64_t ld_out;
};

__global__ void __launch_bounds__(256) pad_kernel(const PadArgs a) {
    pdl_entry();
    const int y = blockIdx.y;
    const uint16_t* src = y == 0 ? a.src[0] : y == 1 ? a.src[1] : y == 2 ? a.src[2] : a.src[3];
    uint16_t* dst = y == 0 ? a.dst[0] : y == 1 ? a.dst[1] : y == 2 ? a.dst[2] : a.dst[3];
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= a.rows_out) return;
    const int runs = a.cols / a.run, chunks_per_run = a.run_ld / 8;
    for (int c = threadIdx.x & 31; c < runs * chunks_per_run; c += 32) {
        const int r = c / chunks_per_run, c0 = (c % chunks_per_run) * 8;
        uint16_t v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            v[e] = (row < a.rows && c0 + e < a.run)
                       ? src[(int64_t)row * a.cols + (int64_t)r * a.run + c0 + e]
                       : (uint16_t)0;
        uint4 o;
        o.x = v[0] | ((uint32_t)v[1] << 16);
        o.y = v[2] | ((uint32_t)v[3] << 16);
        o.z = v[4] | ((uint32_t)v[5] << 16);
        o.w = v[6] | ((uint32_t)v[7] << 16);
        *reinterpret_cast<uint4*>(dst + (int64_t)row * a.ld_out + (int64_t)r * a.run_ld + c0) = o;
    }
}

// ---------------------------------------------------------------------------
// Pooling pass.  CTA (g, c): block means of token block g, columns
// [c*2048, +2048), each thread 8 consecutive columns (16-byte loads, four
// rows in flight, added in row order), written as hi / lo planes [TB][d].
// ---------------------------------------------------------------------------
constexpr int kPoolThreads = 256;
constexpr int kPoolCols = kPoolThreads * 8;

__device__ __forceinline__ void add_row(float* acc, const uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(w[i] << 16);
        acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
    }
}

__global__ void __launch_bounds__(kPoolThreads)
    pool_kernel(const uint16_t* __restrict__ x, int64_t ld_x, int d, const int32_t* __restrict__ cu,
                int batch, int block, const char* __restrict__ ws, WsLayout lay,
                uint16_t* __restrict__ xb_hi, uint16_t* __restrict__ xb_lo) {
    pdl_entry();
    const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(ws + lay.hdr);
    if (!hdr->valid) return;
    const int g = blockIdx.x;
    if (g >= hdr->total_blocks) return;
    const int32_t* blk_prefix = reinterpret_cast<const int32_t*>(ws + lay.blk_prefix);
    const int s = last_le(blk_prefix, batch + 1, g);
    const int m = g - blk_prefix[s];
    const int64_t r0 = (int64_t)cu[s] + (int64_t)m * block;
    const int64_t r1 = min((int64_t)cu[s + 1], r0 + block);
    const int c = blockIdx.y * kPoolCols + threadIdx.x * 8;
    if (c >= d) return;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const uint16_t* p = x + r0 * ld_x + c;
    int64_t r = r0;
    for (; r + 4 <= r1; r += 4, p += 4 * ld_x) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = *reinterpret_cast<const uint4*>(p + u * ld_x);
#pragma unroll
        for (int u = 0; u < 4; ++u) add_row(acc, v[u]);
    }
    for (; r < r1; ++r, p += ld_x) add_row(acc, *reinterpret_cast<const uint4*>(p));
    const float inv = 1.f / (float)(r1 - r0);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] *= inv;
    store_split8(acc, xb_hi + (int64_t)g * d + c, xb_lo + (int64_t)g * d + c);
}

// ---------------------------------------------------------------------------
// Warp-level tensor-core tiles.  A CTA of 4 warps computes a 64 x 64 tile of
// C = A B: A is a pair of bf16 planes [M][lda] (hi, lo) and B either a bf16
// plane [K][ldb] (weights, N contiguous) or a pair of bf16 planes [N][ldb]
// (Khat, K contiguous).  K advances in stages of 32 through a ring of
// shared-memory buffers filled by cp.async (16-byte chunks; chunks outside
// the matrix are zero-filled), so the loads of the next stages are in
// flight while the current one is multiplied.  Each warp owns a 32 x 32
// sub-tile (2 x 4 MMAs of 16 x 8) and takes its fragments with ldmatrix
// (.trans for the N-contiguous weights).  Row pitches of 80 and 144 bytes
// keep every ldmatrix phase on distinct banks.
// ---------------------------------------------------------------------------
constexpr int TM = 64, TN = 64, TK = 32;
constexpr int kMmaThreads = 128;
constexpr int A_PITCH = 80;                 // bytes per row of a [64][32] bf16 tile
constexpr int A_PLANE = TM * A_PITCH;       // 5120 bytes
constexpr int B_PITCH = 144;                // bytes per row of a [32][64] bf16 tile
constexpr int B_PLANE = TK * B_PITCH;       // 4608 bytes
constexpr int GEMM_STAGES = 3;
constexpr int GEMM_STAGE = 2 * A_PLANE + B_PLANE;
constexpr int PROD_STAGES = 3;
constexpr int PROD_STAGE = 4 * A_PLANE;
constexpr int PROD_SMEM = PROD_STAGES * PROD_STAGE;  // dynamic shared memory (60 KB)

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// 16 bytes global -> shared; `valid` false writes 16 zero bytes (nothing is read).
__device__ __forceinline__ void cp16(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(valid ? 16u : 0u)
                 : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t* r) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, const uint32_t* b) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// A [64][32] bf16 tile of a K-contiguous plane (rows r0.., columns k0..)
// into shared memory (pitch A_PITCH): 256 chunks, two per thread.  Chunks of
// rows >= rows or at columns >= kend are zero (kend is a multiple of 8).
__device__ __forceinline__ void load_k_tile(uint8_t* dst, const uint16_t* __restrict__ src,
                                            int64_t ld, int r0, int rows, int k0, int kend) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int c = threadIdx.x + kMmaThreads * i;
        const int r = c >> 2, kc = (c & 3) * 8;
        const bool ok = r0 + r < rows && k0 + kc < kend;
        cp16(smem_addr(dst + r * A_PITCH + kc * 2), ok ? src + (int64_t)(r0 + r) * ld + k0 + kc : src,
             ok);
    }
}

// 4 bytes global -> shared (same zero fill).
__device__ __forceinline__ void cp4(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
                 "r"(valid ? 4u : 0u)
                 : "memory");
}

// A [32][64] bf16 tile of an N-contiguous matrix [K][ld] (rows k0.., columns
// n0..) into shared memory (pitch B_PITCH); rows >= kend, columns >= ncols
// are zero.  VEC16: rows 16-byte aligned, ncols a multiple of 8 (two
// 16-byte chunks per thread); otherwise rows 4-byte aligned, ncols even
// (eight 4-byte copies per thread).
template <bool VEC16>
__device__ __forceinline__ void load_n_tile(uint8_t* dst, const uint16_t* __restrict__ src,
                                            int64_t ld, int k0, int kend, int n0, int ncols) {
    if (VEC16) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int c = threadIdx.x + kMmaThreads * i;
            const int k = c >> 3, nc = (c & 7) * 8;
            const bool ok = k0 + k < kend && n0 + nc < ncols;
            cp16(smem_addr(dst + k * B_PITCH + nc * 2),
                 ok ? src + (int64_t)(k0 + k) * ld + n0 + nc : src, ok);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int c = threadIdx.x + kMmaThreads * i;
            const int k = c >> 5, nc = (c & 31) * 2;
            const bool ok = k0 + k < kend && n0 + nc < ncols;
            cp4(smem_addr(dst + k * B_PITCH + nc * 2),
                ok ? src + (int64_t)(k0 + k) * ld + n0 + nc : src, ok);
        }
    }
}

// A fragments (rows wm + 16 mi ..) of one plane at K offset ks.
__device__ __forceinline__ void frag_a(const uint8_t* tile, int wm, int ks, uint32_t (*a)[4]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int mi = 0; mi < 2; ++mi)
        ldsm4(smem_addr(tile + (wm + mi * 16 + (lane & 15)) * A_PITCH + (ks + (lane >> 4) * 8) * 2),
              a[mi]);
}

// B fragments of the 4 n8 blocks (columns wn ..) at K offset ks, from an
// N-contiguous [32][64] tile (transposing loads) ...
__device__ __forceinline__ void frag_b_n(const uint8_t* tile, int wn, int ks, uint32_t (*b)[2]) {
    const int lane = threadIdx.x & 31, mtx = lane >> 3, r8 = lane & 7;
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        uint32_t r[4];
        ldsm4t(smem_addr(tile + (ks + (mtx & 1) * 8 + r8) * B_PITCH + (wn + 16 * p + (mtx >> 1) * 8) * 2),
               r);
        b[2 * p][0] = r[0];
        b[2 * p][1] = r[1];
        b[2 * p + 1][0] = r[2];
        b[2 * p + 1][1] = r[3];
    }
}

// ... or from a K-contiguous [64][32] tile.
__device__ __forceinline__ void frag_b_k(const uint8_t* tile, int wn, int ks, uint32_t (*b)[2]) {
    const int lane = threadIdx.x & 31, mtx = lane >> 3, r8 = lane & 7;
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        uint32_t r[4];
        ldsm4(smem_addr(tile + (wn + 16 * p + (mtx >> 1) * 8 + r8) * A_PITCH + (ks + (mtx & 1) * 8) * 2),
              r);
        b[2 * p][0] = r[0];
        b[2 * p][1] = r[1];
        b[2 * p + 1][0] = r[2];
        b[2 * p + 1][1] = r[3];
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
// with A = hi + lo bf16 planes [M][lda] (M = number of token blocks, read
// on the device) and W bf16 [K][ldw] with w_cols columns (columns w_cols ..
// N - 1 read as zero).  SPLIT_OUT: C is written as hi / lo planes (c, c_lo)
// for the block products, else as fp32 (split-K partial sums).
// ---------------------------------------------------------------------------
struct GemmArgs {
    const uint16_t* a_hi[2];
    const uint16_t* a_lo[2];
    int64_t lda;
    const uint16_t* w[2];
    int64_t ldw;
    float* c[2];         // fp32 output
    uint16_t* c_hi[2];   // split output
    uint16_t* c_lo[2];
    int64_t ldc;
    int64_t c_split;     // elements between the split-K partial planes
    const PlanHeader* hdr;
    int N, K;
    int w_rows;          // rows of W that exist (rows past it read as zero)
    int w_cols;          // columns of W that exist (a multiple of 8, or even with w_vec4)
    bool w_vec4;         // W rows only 4-byte aligned: 4-byte copies
    int k_chunk;         // K range of one split (a multiple of TK)
    int splits;
};

template <bool SPLIT_OUT>
__global__ void __launch_bounds__(kMmaThreads) gemm_kernel(const GemmArgs p) {
    pdl_entry();
    const int M = p.hdr->total_blocks;
    const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
    if (!p.hdr->valid || m0 >= M) return;
    const int side = blockIdx.z / p.splits, z = blockIdx.z % p.splits;
    const int kb = z * p.k_chunk, ke = min(p.K, kb + p.k_chunk);
    if (kb >= ke) return;
    __shared__ __align__(128) uint8_t sm[GEMM_STAGES][GEMM_STAGE];  // [A hi | A lo | B]
    const uint16_t* Ah = side ? p.a_hi[1] : p.a_hi[0];  // (selects: no local copy of the arrays)
    const uint16_t* Al = side ? p.a_lo[1] : p.a_lo[0];
    const uint16_t* W = side ? p.w[1] : p.w[0];
    const int warp = threadIdx.x >> 5;
    const int wm = (warp >> 1) * 32, wn = (warp & 1) * 32;
    float acc[2][4][4];
    zero_acc(acc);
    const int nst = (ke - kb + TK - 1) / TK;
    auto load_stage = [&](int s) {
        uint8_t* b = sm[s % GEMM_STAGES];
        const int k0 = kb + s * TK;
        load_k_tile(b, Ah, p.lda, m0, M, k0, ke);
        load_k_tile(b + A_PLANE, Al, p.lda, m0, M, k0, ke);
        if (p.w_vec4)
            load_n_tile<false>(b + 2 * A_PLANE, W, p.ldw, k0, min(ke, p.w_rows), n0, p.w_cols);
        else
            load_n_tile<true>(b + 2 * A_PLANE, W, p.ldw, k0, min(ke, p.w_rows), n0, p.w_cols);
    };
#pragma unroll
    for (int s = 0; s < GEMM_STAGES - 1; ++s) {
        if (s < nst) load_stage(s);
        cp_commit();
    }
    for (int s = 0; s < nst; ++s) {
        cp_wait<GEMM_STAGES - 2>();
        __syncthreads();  // stage s landed for every thread; stage s - 1 is no longer read
        if (s + GEMM_STAGES - 1 < nst) load_stage(s + GEMM_STAGES - 1);
        cp_commit();
        const uint8_t* b = sm[s % GEMM_STAGES];
#pragma unroll
        for (int ks = 0; ks < TK; ks += 16) {
            uint32_t ah[2][4], al[2][4], bf[4][2];
            frag_a(b, wm, ks, ah);
            frag_a(b + A_PLANE, wm, ks, al);
            frag_b_n(b + 2 * A_PLANE, wn, ks, bf);
#pragma unroll
            for (int ni = 0; ni < 4; ++ni)
#pragma unroll
                for (int mi = 0; mi < 2; ++mi) {
                    mma16816(acc[mi][ni], ah[mi], bf[ni]);
                    mma16816(acc[mi][ni], al[mi], bf[ni]);
                }
        }
    }
    if (SPLIT_OUT) {
        // hi / lo tiles [64][64] staged in shared memory (pitch B_PITCH),
        // then written as 16-byte row chunks
        uint16_t* Ch = side ? p.c_hi[1] : p.c_hi[0];
        uint16_t* Cl = side ? p.c_lo[1] : p.c_lo[0];
        cp_wait<0>();
        __syncthreads();  // every warp is done with the operand buffers
        uint8_t* th = &sm[0][0];  // 2 x 64 rows of B_PITCH: spans the first two stages
        uint8_t* tl = th + TM * B_PITCH;
        static_assert(2 * TM * B_PITCH <= GEMM_STAGES * GEMM_STAGE, "staging exceeds the ring");
        for_acc(acc, [&](int r, int c, float v) {
            uint16_t h, l;
            split2(v, h, l);
            *reinterpret_cast<uint16_t*>(th + r * B_PITCH + c * 2) = h;
            *reinterpret_cast<uint16_t*>(tl + r * B_PITCH + c * 2) = l;
        });
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = threadIdx.x + kMmaThreads * i;  // 512 chunks of 8 per plane
            const int r = e >> 3, c = (e & 7) * 8;
            if (m0 + r < M && n0 + c < p.N) {
                const int64_t o = (int64_t)(m0 + r) * p.ldc + n0 + c;
                *reinterpret_cast<uint4*>(Ch + o) = *reinterpret_cast<const uint4*>(th + r * B_PITCH + c * 2);
                *reinterpret_cast<uint4*>(Cl + o) = *reinterpret_cast<const uint4*>(tl + r * B_PITCH + c * 2);
            }
        }
    } else {
        float* C = (side ? p.c[1] : p.c[0]) + (int64_t)z * p.c_split;
        for_acc(acc, [&](int r, int c, float v) {
            if (m0 + r < M && n0 + c < p.N) C[(int64_t)(m0 + r) * p.ldc + n0 + c] = v;
        });
    }
}

// hid[s][m][n] = relu(sum_z part[s][z][m][n]), z in increasing order, for
// both sides (blockIdx.y = side), written as hi / lo planes.  Partial
// planes are `plane` elements apart, rows N apart (N a multiple of 8); each
// thread takes 4 consecutive elements and keeps the loads of 8 splits in
// flight at a time.
__global__ void __launch_bounds__(256)
    reduce_kernel(const float* __restrict__ part, int64_t side_stride, int64_t plane, int splits,
                  const PlanHeader* __restrict__ hdr, int N, uint16_t* __restrict__ hid_hi,
                  uint16_t* __restrict__ hid_lo, int64_t hid_side_stride) {
    pdl_entry();
    if (!hdr->valid) return;
    const int64_t total = (int64_t)hdr->total_blocks * N / 4;
    const float* src = part + blockIdx.y * side_stride;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        int z = 0;
        for (; z + 8 <= splits; z += 8) {
            float4 t[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                t[u] = *reinterpret_cast<const float4*>(src + (int64_t)(z + u) * plane + i * 4);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                v.x += t[u].x; v.y += t[u].y; v.z += t[u].z; v.w += t[u].w;
            }
        }
        for (; z < splits; ++z) {
            const float4 t = *reinterpret_cast<const float4*>(src + (int64_t)z * plane + i * 4);
            v.x += t.x; v.y += t.y; v.z += t.z; v.w += t.w;
        }
        const float r[4] = {fmaxf(v.x, 0.f), fmaxf(v.y, 0.f), fmaxf(v.z, 0.f), fmaxf(v.w, 0.f)};
        uint16_t h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) split2(r[e], h[e], l[e]);
        const int64_t o = blockIdx.y * hid_side_stride + i * 4;
        *reinterpret_cast<uint2*>(hid_hi + o) =
            make_uint2(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16));
        *reinterpret_cast<uint2*>(hid_lo + o) =
            make_uint2(l[0] | ((uint32_t)l[1] << 16), l[2] | ((uint32_t)l[3] << 16));
    }
}

// ---------------------------------------------------------------------------
// Block products.  CTA (tile, head group): the 64 x 64 tile of block pairs
// (n, m) number `tile` of the lower triangle (tile rows tn >= tile columns
// tm), heads [g * hpg, (g + 1) * hpg).  For each head the tile's dot
// products Qhat_n^h . Khat_m^h are accumulated over its ldh columns (dh
// values and zero padding), then their positive parts are added up.  With
// one head group the CTA writes P[n][m] = inv_h * sum directly (per-sequence
// [N_b, N_b] layout, pairs of one sequence with n >= m only); otherwise it
// writes its partial sums to plane g of `part` ([groups][tb_cap][tb_cap])
// for products_reduce_kernel.
// ---------------------------------------------------------------------------
struct ProductsArgs {
    const uint16_t* q_hi;   // [TB][H * ldh]
    const uint16_t* q_lo;
    const uint16_t* k_hi;
    const uint16_t* k_lo;
    int H, ldh, hpg, groups, batch;
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
    const int64_t HD = (int64_t)a.H * a.ldh;
    extern __shared__ __align__(128) uint8_t prod_smem[];  // stages of [Q hi | Q lo | K hi | K lo]
    const int warp = threadIdx.x >> 5;
    const int wm = (warp >> 1) * 32, wn = (warp & 1) * 32;
    float acc[2][4][4], tot[2][4][4];
    zero_acc(tot);
    zero_acc(acc);
    const int h0 = blockIdx.y * a.hpg, h1 = min(a.H, h0 + a.hpg);
    const int per_head = (a.ldh + TK - 1) / TK;
    const int nst = (h1 - h0) * per_head;
    auto load_stage = [&](int s) {
        uint8_t* b = prod_smem + (s % PROD_STAGES) * PROD_STAGE;
        const int h = h0 + s / per_head;
        const int k0 = h * a.ldh + (s % per_head) * TK, ke = (h + 1) * a.ldh;
        load_k_tile(b, a.q_hi, HD, n0, TB, k0, ke);
        load_k_tile(b + A_PLANE, a.q_lo, HD, n0, TB, k0, ke);
        load_k_tile(b + 2 * A_PLANE, a.k_hi, HD, mb0, TB, k0, ke);
        load_k_tile(b + 3 * A_PLANE, a.k_lo, HD, mb0, TB, k0, ke);
    };
#pragma unroll
    for (int s = 0; s < PROD_STAGES - 1; ++s) {
        if (s < nst) load_stage(s);
        cp_commit();
    }
    for (int s = 0; s < nst; ++s) {
        cp_wait<PROD_STAGES - 2>();
        __syncthreads();  // stage s landed for every thread; stage s - 1 is no longer read
        if (s + PROD_STAGES - 1 < nst) load_stage(s + PROD_STAGES - 1);
        cp_commit();
        const uint8_t* b = prod_smem + (s % PROD_STAGES) * PROD_STAGE;
#pragma unroll
        for (int ks = 0; ks < TK; ks += 16) {
            uint32_t ah[2][4], al[2][4], bh[4][2], bl[4][2];
            frag_a(b, wm, ks, ah);
            frag_a(b + A_PLANE, wm, ks, al);
            frag_b_k(b + 2 * A_PLANE, wn, ks, bh);
            frag_b_k(b + 3 * A_PLANE, wn, ks, bl);
#pragma unroll
            for (int ni = 0; ni < 4; ++ni) {
#pragma unroll
                for (int mi = 0; mi < 2; ++mi) {
                    mma16816(acc[mi][ni], ah[mi], bh[ni]);
                    mma16816(acc[mi][ni], al[mi], bh[ni]);
                }
#pragma unroll
                for (int mi = 0; mi < 2; ++mi) mma16816(acc[mi][ni], ah[mi], bl[ni]);
            }
        }
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
