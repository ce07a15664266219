// predict.cuh - predicted token-block scores from low-rank ReLU predictors
// (step a8; Jenga summary section 4.2.2, Eq. 3 and the overhead analysis).
//
//   xbar_g   = mean of the rows of token block g of X                  (pool)
//   Qhat     = relu(xbar W1q) W2q,  Khat = relu(xbar W1k) W2k           (GEMMs)
//   P[n][m]  = (1/H) sum_h max(Qhat_n^h . Khat_m^h, 0),  n >= m          (block products)
//   score[m] = sum_{n >= m} P[n][m]                                      (column sum)
//
// Two kernels (after the per-call plan kernel when the batch has several
// sequences; for one sequence the pooling pass writes the plan itself):
//
//   pool_kernel     streams X once (bound by HBM bandwidth) and writes the
//                   block means as bf16 hi / lo planes already laid out as
//                   tensor-core operand tiles; a few extra CTAs copy weights
//                   whose rows are not 16-byte aligned into padded planes;
//   predict_kernel  one persistent CTA per SM runs everything else as
//                   phases separated by grid-wide barriers:
//                     A  split-K partial products xbar W1 (both predictors)
//                     B  sum of the split-K partials, ReLU, hi / lo split
//                     C  the hidden activations times W2 -> Qhat, Khat tiles, in
//                        column units sized to about one per SM
//                     D  Eq. 3 block products, positive part, per head group
//                     E  per token block: the head groups and the rows n >= m
//                        summed in a fixed order -> the block score.
//
// Every contraction runs on the tensor cores: tcgen05.mma (cta_group::1,
// M = 128, kind::f16, bf16 operands from shared memory, fp32 accumulators in
// tensor memory, read back with tcgen05.ld).  fp32 operands are split into
// two bf16 parts, v = hi + lo with hi = bf16(v) and lo = bf16(v - hi), and a
// product a.b is taken as a_hi b_hi + a_lo b_hi + a_hi b_lo in one fp32
// accumulator (a_hi b + a_lo b when b is a bf16 weight).  The dropped term is
// below 2^-16 of each product, so scores keep about fp32 accuracy.
//
// Operand tiles ("images") are [128 rows x 64] bf16 K-major blocks of 16 KB
// in the layout a 128-byte-swizzled TMA box would have: 8-row groups of 1024
// bytes, row r at 128 (r % 8), its 16-byte chunk j at (j ^ (r % 8)) * 16.
// Every intermediate is written by its producer directly in that layout, so
// a consumer fetches a whole tile with one bulk copy (cp.async.bulk).  The
// weights arrive through TMA as MN-major 64 x 64 boxes (64 rows of K, 64
// columns, 128-byte swizzle), four per 256-column tile.
//
// Per CTA: warp 0 issues the copies into a 3-stage ring of 64 KB, warp 1 the
// MMAs into two 256-column accumulators, warps 2-9 run the epilogues and the
// reductions.  Sums are taken in a fixed order everywhere (split-K partials,
// head groups, rows): results are the same bits on every run.  Every wait -
// mbarriers and the grid barriers - is bounded in time; a wait that runs out
// records LEMO_ERR_TIMEOUT, raises a flag that makes every CTA skip the rest,
// and each CTA drains what it issued and frees its tensor memory before it
// returns.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "score.cuh"

namespace lemo {
namespace predict {

using score::mbar_arrive;
using score::mbar_arrive_expect_tx;
using score::mbar_init;
using score::mbar_try_wait;
using score::smem_u32;
using score::tc_fence_after;
using score::tc_fence_before;
using score::tmem_ld16;
using score::tmem_wait_ld;

constexpr int TILE = 128;                 // rows of a row tile (MMA M, TMEM lanes)
constexpr int KCH = 64;                   // K elements of one image (one 128-byte row)
constexpr int IMG = TILE * KCH * 2;       // 16 KB
constexpr int WBOX = 64 * 64 * 2;         // one 64 x 64 weight box: 8 KB
constexpr int STAGES = 3;
constexpr int STAGE_BYTES = 4 * IMG;      // A hi | A lo | B (hi) | B lo
constexpr int EPI_WARPS = 8;              // epilogue / reduction warps (2..9)
constexpr int THREADS = 32 * (2 + EPI_WARPS);
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 2 * ACC_COLS;
constexpr int MAX_NT = 256;               // widest MMA N
constexpr int kPoolThreads = 128;
constexpr int kPoolCols = kPoolThreads * 8;  // columns of X per pooling CTA
constexpr int kPadCtas = 148;                // CTAs of the weight-padding part

// Grid-barrier words (in the workspace; zeroed by the pooling pass).
constexpr int kSyncA = 0, kSyncB = 1, kSyncC = 2, kSyncD = 3, kSyncAbort = 7;
constexpr int kSyncWords = 8;

struct Smem {
    uint64_t full[STAGES];      // the stage's copies landed
    uint64_t empty[STAGES];     // the MMAs reading the stage completed
    uint64_t acc_full[2];       // accumulator holds a finished product
    uint64_t acc_empty[2];      // the epilogue warps read the accumulator
    uint64_t done;              // every MMA of this CTA completed
    uint32_t tmem_base;
    int abort_flag;
    float red[EPI_WARPS + 2];   // per-warp partial sums of phase E (first column)
    float red2[EPI_WARPS + 2];  // (second column)
};
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align slack*/ + (int)sizeof(Smem);
static_assert(SMEM_BYTES <= 232448, "exceeds the 227 KB of shared memory per CTA");

// Byte offset of element e (0..63) of row r (0..127) inside an image.
__host__ __device__ __forceinline__ uint32_t img_off(int r, int e) {
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((((e >> 3) ^ (r & 7)) & 7) << 4) +
                      ((e & 7) << 1));
}

// Split 8 fp32 values into two 16-byte chunks (8 bf16 each): hi = bf16(v),
// lo = bf16(v - hi), both rounded to nearest even, two values per conversion
// instruction.
__device__ __forceinline__ void split8(const float* v, uint4& a, uint4& b) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 hh = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        const __nv_bfloat162 ll = __floats2bfloat162_rn(v[2 * i] - __low2float(hh),
                                                        v[2 * i + 1] - __high2float(hh));
        h[i] = *reinterpret_cast<const uint32_t*>(&hh);
        l[i] = *reinterpret_cast<const uint32_t*>(&ll);
    }
    a = make_uint4(h[0], h[1], h[2], h[3]);
    b = make_uint4(l[0], l[1], l[2], l[3]);
}

// 8 consecutive bf16 starting at src; elements at or past `valid` are zero.
// vec4: src is 4-byte aligned (4-byte loads for whole pairs), else 2-byte loads.
__device__ __forceinline__ uint4 load8_any(const uint16_t* src, int valid, bool vec4) {
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (vec4) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (2 * i + 1 < valid)
                w[i] = __ldg(reinterpret_cast<const uint32_t*>(src) + i);
            else if (2 * i < valid)
                w[i] = __ldg(src + 2 * i);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (i < valid) w[i >> 1] |= (uint32_t)__ldg(src + i) << ((i & 1) * 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// ---------------------------------------------------------------------------
// Pooling pass.  CTA npad + g * nch + y (block g, column chunk y of nch, so
// that the grid is one wave of plain CTAs): block means of token block g over columns
// [y*1024, +1024), each thread 8 consecutive columns (16-byte
// loads, eight rows in flight, added in row order).  The means are written
// as hi / lo images [row tile][64-column chunk][plane]; rows g >= TB and
// columns >= d of the last tile / chunk are written as zeros.  CTA 0 also
// clears the grid-barrier words of predict_kernel and, for a batch of one
// sequence (`own_plan`), writes the plan itself (no separate plan launch;
// the pooling CTAs then take block g as rows [g b, g b + b)).  The first `npad`
// CTAs (scheduled first, beside the pooling CTAs) copy the
// weights that TMA cannot read in place (rows not 16-byte aligned, or a head
// dimension that is not a multiple of 64) into padded planes.
// ---------------------------------------------------------------------------
struct PadArgs {
    const uint16_t* w1[2];   // [d, rank] sources
    uint16_t* w1p[2];        // [d, ldw1] planes (null: not padded)
    const uint16_t* w2[2];   // [rank, H dh] sources
    uint16_t* w2p[2];        // [rank, H dhp] planes, head h at columns h dhp (null: not padded)
    int d, rank, ldw1, H, dh, dhp;
    int w2_vec4;             // the W2 source rows allow 4-byte loads
};

__device__ __forceinline__ void add_row(float* acc, const uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(w[i] << 16);
        acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
    }
}

// 8 bf16 of the contiguous matrix `src` starting at element e (any 2-byte
// alignment of src + e), elements at or past `valid` zero: one or two aligned
// 16-byte loads and a byte funnel shift.  Consecutive threads taking
// consecutive chunks read consecutive 16-byte words (coalesced).  The second
// load is made only when valid elements lie in it, so nothing past the last
// element of the matrix is read.
__device__ __forceinline__ uint4 load8_shifted(const uint16_t* src, int64_t e, int valid) {
    if (valid <= 0) return make_uint4(0u, 0u, 0u, 0u);
    const uintptr_t b = reinterpret_cast<uintptr_t>(src + e);
    const uint32_t sh = (uint32_t)(b & 15u);  // even
    const uint4* a0 = reinterpret_cast<const uint4*>(b - sh);
    const int nbytes = (valid < 8 ? valid : 8) * 2;
    const uint4 v0 = __ldg(a0);
    const uint4 v1 = (int)sh + nbytes > 16 ? __ldg(a0 + 1) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    const uint32_t q = sh >> 2, bits = (sh & 3u) * 8u;
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        // words q + k and q + k + 1 (q <= 3), selected without local memory
        uint32_t lo = w[k], hi = w[k + 1];
        if (q == 1) { lo = w[k + 1]; hi = w[k + 2]; }
        if (q == 2) { lo = w[k + 2]; hi = w[k + 3]; }
        if (q == 3) { lo = w[k + 3]; hi = w[k + 4]; }
        o[k] = __funnelshift_r(lo, hi, bits);
    }
    // zero the elements at or past `valid`
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        if (2 * k >= valid) o[k] = 0u;
        else if (2 * k + 1 >= valid) o[k] &= 0xffffu;
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// Thread t of T copies the 16-byte chunks t, t + T, ... of both padded W1
// planes, then of both padded W2 planes, with eight loads in flight per
// thread (consecutive threads take consecutive chunks of a row).  Chunk
// indices are kept as (row, chunk) pairs advanced by T, so no integer
// division runs per chunk.
struct PadCursor {
    int64_t r;  // row (of one plane; rows of the second plane follow the first's)
    int c;      // 16-byte chunk within the row
};
__device__ __forceinline__ PadCursor pad_cursor(int64_t i, int cpr) {
    PadCursor k;
    k.r = i / cpr;
    k.c = (int)(i - k.r * cpr);
    return k;
}
__device__ __forceinline__ void pad_advance(PadCursor& k, int dr, int dc, int cpr) {
    k.r += dr;
    k.c += dc;
    if (k.c >= cpr) {
        k.c -= cpr;
        ++k.r;
    }
}

__device__ __noinline__ void pad_weights(const PadArgs& pa, int cta, int nctas) {
    const int64_t T = (int64_t)nctas * kPoolThreads;
    const int64_t t = (int64_t)cta * kPoolThreads + threadIdx.x;
    if (pa.w1p[0]) {
        // rows 0 .. 2d-1: plane p = row / d
        const int cpr = pa.ldw1 / 8;
        const int64_t rows = 2 * (int64_t)pa.d;
        const int dr = (int)(T / cpr), dc = (int)(T % cpr);
        PadCursor k = pad_cursor(t, cpr);
        while (k.r < rows) {
            PadCursor kk = k;
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const bool live = kk.r < rows;
                const int p = kk.r >= pa.d ? 1 : 0;
                const int64_t r = kk.r - (int64_t)p * pa.d;
                const int c = kk.c * 8;
                v[u] = live ? load8_shifted(pa.w1[p], r * pa.rank + c, pa.rank - c)
                            : make_uint4(0u, 0u, 0u, 0u);
                pad_advance(kk, dr, dc, cpr);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (k.r < rows) {
                    const int p = k.r >= pa.d ? 1 : 0;
                    const int64_t r = k.r - (int64_t)p * pa.d;
                    *reinterpret_cast<uint4*>(pa.w1p[p] + r * pa.ldw1 + k.c * 8) = v[u];
                }
                pad_advance(k, dr, dc, cpr);
            }
        }
    }
    if (pa.w2p[0]) {
        // rows 0 .. 2 rank - 1: plane p = row / rank
        const int cpr = pa.H * pa.dhp / 8;
        const int64_t rows = 2 * (int64_t)pa.rank;
        const int dr = (int)(T / cpr), dc = (int)(T % cpr);
        PadCursor k = pad_cursor(t, cpr);
        while (k.r < rows) {
            PadCursor kk = k;
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const bool live = kk.r < rows;
                const int p = kk.r >= pa.rank ? 1 : 0;
                const int64_t r = kk.r - (int64_t)p * pa.rank;
                const int nn = kk.c * 8;
                const int h = nn / pa.dhp, e = nn - h * pa.dhp;
                v[u] = live ? load8_any(pa.w2[p] + r * pa.H * pa.dh + (int64_t)h * pa.dh + e,
                                        pa.dh - e, pa.w2_vec4 != 0)
                            : make_uint4(0u, 0u, 0u, 0u);
                pad_advance(kk, dr, dc, cpr);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (k.r < rows) {
                    const int p = k.r >= pa.rank ? 1 : 0;
                    const int64_t r = k.r - (int64_t)p * pa.rank;
                    *reinterpret_cast<uint4*>(pa.w2p[p] + r * pa.H * pa.dhp + k.c * 8) = v[u];
                }
                pad_advance(k, dr, dc, cpr);
            }
        }
    }
}

__global__ void __launch_bounds__(kPoolThreads)
    pool_kernel(const uint16_t* __restrict__ x, int64_t ld_x, int d, int kc, int npad,
                const int32_t* __restrict__ cu, int batch, int total_L, int max_seqlen, int block,
                char* __restrict__ ws, WsLayout lay, uint8_t* __restrict__ xb,
                uint32_t* __restrict__ sync, const PadArgs pa, int own_plan) {
    pdl_entry();
    if (blockIdx.x == 0) {
        if (threadIdx.x < kSyncWords) sync[threadIdx.x] = 0u;
        // one sequence: this CTA writes the plan (read by predict_kernel); the
        // pooling CTAs below do not need it
        if (own_plan)
            plan_body(cu, batch, total_L, max_seqlen, block, ws, lay, nullptr, nullptr, 0, 1);
    }
    if ((int)blockIdx.x < npad) {
        pad_weights(pa, blockIdx.x, npad);
        return;
    }
    int nblocks;
    const int32_t* blk_prefix = reinterpret_cast<const int32_t*>(ws + lay.blk_prefix);
    if (own_plan) {
        nblocks = (total_L + block - 1) / block;
    } else {
        const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(ws + lay.hdr);
        if (!hdr->valid) return;
        nblocks = hdr->total_blocks;
    }
    // neighbouring CTAs take the column chunks of the same block, so the
    // 128 rows are read whole at about the same time (DRAM page locality)
    const int u = blockIdx.x - npad;
    const int nch = (kc * KCH + kPoolCols - 1) / kPoolCols;
    const int g = u / nch;
    const int c0 = (u % nch) * kPoolCols + threadIdx.x * 8;
    if (c0 >= kc * KCH) return;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (g < nblocks && c0 < d) {
        int64_t r0, r1;
        if (own_plan) {  // one sequence of total_L rows
            r0 = (int64_t)g * block;
            r1 = min((int64_t)total_L, r0 + block);
        } else {
            const int s = last_le(blk_prefix, batch + 1, g);
            const int m = g - blk_prefix[s];
            r0 = (int64_t)cu[s] + (int64_t)m * block;
            r1 = min((int64_t)cu[s + 1], r0 + block);
        }
        const uint16_t* p = x + r0 * ld_x + c0;
        int64_t r = r0;
        for (; r + 8 <= r1; r += 8, p += 8 * ld_x) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                v[u] = __ldg(reinterpret_cast<const uint4*>(p + u * ld_x));
#pragma unroll
            for (int u = 0; u < 8; ++u) add_row(acc, v[u]);
        }
        for (; r < r1; ++r, p += ld_x) add_row(acc, __ldg(reinterpret_cast<const uint4*>(p)));
        const float inv = 1.f / (float)(r1 - r0);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] *= inv;
    }
    uint4 hi, lo;
    split8(acc, hi, lo);
    const int R = g / TILE, r = g % TILE, c = c0 / KCH;
    uint8_t* im = xb + ((size_t)(R * kc + c) * 2) * IMG + img_off(r, c0 % KCH);
    *reinterpret_cast<uint4*>(im) = hi;
    *reinterpret_cast<uint4*>(im + IMG) = lo;
}

// ---------------------------------------------------------------------------
// predict_kernel
// ---------------------------------------------------------------------------
struct Maps {
    CUtensorMap w1[2];   // [d rows, >= rank columns] bf16, boxes of 64 x 64
    CUtensorMap w2[2];   // [rank rows, H dhp (padded) or H dh columns], boxes of 64 x 64
};

struct Args {
    const char* ws;
    WsLayout lay;
    int batch;
    // shapes
    int d, rank, H, dh, dhp, dc;   // dhp: dh padded to 64; dc = dhp / 64
    int rt;                        // row tiles of 128 token blocks
    int tba;                       // rt * 128
    int kc;                        // 64-column chunks of d
    int kc2;                       // 64-column chunks of rank
    int ldr;                       // rank padded to 32 (columns of the split-K partials)
    int nj, nt;                    // n tiles of the first GEMM and their width
    int zk, cps;                   // K splits of the first GEMM and chunks per split
    int np, nc, nj2;               // H * dhp, the second GEMM's unit width and units per row tile
    int pt, groups, hpg;           // block-product tiles, head groups, heads per group
    float inv_h;
    // workspace
    const uint8_t* xb;    // [rt][kc][2] images
    float* part;          // [2][zk][tba][ldr]
    uint8_t* hid;         // [2][rt][kc2][2] images
    uint8_t* qk;          // [2][rt][H][dc][2] images
    float* ppart;         // [groups][tba m][tba n] positive parts per head group
    uint32_t* sync;
    float* scores;
    uint64_t spin_limit_ns;
    int skip_cta;         // test hook: this CTA does not arrive at the first grid barrier (-1: off)
};

__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Instruction descriptor of tcgen05.mma kind::f16: D fp32, A and B bf16,
// A K-major, B K-major or MN-major (bit 16), M = 128, N = n.
__device__ __forceinline__ uint32_t idesc(int n, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn_major ? (1u << 16) : 0u) |
           ((uint32_t)(n >> 3) << 17) | ((uint32_t)(TILE >> 4) << 24);
}

__device__ __forceinline__ void umma(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t id,
                                     uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %3, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p;\n\t}\n" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(accumulate), "r"(id));
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// One 64 x 64 box of a weight tensor map at (column x, row y) into shared memory.
__device__ __forceinline__ void tma_box(uint32_t dst, const CUtensorMap* tm, int x, int y,
                                        uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// shared -> global bulk copy (bytes a multiple of 16, both addresses 16-byte aligned)
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t* r) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}

__device__ __forceinline__ bool aborted(const Smem* sm) {
    return *reinterpret_cast<const volatile int*>(&sm->abort_flag) != 0;
}

__device__ __forceinline__ void give_up(Smem* sm, uint32_t* sync) {
    *reinterpret_cast<volatile int*>(&sm->abort_flag) = 1;
    atomicExch(&sync[kSyncAbort], 1u);
}

__device__ __noinline__ bool wait_slow(uint64_t* bar, uint32_t parity, Smem* sm, uint32_t* sync,
                                       uint64_t limit_ns) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 63) == 0) {
            if (aborted(sm)) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                raise_error(LEMO_ERR_TIMEOUT);
                give_up(sm, sync);
                return false;
            }
        }
    }
}

// Wait for the phase of the given parity (false: this CTA gave up).
__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, Smem* sm, uint32_t* sync,
                                     uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_slow(bar, parity, sm, sync, limit_ns);
}

// wait() by every lane of a warp with a warp-uniform result, so that the
// warp runs its collective instructions (tcgen05.ld) together or not at all.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, Smem* sm, uint32_t* sync,
                                          uint64_t limit_ns) {
    const bool ok = wait(bar, parity, sm, sync, limit_ns);
    return __all_sync(0xffffffffu, ok);
}

// Bounded wait for work already issued (copies, MMAs), ignoring the abort
// flag: used before the CTA exits.
__device__ __noinline__ void wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > limit_ns) {
            raise_error(LEMO_ERR_TIMEOUT);
            return;
        }
    }
}

// Grid-wide barrier on counter `word` (every CTA of the grid is resident: one
// per SM).  Every thread of the CTA calls it, after every phase, whether or
// not the CTA has given up (a CTA that gave up passes straight through);
// returns false once this CTA or any other gave up.
__device__ __noinline__ bool grid_sync(const Args& a, Smem* sm, int word) {
    __syncthreads();
    if (threadIdx.x == 0 && !aborted(sm)) {
        uint32_t* ctr = a.sync + word;
        const volatile uint32_t* abort_word = a.sync + kSyncAbort;
        fence_proxy_global();  // this CTA's stores -> later bulk copies of other CTAs
        if (!(word == kSyncA && (int)blockIdx.x == a.skip_cta))
            asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t n = 1;; ++n) {
            uint32_t v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
            if (v >= gridDim.x) break;
            if ((n & 15) == 0) {
                if (*abort_word) {
                    *reinterpret_cast<volatile int*>(&sm->abort_flag) = 1;
                    break;
                }
                if (globaltimer_ns() - t0 > a.spin_limit_ns) {
                    raise_error(LEMO_ERR_TIMEOUT);
                    give_up(sm, a.sync);
                    break;
                }
            }
        }
        fence_proxy_global();  // other CTAs' stores -> this CTA's bulk copies
    }
    __syncthreads();
    return !aborted(sm);
}

// ------------------------------------------------------------ phase geometry
// Every role walks the same sequence of units and chunks; these describe it.
struct UnitA {  // split-K partial of the first GEMM
    int p, R, j, z, c0, nc, n0, nt;
};
__device__ __forceinline__ UnitA unit_a(const Args& a, int u) {
    UnitA t;
    t.z = u % a.zk;
    int v = u / a.zk;
    t.j = v % a.nj;
    v /= a.nj;
    t.R = v % a.rt;
    t.p = v / a.rt;
    t.c0 = t.z * a.cps;
    t.nc = min(a.kc, t.c0 + a.cps) - t.c0;
    t.n0 = t.j * a.nt;
    t.nt = min(a.nt, a.ldr - t.n0);
    return t;
}
struct UnitC {  // nc columns (a multiple of 16, at most 256) of the second GEMM
    int p, R, j, n0, nt;
};
__device__ __forceinline__ UnitC unit_c(const Args& a, int u) {
    UnitC t;
    t.j = u % a.nj2;
    const int v = u / a.nj2;
    t.R = v % a.rt;
    t.p = v / a.rt;
    t.n0 = t.j * a.nc;
    t.nt = min(a.nc, a.np - t.n0);
    return t;
}
struct UnitD {  // lower-triangle tile (tn >= tm) of block pairs, one head group
    int tn, tm, g, h0, nh;
};
__device__ __forceinline__ UnitD unit_d(const Args& a, int u) {
    UnitD t;
    t.g = u % a.groups;
    const int idx = u / a.groups;
    int tn = 0;
    while ((tn + 1) * (tn + 2) / 2 <= idx) ++tn;
    t.tn = tn;
    t.tm = idx - tn * (tn + 1) / 2;
    t.h0 = t.g * a.hpg;
    t.nh = min(a.H, t.h0 + a.hpg) - t.h0;
    return t;
}

__device__ __forceinline__ const uint8_t* xb_img(const Args& a, int R, int c, int plane) {
    return a.xb + ((size_t)(R * a.kc + c) * 2 + plane) * IMG;
}
__device__ __forceinline__ uint8_t* hid_img(const Args& a, int p, int R, int c, int plane) {
    return a.hid + ((size_t)((p * a.rt + R) * a.kc2 + c) * 2 + plane) * IMG;
}
__device__ __forceinline__ uint8_t* qk_img(const Args& a, int p, int R, int h, int c, int plane) {
    return a.qk + ((size_t)(((p * a.rt + R) * a.H + h) * a.dc + c) * 2 + plane) * IMG;
}

// MMAs of one 64-deep K chunk of a GEMM unit: A hi / lo images at st, the
// MN-major weight boxes at st + 2 IMG (64-column groups WBOX apart).
__device__ __forceinline__ void mma_weight_chunk(uint32_t d_tmem, uint32_t st, uint32_t id,
                                                 bool first) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint64_t bd = sdesc(st + 2 * IMG + k * 2048, WBOX);
        umma(d_tmem, sdesc(st + k * 32, 16), bd, id, (!first || k > 0) ? 1u : 0u);
        umma(d_tmem, sdesc(st + IMG + k * 32, 16), bd, id, 1u);
    }
}

__global__ void __launch_bounds__(THREADS, 1)
    predict_kernel(const __grid_constant__ Maps maps, const Args a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* tiles = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Smem* sm = reinterpret_cast<Smem*>(tiles + STAGES * STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t lim = a.spin_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm->full[s], 1);
            mbar_init(&sm->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm->acc_full[b], 1);
            mbar_init(&sm->acc_empty[b], EPI_WARPS);
        }
        mbar_init(&sm->done, 1);
        sm->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int i = 0; i < 2; ++i) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.w1[i])) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.w2[i])) : "memory");
        }
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sm->tmem_base)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;

    // Nothing above reads what the pooling pass writes, so it overlaps that
    // pass's tail; from here on the pass has completed.
    pdl_entry();
    fence_proxy_global();  // the pooling pass's stores -> this kernel's bulk copies
    const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(a.ws + a.lay.hdr);
    if (!hdr->valid) {  // the same in every CTA: leave before any barrier
        tc_fence_before();
        __syncthreads();
        if (warp == 1) {
            tc_fence_after();
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                         "r"(TMEM_COLS));
        }
        return;
    }
    const int TB = hdr->total_blocks;
    const int32_t* blk_prefix = reinterpret_cast<const int32_t*>(a.ws + a.lay.blk_prefix);

    // Role state, carried across phases (producer and MMA count the same
    // stage uses; MMA and epilogue the same accumulations).
    uint32_t it = 0;      // stage uses
    uint32_t acc_it = 0;  // accumulations
    const uint32_t ring = smem_u32(tiles);
    const int q4 = warp & 3;            // TMEM lane quadrant of an epilogue warp
    const int hf = (warp - 2) >> 2;     // which half of the accumulator's columns
    const int erow = q4 * 32 + lane;    // row of the tile (TMEM lane) of this thread
    bool ok = true;

    // ================================================================ phase A
    {
        const int nunits = 2 * a.rt * a.nj * a.zk;
        if (warp == 0 && lane == 0) {
            for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                const UnitA t = unit_a(a, u);
                const int groups = (t.nt + 63) >> 6;
                for (int ci = 0; ci < t.nc && ok; ++ci, ++it) {
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    if (!(ok = wait(&sm->empty[s], ph ^ 1, sm, a.sync, lim))) break;
                    const uint32_t st = ring + s * STAGE_BYTES;
                    const int c = t.c0 + ci;
                    mbar_arrive_expect_tx(&sm->full[s], 2 * IMG + groups * WBOX);
                    bulk_load(st, xb_img(a, t.R, c, 0), IMG, &sm->full[s]);
                    bulk_load(st + IMG, xb_img(a, t.R, c, 1), IMG, &sm->full[s]);
                    for (int g = 0; g < groups; ++g)
                        tma_box(st + 2 * IMG + g * WBOX, &maps.w1[t.p], t.n0 + 64 * g, c * KCH,
                                &sm->full[s]);
                }
            }
        } else if (warp == 1 && lane == 0) {
            for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                const UnitA t = unit_a(a, u);
                const uint32_t b = acc_it & 1;
                if (!(ok = wait(&sm->acc_empty[b], ((acc_it >> 1) & 1) ^ 1, sm, a.sync, lim))) break;
                const uint32_t id = idesc(t.nt, true);
                for (int ci = 0; ci < t.nc && ok; ++ci, ++it) {
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    if (!(ok = wait(&sm->full[s], ph, sm, a.sync, lim))) break;
                    tc_fence_after();
                    mma_weight_chunk(tmem + b * ACC_COLS, ring + s * STAGE_BYTES, id, ci == 0);
                    umma_commit(&sm->empty[s]);
                }
                if (!ok) break;
                umma_commit(&sm->acc_full[b]);
                ++acc_it;
            }
        } else if (warp >= 2) {
            // epilogue: the fp32 partial of rows [128 R, +128), columns [n0, n0 + nt).
            // For the CTA's last unit of the phase the ring is idle (every load of
            // the phase was consumed by the MMAs that completed before acc_full),
            // so each thread stages its half row there and sends it with one bulk
            // copy; otherwise it stores directly.
            for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                const UnitA t = unit_a(a, u);
                const uint32_t b = acc_it & 1;
                if (!(ok = wait_warp(&sm->acc_full[b], (acc_it >> 1) & 1, sm, a.sync, lim))) break;
                tc_fence_after();
                const int half = t.nt >> 1;
                const uint32_t taddr = tmem + b * ACC_COLS + ((uint32_t)(q4 * 32) << 16) + hf * half;
                float* dst = a.part + ((size_t)(t.p * a.zk + t.z) * a.tba + t.R * TILE + erow) * a.ldr +
                             t.n0 + hf * half;
                const bool staged = u + (int)gridDim.x >= nunits;
                // row pitch nt * 4 + 16 bytes: 16-byte stores of 32 rows hit distinct banks
                uint8_t* srow = tiles + (size_t)erow * (t.nt * 4 + 16) + hf * half * 4;
                for (int c = 0; c < half; c += 16) {
                    uint32_t r[16];
                    tmem_ld16(taddr + c, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; i += 4) {
                        const uint4 v = make_uint4(r[i], r[i + 1], r[i + 2], r[i + 3]);
                        if (staged)
                            *reinterpret_cast<uint4*>(srow + (c + i) * 4) = v;
                        else
                            *reinterpret_cast<uint4*>(dst + c + i) = v;
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->acc_empty[b]);
                ++acc_it;
                if (staged) {
                    fence_proxy_smem();
                    bulk_store(dst, smem_u32(srow), (uint32_t)half * 4u);
                    bulk_commit();
                }
            }
            bulk_wait_all();  // every staged copy landed (and read the ring) before the barrier
        }
    }
    ok = grid_sync(a, sm, kSyncA);

    // ================================================================ phase B
    // hid[p][row][col] = relu(sum_z part[p][z][row][col]), as hi / lo images;
    // rows >= TB and columns >= rank are zero.  Four lanes share an item of 8
    // columns below the rank: lane j sums its quarter of z in order, then the
    // quarters are added as (q0 + q1) + (q2 + q3) - a fixed order.  The
    // chunks of padding columns past the rank take one lane each (zeros), so
    // that every item fits in one pass of the grid.
    if (ok) {
        const int cpr = a.kc2 * 8;            // 8-column chunks of a hid row
        const int lcpr = (a.rank + 7) / 8;    // chunks holding columns below the rank
        const int64_t live4 = 4LL * 2 * a.tba * lcpr;
        const int64_t lanes = live4 + 2LL * a.tba * (cpr - lcpr);
        const int zq = (a.zk + 3) / 4;
        const int64_t span = (int64_t)gridDim.x * THREADS;
        for (int64_t base = (int64_t)blockIdx.x * THREADS; base < lanes; base += span) {
            // every lane runs the loop the same number of times (the shuffles below)
            const int64_t t = base + threadIdx.x;
            const bool is_live = t < live4;  // groups of four lanes never straddle live4
            const int64_t i = t >> 2;
            const int quarter = (int)(t & 3);
            const int cj = (int)(i % lcpr);
            const int row = (int)((i / lcpr) % a.tba);
            const int p = (int)(i / ((int64_t)lcpr * a.tba));
            const int col0 = cj * 8;
            const bool live = is_live && row < TB;
            float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (live) {
                const float* src = a.part + ((size_t)p * a.zk * a.tba + row) * a.ldr + col0;
                const size_t plane = (size_t)a.tba * a.ldr;
                const int z0 = quarter * zq, z1 = min(a.zk, z0 + zq);
                for (int z = z0; z < z1; z += 8) {
                    float4 tt[16];
#pragma unroll
                    for (int uu = 0; uu < 8; ++uu)
                        if (z + uu < z1) {
                            tt[2 * uu] = *reinterpret_cast<const float4*>(src + (z + uu) * plane);
                            tt[2 * uu + 1] = *reinterpret_cast<const float4*>(src + (z + uu) * plane + 4);
                        }
#pragma unroll
                    for (int uu = 0; uu < 8; ++uu)
                        if (z + uu < z1) {
                            v[0] += tt[2 * uu].x; v[1] += tt[2 * uu].y; v[2] += tt[2 * uu].z; v[3] += tt[2 * uu].w;
                            v[4] += tt[2 * uu + 1].x; v[5] += tt[2 * uu + 1].y; v[6] += tt[2 * uu + 1].z; v[7] += tt[2 * uu + 1].w;
                        }
                }
            }
            // (q0 + q1) + (q2 + q3): the four lanes of an item are adjacent
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                v[e] += __shfl_xor_sync(0xffffffffu, v[e], 1);
                v[e] += __shfl_xor_sync(0xffffffffu, v[e], 2);
            }
            if (is_live && quarter == 0) {
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = (live && col0 + e < a.rank) ? fmaxf(v[e], 0.f) : 0.f;
                uint4 hi, lo;
                split8(v, hi, lo);
                uint8_t* im = hid_img(a, p, row / TILE, col0 / KCH, 0) + img_off(row % TILE, col0 % KCH);
                *reinterpret_cast<uint4*>(im) = hi;
                *reinterpret_cast<uint4*>(im + IMG) = lo;
            } else if (!is_live && t < lanes) {
                const int64_t dd = t - live4;
                const int dcnt = cpr - lcpr;
                const int dcol0 = (lcpr + (int)(dd % dcnt)) * 8;
                const int drow = (int)((dd / dcnt) % a.tba);
                const int dp = (int)(dd / ((int64_t)dcnt * a.tba));
                uint8_t* im = hid_img(a, dp, drow / TILE, dcol0 / KCH, 0) + img_off(drow % TILE, dcol0 % KCH);
                *reinterpret_cast<uint4*>(im) = make_uint4(0u, 0u, 0u, 0u);
                *reinterpret_cast<uint4*>(im + IMG) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
    }
    ok = grid_sync(a, sm, kSyncB);

    // ================================================================ phase C
    // Qhat / Khat: hid[p] (hi, lo) x W2[p] in units of nc columns (about one
    // unit per SM), written as hi / lo images per (row tile, head, 64-column
    // chunk of dhp); a unit's columns need not start at an image boundary.
    if (ok) {
        const int nunits = 2 * a.rt * a.nj2;
        if (warp == 0 && lane == 0) {
            for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                const UnitC t = unit_c(a, u);
                const int groups = (t.nt + 63) >> 6;
                for (int c = 0; c < a.kc2 && ok; ++c, ++it) {
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    if (!(ok = wait(&sm->empty[s], ph ^ 1, sm, a.sync, lim))) break;
                    const uint32_t st = ring + s * STAGE_BYTES;
                    mbar_arrive_expect_tx(&sm->full[s], 2 * IMG + groups * WBOX);
                    bulk_load(st, hid_img(a, t.p, t.R, c, 0), IMG, &sm->full[s]);
                    bulk_load(st + IMG, hid_img(a, t.p, t.R, c, 1), IMG, &sm->full[s]);
                    for (int g = 0; g < groups; ++g)
                        tma_box(st + 2 * IMG + g * WBOX, &maps.w2[t.p], t.n0 + 64 * g, c * KCH,
                                &sm->full[s]);
                }
            }
        } else if (warp == 1 && lane == 0) {
            for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                const UnitC t = unit_c(a, u);
                const uint32_t b = acc_it & 1;
                if (!(ok = wait(&sm->acc_empty[b], ((acc_it >> 1) & 1) ^ 1, sm, a.sync, lim))) break;
                const uint32_t id = idesc(t.nt, true);
                for (int c = 0; c < a.kc2 && ok; ++c, ++it) {
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    if (!(ok = wait(&sm->full[s], ph, sm, a.sync, lim))) break;
                    tc_fence_after();
                    mma_weight_chunk(tmem + b * ACC_COLS, ring + s * STAGE_BYTES, id, c == 0);
                    umma_commit(&sm->empty[s]);
                }
                if (!ok) break;
                umma_commit(&sm->acc_full[b]);
                ++acc_it;
            }
        } else if (warp >= 2) {
            // The unit's 8-column chunks are split between the two warp
            // groups; each thread loads four chunks of its row at a time.
            for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                const UnitC t = unit_c(a, u);
                const uint32_t b = acc_it & 1;
                if (!(ok = wait_warp(&sm->acc_full[b], (acc_it >> 1) & 1, sm, a.sync, lim))) break;
                tc_fence_after();
                const int nch = t.nt >> 3, mine = nch >> 1, ch0 = hf * mine;
                const uint32_t taddr = tmem + b * ACC_COLS + ((uint32_t)(q4 * 32) << 16) + ch0 * 8;
                for (int c = 0; c < mine; c += 4) {
                    uint32_t r[32];
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (c + q < mine) tmem_ld8(taddr + (c + q) * 8, &r[8 * q]);
                    tmem_wait_ld();
                    if (c + 4 >= mine) {  // every read of the accumulator landed: free it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm->acc_empty[b]);
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (c + q >= mine) break;
                        const int n = t.n0 + (ch0 + c + q) * 8;  // padded column (multiple of 8)
                        const int h = n / a.dhp, e = n - h * a.dhp;
                        float v[8];
#pragma unroll
                        for (int e8 = 0; e8 < 8; ++e8) v[e8] = __uint_as_float(r[8 * q + e8]);
                        uint4 hi, lo;
                        split8(v, hi, lo);
                        uint8_t* im = qk_img(a, t.p, t.R, h, e / KCH, 0) + img_off(erow, e % KCH);
                        *reinterpret_cast<uint4*>(im) = hi;
                        *reinterpret_cast<uint4*>(im + IMG) = lo;
                    }
                }
                ++acc_it;
            }
        }
    }
    ok = grid_sync(a, sm, kSyncC);

    // ================================================================ phase D
    // Block products of one lower-triangle tile (query row tile tn, key row
    // tile tm) for the heads of one group: per head 3 MMAs per K step (hi hi,
    // lo hi, hi lo), then the positive part is added into 64 running sums per
    // thread; the group's sums go to its plane of ppart.
    if (ok) {
        const int nunits = a.pt * a.groups;
        if (warp == 0 && lane == 0) {
            for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                const UnitD t = unit_d(a, u);
                for (int hh = 0; hh < t.nh && ok; ++hh)
                    for (int c = 0; c < a.dc && ok; ++c, ++it) {
                        const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                        if (!(ok = wait(&sm->empty[s], ph ^ 1, sm, a.sync, lim))) break;
                        const int h = t.h0 + hh;
                        const uint32_t st = ring + s * STAGE_BYTES;
                        mbar_arrive_expect_tx(&sm->full[s], 4 * IMG);
                        bulk_load(st, qk_img(a, 0, t.tn, h, c, 0), IMG, &sm->full[s]);
                        bulk_load(st + IMG, qk_img(a, 0, t.tn, h, c, 1), IMG, &sm->full[s]);
                        bulk_load(st + 2 * IMG, qk_img(a, 1, t.tm, h, c, 0), IMG, &sm->full[s]);
                        bulk_load(st + 3 * IMG, qk_img(a, 1, t.tm, h, c, 1), IMG, &sm->full[s]);
                    }
            }
        } else if (warp == 1 && lane == 0) {
            const uint32_t id = idesc(TILE, false);
            for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                const UnitD t = unit_d(a, u);
                for (int hh = 0; hh < t.nh && ok; ++hh) {
                    const uint32_t b = acc_it & 1;
                    if (!(ok = wait(&sm->acc_empty[b], ((acc_it >> 1) & 1) ^ 1, sm, a.sync, lim))) break;
                    for (int c = 0; c < a.dc && ok; ++c, ++it) {
                        const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                        if (!(ok = wait(&sm->full[s], ph, sm, a.sync, lim))) break;
                        tc_fence_after();
                        const uint32_t st = ring + s * STAGE_BYTES;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint64_t ah = sdesc(st + k * 32, 16), al = sdesc(st + IMG + k * 32, 16);
                            const uint64_t bh = sdesc(st + 2 * IMG + k * 32, 16);
                            const uint64_t bl = sdesc(st + 3 * IMG + k * 32, 16);
                            umma(tmem + b * ACC_COLS, ah, bh, id, (c > 0 || k > 0) ? 1u : 0u);
                            umma(tmem + b * ACC_COLS, al, bh, id, 1u);
                            umma(tmem + b * ACC_COLS, ah, bl, id, 1u);
                        }
                        umma_commit(&sm->empty[s]);
                    }
                    if (!ok) break;
                    umma_commit(&sm->acc_full[b]);
                    ++acc_it;
                }
            }
        } else if (warp >= 2) {
            for (int u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
                const UnitD t = unit_d(a, u);
                float tot[64];
#pragma unroll
                for (int i = 0; i < 64; ++i) tot[i] = 0.f;
                for (int hh = 0; hh < t.nh; ++hh) {
                    const uint32_t b = acc_it & 1;
                    if (!(ok = wait_warp(&sm->acc_full[b], (acc_it >> 1) & 1, sm, a.sync, lim))) break;
                    tc_fence_after();
                    const uint32_t taddr = tmem + b * ACC_COLS + ((uint32_t)(q4 * 32) << 16) + hf * 64;
                    uint32_t r[64];
                    tmem_ld16(taddr, &r[0]);
                    tmem_ld16(taddr + 16, &r[16]);
                    tmem_ld16(taddr + 32, &r[32]);
                    tmem_ld16(taddr + 48, &r[48]);
                    tmem_wait_ld();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm->acc_empty[b]);
                    ++acc_it;
#pragma unroll
                    for (int i = 0; i < 64; ++i) tot[i] += fmaxf(__uint_as_float(r[i]), 0.f);
                }
                if (!ok) break;
                // ppart[g][m][n]: the lanes of a warp hold consecutive n, so each
                // store of the 64 columns m is one coalesced 128-byte row
                const int n = t.tn * TILE + erow;
                float* col = a.ppart + ((size_t)t.g * a.tba + t.tm * TILE + hf * 64) * a.tba + n;
#pragma unroll
                for (int i = 0; i < 64; ++i) col[(size_t)i * a.tba] = tot[i];
            }
        }
    }
    ok = grid_sync(a, sm, kSyncD);

    // ================================================================ phase E
    // score[m] = sum_{n = m}^{end of m's sequence} P[n][m] with
    // P[n][m] = (1/H) sum_g ppart[g][m][n].  One CTA per pair of block
    // columns m1 = cp and m2 = TB-1-cp (so every CTA adds about TB + 1
    // values): the rows of m1 then those of m2 are dealt to the threads in
    // order, each thread adds the head groups of its rows in order into its
    // share of either column, and the shares are combined by a fixed butterfly
    // per warp and the ten warp sums in warp order.
    if (ok) {
        const size_t plane = (size_t)a.tba * a.tba;
        const int ncols2 = (TB + 1) / 2;
        for (int cp = blockIdx.x; cp < ncols2; cp += gridDim.x) {
            const int m1 = cp, m2 = TB - 1 - cp;
            const int e1 = blk_prefix[last_le(blk_prefix, a.batch + 1, m1) + 1];
            const int e2 = blk_prefix[last_le(blk_prefix, a.batch + 1, m2) + 1];
            const int c1 = e1 - m1, c2 = m2 != m1 ? e2 - m2 : 0;
            float s1 = 0.f, s2 = 0.f;
            for (int idx = threadIdx.x; idx < c1 + c2; idx += THREADS) {
                const bool first = idx < c1;
                const int m = first ? m1 : m2;
                const int n = first ? m1 + idx : m2 + idx - c1;
                const float* src = a.ppart + (size_t)m * a.tba + n;
                float v = 0.f;
                for (int g = 0; g < a.groups; g += 32) {
                    float t[32];
#pragma unroll
                    for (int uu = 0; uu < 32; ++uu)
                        if (g + uu < a.groups) t[uu] = src[(g + uu) * plane];
#pragma unroll
                    for (int uu = 0; uu < 32; ++uu)
                        if (g + uu < a.groups) v += t[uu];
                }
                if (first) s1 += v * a.inv_h;
                else s2 += v * a.inv_h;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                s1 += __shfl_xor_sync(0xffffffffu, s1, o);
                s2 += __shfl_xor_sync(0xffffffffu, s2, o);
            }
            if (lane == 0) {
                sm->red[warp] = s1;
                sm->red2[warp] = s2;
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                float t1 = 0.f, t2 = 0.f;
                for (int w = 0; w < THREADS / 32; ++w) {
                    t1 += sm->red[w];
                    t2 += sm->red2[w];
                }
                a.scores[m1] = t1;
                if (m2 != m1) a.scores[m2] = t2;
            }
            __syncthreads();
        }
    }

    // ---------------------------------------------------------------- teardown
    // Every MMA this CTA issued completes before its tensor memory is freed;
    // every bulk copy completes before the CTA exits.
    if (warp == 1 && lane == 0) {
        umma_commit(&sm->done);
        wait_drain(&sm->done, 0, lim);
    }
    if (warp == 0 && lane == 0 && aborted(sm)) {
        const uint32_t first = it > STAGES ? it - STAGES : 0;
        for (uint32_t j = first; j < it; ++j) wait_drain(&sm->full[j % STAGES], (j / STAGES) & 1, lim);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS));
    }
}

}  // namespace predict
}  // namespace lemo
