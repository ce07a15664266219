// gemm.cuh - the tensor-core GEMMs of segment-based peak cutting (Jenga
// summary section 4.2.3, "Segment-based Peak Cutting").
//
// For one segment of S tokens the loss needs three products:
//
//   z  = h_seg W^T    [S, V] fp32    A = h_seg (K-major), B = W (K-major)
//   dh = dz W         [S, d] bf16    A = dz    (K-major), B = W (MN-major)
//   dW += dz^T h_seg  [V, d] fp32    A = dz^T  (MN-major), B = h_seg (MN-major)
//
// One persistent, warp-specialised kernel computes C = A B for one of them:
// clusters of two CTAs on neighbouring SMs take 256 x 256 output tiles with
// 2-SM tensor-core instructions (tcgen05.mma.cta_group::2, M = 256, N = 256,
// K = 16, bf16 operands, fp32 accumulation in tensor memory).  CTA r of a pair
// holds rows [128 r, +128) of the tile's A and columns [128 r, +128) of its
// B in shared memory and receives its 128 rows x 256 columns of the result
// in its own tensor memory.
//
//   warp 0 (both CTAs)  TMA: A and B slices of 64 K-elements per stage
//                       (128-byte swizzle, no multicast) into a 5-stage ring
//                       of 32 KB; completion is signalled on the leader's
//                       barrier.  K-major operands come as one box of 64 x 128,
//                       MN-major ones as two boxes of 64 (MN) x 64 (K) rows.
//   warp 1 (leader)     MMA issue into one of two 256-column accumulators, so
//                       the epilogue of a tile overlaps the MMAs of the next;
//                       commits are multicast to both CTAs.
//   warps 2-9           epilogue: tcgen05.ld of 128 rows x 256 columns (two
//                       warps per TMEM lane quadrant, 128 columns each); each
//                       warp stages 32 rows x 128 bytes at a time in its own
//                       double buffer (128-byte swizzle) and hands it to a TMA
//                       store (fp32 logits, bf16 dh rounded to nearest even)
//                       or a TMA reduce-add (dW += ..., the fp32 additions
//                       done at L2, one per element per launch, so the result
//                       does not depend on timing).  Rows and columns past the
//                       output are clipped by the TMA unit.
//
// Tiles are taken round-robin by the pairs; consecutive tiles share the
// operand that is read the most, so it is read from DRAM about once.  Every
// wait is bounded in time; a wait that runs out records LEMO_ERR_TIMEOUT and
// makes both CTAs of the pair drain what they issued, free their tensor
// memory and return.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "score.cuh"

namespace lemo {
namespace gemm {

using score::cluster_sync;
using score::cta_rank;
using score::map_to_rank;
using score::mbar_arrive_cluster;
using score::mbar_arrive_expect_tx;
using score::mbar_init;
using score::mbar_try_wait;
using score::smem_u32;
using score::tc_fence_after;
using score::tc_fence_before;
using score::tmem_ld16;
using score::tmem_wait_ld;
using score::umma_commit_pair;

constexpr int TM = 256;              // tile rows per pair (MMA M)
constexpr int TN = 256;              // tile columns (MMA N)
constexpr int ROWS = 128;            // A rows / B columns held by one CTA
constexpr int KB = 64;               // K elements per stage (one 128-byte swizzle row)
constexpr int STAGES = 5;
constexpr int A_BYTES = ROWS * KB * 2;   // 16 KB
constexpr int B_BYTES = ROWS * KB * 2;   // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 32 * (2 + EPI_WARPS);
constexpr int ACC_COLS = TN;
constexpr int TMEM_COLS = 2 * ACC_COLS;
constexpr int COLS_PER_THREAD = TN / 2;
constexpr int STG_BYTES = 32 * 128;          // one staging buffer: 32 rows x 128 bytes
constexpr int STG_PER_WARP = 2 * STG_BYTES;   // double buffered

enum Epi : int { kStoreF32 = 0, kStoreBF16 = 1, kAddF32 = 2 };

struct Smem {
    uint64_t full[STAGES];   // leader: both CTAs' slices of a stage landed
    uint64_t empty[STAGES];  // each CTA: the pair's MMAs are done with a stage
    uint64_t acc_full[2];    // each CTA: accumulator holds a finished tile
    uint64_t acc_empty[2];   // leader: both CTAs' epilogues drained an accumulator
    uint64_t done;           // each CTA: every MMA of the leader has completed
    uint32_t tmem_base;
    int abort_flag;
};
constexpr int SMEM_BYTES =
    STAGES * STAGE_BYTES + EPI_WARPS * STG_PER_WARP + 1024 /*align slack*/ + (int)sizeof(Smem);
static_assert(SMEM_BYTES <= 232448, "exceeds the 227 KB of shared memory per CTA");

struct Args {
    int M, N, K;
    int a_mn, b_mn;        // 1: the operand is MN-major (MN contiguous in memory)
    int epi;               // Epi (the output itself is the tensor map tm_c)
    float2* stats;         // kStoreF32 only, optional: per row and 128-column half tile the
                           // running (max, sum of 2^(u - max)) of u = C * log2(e), columns < N
    int64_t ld_stats;      // float2 elements between the rows of stats (2 * tiles_n)
    int tiles_m, tiles_n;
    int m_fastest;         // 1: consecutive tiles step along M (they share a B tile)
    uint64_t spin_limit_ns;
};

__device__ __forceinline__ void abort_pair(Smem* sm) {
    *reinterpret_cast<volatile int*>(&sm->abort_flag) = 1;
    const uint32_t peer = map_to_rank(smem_u32(&sm->abort_flag), cta_rank() ^ 1u);
    asm volatile("st.relaxed.cluster.shared::cluster.u32 [%0], %1;" ::"r"(peer), "r"(1)
                 : "memory");
}

__device__ __noinline__ bool wait_slow(uint64_t* bar, uint32_t parity, Smem* sm,
                                       uint64_t limit_ns) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 63) == 0) {
            if (*reinterpret_cast<volatile int*>(&sm->abort_flag)) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                raise_error(LEMO_ERR_TIMEOUT);
                abort_pair(sm);
                return false;
            }
        }
    }
}

__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, Smem* sm, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_slow(bar, parity, sm, limit_ns);
}

// warp-uniform result: the warp runs its tcgen05.ld together or not at all
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, Smem* sm,
                                          uint64_t limit_ns) {
    const bool ok = wait(bar, parity, sm, limit_ns);
    return __all_sync(0xffffffffu, ok);
}

// 2-D tiled TMA load into this CTA's shared memory, completion signalled on
// the barrier at cluster address bar_caddr (the leader's).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* tm, int x, int y,
                                                 uint32_t bar_caddr) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar_caddr)
        : "memory");
}

// Shared-memory descriptor of a 128-byte-swizzled operand slice: K-major
// (rows of 64 K-elements, 8-row groups 1024 bytes apart) or MN-major (rows of
// 64 MN-elements per K index, 8-row groups 1024 bytes apart, the two 64-wide
// MN groups lbo = 8 KB apart).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Instruction descriptor of tcgen05.mma kind::f16: D fp32, A and B bf16,
// M = 256, N = 256, operand majorness from the problem (bit 15 A, bit 16 B).
__device__ __forceinline__ uint32_t idesc(int a_mn, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn ? (1u << 15) : 0u) |
           (b_mn ? (1u << 16) : 0u) | ((uint32_t)(TN >> 3) << 17) | ((uint32_t)(TM >> 4) << 24);
}

__device__ __forceinline__ void umma_pair(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t id,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %3, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %4, p;\n\t}\n" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(accumulate), "r"(id));
}

__device__ __forceinline__ void tile_of(const Args& a, int64_t t, int* tm, int* tn) {
    if (a.m_fastest) {
        *tm = (int)(t % a.tiles_m);
        *tn = (int)(t / a.tiles_m);
    } else {
        *tn = (int)(t % a.tiles_n);
        *tm = (int)(t / a.tiles_n);
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&r);
}

// TMA store / reduce-add of a staged 32-row box at output (x = column, y = row).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* tm, uint32_t src, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(tm)),
        "r"(src), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* tm, uint32_t src, int x, int y) {
    asm volatile(
        "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(tm)),
        "r"(src), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the staging buffer of the group before the last may be rewritten
__device__ __forceinline__ void bulk_wait_read1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// One 128-byte row of a staging buffer: eight 16-byte chunks of row `lane`,
// chunk j at (j ^ (lane % 8)) * 16 (the 128-byte swizzle the tensor map names).
__device__ __forceinline__ void stage_row(uint32_t buf, int lane, const uint32_t* w) {
    const uint32_t row = buf + (uint32_t)lane * 128u;
#pragma unroll
    for (int j = 0; j < 8; ++j)
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + (((j ^ lane) & 7) << 4)),
                     "r"(w[4 * j]), "r"(w[4 * j + 1]), "r"(w[4 * j + 2]), "r"(w[4 * j + 3])
                     : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_c, const Args a) {
    pdl_entry();
    const int64_t total_tiles = (int64_t)a.tiles_m * a.tiles_n;
    const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    if (pair >= total_tiles) return;  // both CTAs of the pair leave together
    const int kblocks = (a.K + KB - 1) / KB;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* tiles = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* stg = tiles + STAGES * STAGE_BYTES;  // epilogue staging buffers
    Smem* sm = reinterpret_cast<Smem*>(stg + EPI_WARPS * STG_PER_WARP);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cta_rank();
    const bool leader = rank == 0;
    const uint64_t lim = a.spin_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm->full[s], 1);
            mbar_init(&sm->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm->acc_full[b], 1);
            mbar_init(&sm->acc_empty[b], 2 * EPI_WARPS);
        }
        mbar_init(&sm->done, 1);
        sm->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sm->tmem_base)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = sm->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_a)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_b)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_c)) : "memory");
            const uint32_t ring = smem_u32(tiles);
            uint32_t it = 0;
            bool ok = true;
            for (int64_t t = pair; ok && t < total_tiles; t += npairs) {
                int tm, tn;
                tile_of(a, t, &tm, &tn);
                const int arow = tm * TM + (int)rank * ROWS;  // this CTA's A rows (M)
                const int bcol = tn * TN + (int)rank * ROWS;  // this CTA's B columns (N)
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    if (!(ok = wait(&sm->empty[s], ph ^ 1, sm, lim))) break;
                    if (leader) mbar_arrive_expect_tx(&sm->full[s], 2 * STAGE_BYTES);
                    const uint32_t full_c = map_to_rank(smem_u32(&sm->full[s]), 0);
                    const uint32_t sa = ring + s * STAGE_BYTES, sb = sa + A_BYTES;
                    const int k0 = kb * KB;
                    if (a.a_mn) {
                        tma_load_2d_pair(sa, &tm_a, arow, k0, full_c);
                        tma_load_2d_pair(sa + A_BYTES / 2, &tm_a, arow + 64, k0, full_c);
                    } else {
                        tma_load_2d_pair(sa, &tm_a, k0, arow, full_c);
                    }
                    if (a.b_mn) {
                        tma_load_2d_pair(sb, &tm_b, bcol, k0, full_c);
                        tma_load_2d_pair(sb + B_BYTES / 2, &tm_b, bcol + 64, k0, full_c);
                    } else {
                        tma_load_2d_pair(sb, &tm_b, k0, bcol, full_c);
                    }
                }
            }
            if (!ok && leader) {
                const uint32_t first = it > STAGES ? it - STAGES : 0;
                for (uint32_t j = first; j < it; ++j)
                    wait(&sm->full[j % STAGES], (j / STAGES) & 1, sm, lim);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && leader) {
            const uint32_t ring = smem_u32(tiles);
            const uint32_t id = idesc(a.a_mn, a.b_mn);
            const uint32_t a_step = a.a_mn ? 2048u : 32u;  // bytes per K step of 16
            const uint32_t b_step = a.b_mn ? 2048u : 32u;
            uint32_t it = 0, acc_it = 0;
            bool ok = true;
            for (int64_t t = pair; ok && t < total_tiles; t += npairs, ++acc_it) {
                const uint32_t buf = acc_it & 1;
                if (!(ok = wait(&sm->acc_empty[buf], ((acc_it >> 1) & 1) ^ 1, sm, lim))) break;
                const uint32_t d_tmem = tmem_base + buf * ACC_COLS;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    if (!(ok = wait(&sm->full[s], ph, sm, lim))) break;
                    tc_fence_after();
                    const uint32_t sa = ring + s * STAGE_BYTES, sb = sa + A_BYTES;
#pragma unroll
                    for (int k = 0; k < KB / 16; ++k)
                        umma_pair(d_tmem, sdesc(sa + k * a_step, A_BYTES / 2),
                                  sdesc(sb + k * b_step, B_BYTES / 2), id,
                                  (kb > 0 || k > 0) ? 1u : 0u);
                    umma_commit_pair(&sm->empty[s]);
                }
                if (!ok) break;
                umma_commit_pair(&sm->acc_full[buf]);
            }
            umma_commit_pair(&sm->done);
        }
        if (lane == 0) {
            // bounded: every MMA the leader issued completes before TMEM is freed
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&sm->done, 0)) {
                if (globaltimer_ns() - t0 > lim) {
                    raise_error(LEMO_ERR_TIMEOUT);
                    break;
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int colhalf = (warp - 2) >> 2;
        const uint32_t lane_addr =
            tmem_base + ((uint32_t)(q * 32) << 16) + colhalf * COLS_PER_THREAD;
        const uint32_t my_stg = smem_u32(stg) + (uint32_t)(warp - 2) * STG_PER_WARP;
        uint32_t acc_empty_c[2];
        acc_empty_c[0] = map_to_rank(smem_u32(&sm->acc_empty[0]), 0);
        acc_empty_c[1] = map_to_rank(smem_u32(&sm->acc_empty[1]), 0);
        const bool bf16_out = a.epi == kStoreBF16;
        const int chunk = bf16_out ? 64 : 32;  // columns per staged box (128 bytes a row)
        uint32_t acc_it = 0, nst = 0;
        bool ok = true;
        for (int64_t t = pair; ok && t < total_tiles; t += npairs, ++acc_it) {
            int tm, tn;
            tile_of(a, t, &tm, &tn);
            const uint32_t buf = acc_it & 1;
            if (!(ok = wait_warp(&sm->acc_full[buf], (acc_it >> 1) & 1, sm, lim))) break;
            tc_fence_after();
            const int row0 = tm * TM + (int)rank * ROWS + q * 32;  // first output row of this warp
            const int col0 = tn * TN + colhalf * COLS_PER_THREAD;
            const uint32_t base = lane_addr + buf * ACC_COLS;
            float st_m = -__int_as_float(0x7f800000), st_s = 0.f;  // this thread's row statistics
#pragma unroll 1
            for (int ch = 0; ch < COLS_PER_THREAD; ch += chunk, ++nst) {
                uint32_t r[64];
                tmem_ld16(base + ch, &r[0]);
                tmem_ld16(base + ch + 16, &r[16]);
                if (bf16_out) {
                    tmem_ld16(base + ch + 32, &r[32]);
                    tmem_ld16(base + ch + 48, &r[48]);
                }
                tmem_wait_ld();
                if (ch + chunk == COLS_PER_THREAD) {
                    // every read of this accumulator has landed: free it
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(acc_empty_c[buf]);
                }
                if (bf16_out) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        r[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                } else if (a.stats) {
                    // online max / sum of 2^(u - max) over the columns < N of this chunk
                    constexpr float kLog2e = 1.4426950408889634f;
                    float cm = st_m;
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (col0 + ch + i < a.N) cm = fmaxf(cm, __uint_as_float(r[i]) * kLog2e);
                    if (cm > st_m) {
                        st_s *= exp2f(st_m - cm);
                        st_m = cm;
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (col0 + ch + i < a.N) st_s += exp2f(__uint_as_float(r[i]) * kLog2e - st_m);
                }
                // the staging buffer used two boxes ago has been read by its TMA
                const uint32_t sb = my_stg + (nst & 1) * STG_BYTES;
                if (lane == 0 && nst >= 2) bulk_wait_read1();
                __syncwarp();
                stage_row(sb, lane, r);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) {
                    if (a.epi == kAddF32)
                        tma_reduce_add_2d(&tm_c, sb, col0 + ch, row0);
                    else
                        tma_store_2d(&tm_c, sb, col0 + ch, row0);
                    bulk_commit();
                }
            }
            if (a.stats && !bf16_out && row0 + lane < a.M)
                a.stats[(int64_t)(row0 + lane) * a.ld_stats + 2 * tn + colhalf] = make_float2(st_m, st_s);
        }
        if (lane == 0) bulk_wait_all();  // every store landed before the CTA exits
        __syncwarp();
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(TMEM_COLS));
    }
    cluster_sync();  // no CTA leaves while its peer may still signal its barriers
}

}  // namespace gemm
}  // namespace lemo
