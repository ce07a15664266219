// score.cuh - block-wise token informativeness scores on the tensor cores
// (steps a1-a3; Jenga summary section 4.2.1, Eq. 1, Eq. 2 and Fig. 6).
//
// Persistent, warp-specialised sm_100a kernel.  For every lower-triangular
// tile of 128 query rows x 256 key columns of one sequence and every head h:
//
//   TMA (warp 0)      Q[rows, h, kb*64 : kb*64+64] and K[cols, h, ...] into a
//                     4-stage ring of 128B-swizzled shared-memory tiles;
//   MMA (warp 1)      tcgen05.mma kind::f16 (bf16 x bf16 -> fp32) builds
//                     S^h = Q_h K_h^T in one of two 128x256 fp32 accumulators
//                     in tensor memory (512 TMEM columns), so the MMA of head
//                     h+1 overlaps the read-out of head h;
//   epilogue (8 warps) tcgen05.ld pulls S^h into registers and folds it into
//                     the running sum A += max(S^h, 0) (128 fp32 per thread).
//
// After the last head the epilogue applies the causal mask (j < i, rows
// inside the sequence), takes the maximum of A over each b x b block and
// writes M[n][m] = max * scale / H.  S is never written to memory.  A second
// small kernel sums M's columns in a fixed order (deterministic).
//
// Every mbarrier wait is bounded in time; a wait that runs out records
// LEMO_ERR_TIMEOUT, makes the CTA drain what it issued, free its tensor
// memory and return.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tile_plan.h"

namespace lemo {
namespace score {

constexpr int BM = lemo_plan::BM;  // 128 query rows = MMA M
constexpr int BN = lemo_plan::BN;  // 256 key columns = MMA N
constexpr int KB = 64;             // contraction slice per stage (128 bytes of bf16)
constexpr int UMMA_K = 16;         // K of one tcgen05.mma kind::f16
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * KB * 2;  // 16 KB
constexpr int B_BYTES = BN * KB * 2;  // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 32 * (2 + EPI_WARPS);
constexpr int ACC_COLS = BN;      // fp32 columns of one accumulator
constexpr int TMEM_COLS = 2 * ACC_COLS;
constexpr int COLS_PER_THREAD = BN / 2;  // two epilogue warps per TMEM lane quadrant

struct Smem {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t done;
    uint64_t red_bar;  // the 8 epilogue warps meet here once per tile
    uint32_t tmem_base;
    int abort_flag;
    float red[2][4][4];  // [tile parity][lane quadrant][block column slot]
};
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align slack*/ + (int)sizeof(Smem);

// Instruction descriptor of tcgen05.mma kind::f16: D fp32, A and B bf16, both
// K-major, N = BN, M = BM (bit layout of the PTX ISA instruction-descriptor
// table for .kind::f16).
constexpr uint32_t kIdesc = (1u << 4)              // D format: F32
                            | (1u << 7)            // A format: BF16
                            | (1u << 10)           // B format: BF16
                            | ((uint32_t)(BN >> 3) << 17)
                            | ((uint32_t)(BM >> 4) << 24);

struct Args {
    const int32_t* cu;
    int batch;
    int H;
    int dh;
    int block;
    float out_scale;  // scale / H
    float* mblk;      // M, per-sequence [N_b, N_b]
    const char* ws;
    WsLayout lay;
    uint64_t spin_limit_ns;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete.  Gives up (and
// returns false) once another role of the CTA aborted or `limit_ns` passed.
__device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Smem* sm, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 63) == 0) {
            if (*reinterpret_cast<volatile int*>(&sm->abort_flag)) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                raise_error(LEMO_ERR_TIMEOUT);
                *reinterpret_cast<volatile int*>(&sm->abort_flag) = 1;
                return false;
            }
        }
    }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int x, int y,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Shared-memory matrix descriptor (tcgen05 format) of a K-major operand tile
// written by TMA with 128-byte swizzle: rows of 128 bytes, 8-row groups
// 1024 bytes apart.  Bits: start address >> 4 [0,14), leading byte offset
// >> 4 [16,30) (unused for swizzled K-major, set to 1), stride byte offset
// >> 4 [32,46), version 1 [46,48), layout SWIZZLE_128B = 2 [61,64).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t da, uint64_t db,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %3, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p;\n\t}\n" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(accumulate), "r"(kIdesc));
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

struct TileCoord {
    int seq;
    int qi, kj;
    int seq_start;
    int L;
};

__device__ __forceinline__ TileCoord tile_coord(const Args& a, const int64_t* tile_prefix,
                                                int64_t t) {
    TileCoord c;
    c.seq = last_le(tile_prefix, a.batch + 1, t);
    // several sequences can share a prefix value (empty ones): last_le picks
    // the last, which is the one whose tiles contain t.
    c.seq_start = a.cu[c.seq];
    c.L = a.cu[c.seq + 1] - c.seq_start;
    lemo_plan::decode_tile(c.L, t - tile_prefix[c.seq], &c.qi, &c.kj);
    return c;
}

__global__ void __launch_bounds__(THREADS, 1)
    score_tiles_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k, const Args a) {
    const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(a.ws + a.lay.hdr);
    const int64_t* tile_prefix = reinterpret_cast<const int64_t*>(a.ws + a.lay.tile_prefix);
    const int64_t* m_prefix = reinterpret_cast<const int64_t*>(a.ws + a.lay.m_prefix);
    const int64_t total_tiles = hdr->total_tiles;
    if ((int64_t)blockIdx.x >= total_tiles) return;  // whole CTA leaves together

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* tiles = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Smem* sm = reinterpret_cast<Smem*>(tiles + STAGES * STAGE_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kblocks = a.dh / KB;

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
        mbar_init(&sm->red_bar, EPI_WARPS);
        sm->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {  // whole warp allocates the 512 TMEM columns
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sm->tmem_base)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = sm->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_q))
                         : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_k))
                         : "memory");
            uint32_t it = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; ok && t < total_tiles; t += gridDim.x) {
                const TileCoord c = tile_coord(a, tile_prefix, t);
                const int qrow = c.seq_start + c.qi * BM;
                const int krow = c.seq_start + c.kj * BN;
                for (int h = 0; ok && h < a.H; ++h) {
                    for (int kb = 0; kb < kblocks; ++kb, ++it) {
                        const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                        if (!mbar_wait(&sm->empty[s], ph ^ 1, sm, a.spin_limit_ns)) {
                            ok = false;
                            break;
                        }
                        uint8_t* sa = tiles + s * STAGE_BYTES;
                        mbar_arrive_expect_tx(&sm->full[s], STAGE_BYTES);
                        const int x = h * a.dh + kb * KB;
                        tma_load_2d(sa, &tm_q, x, qrow, &sm->full[s]);
                        tma_load_2d(sa + A_BYTES, &tm_k, x, krow, &sm->full[s]);
                    }
                }
            }
            if (!ok) {
                // Drain: every load issued lands before the CTA may exit.
                const uint32_t first = it > STAGES ? it - STAGES : 0;
                for (uint32_t j = first; j < it; ++j)
                    mbar_wait(&sm->full[j % STAGES], (j / STAGES) & 1, sm, a.spin_limit_ns);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t it = 0, acc_it = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; ok && t < total_tiles; t += gridDim.x) {
                for (int h = 0; ok && h < a.H; ++h, ++acc_it) {
                    const uint32_t buf = acc_it & 1, aph = (acc_it >> 1) & 1;
                    if (!mbar_wait(&sm->acc_empty[buf], aph ^ 1, sm, a.spin_limit_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + buf * ACC_COLS;
                    for (int kb = 0; kb < kblocks; ++kb, ++it) {
                        const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                        if (!mbar_wait(&sm->full[s], ph, sm, a.spin_limit_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t sa = smem_u32(tiles + s * STAGE_BYTES);
                        const uint64_t da = sdesc_sw128(sa);
                        const uint64_t db = sdesc_sw128(sa + A_BYTES);
#pragma unroll
                        for (int k = 0; k < KB / UMMA_K; ++k) {
                            // advance 32 bytes (16 bf16) along K inside the swizzle atom
                            umma_bf16(d_tmem, da + (uint64_t)(k * 2), db + (uint64_t)(k * 2),
                                      (kb > 0 || k > 0) ? 1u : 0u);
                        }
                        umma_commit(&sm->empty[s]);  // stage free once these MMAs are done
                    }
                    if (!ok) break;
                    umma_commit(&sm->acc_full[buf]);  // accumulator ready for the epilogue
                }
            }
            // All MMAs issued by this thread complete before TMEM is released.
            umma_commit(&sm->done);
            mbar_wait(&sm->done, 0, sm, a.spin_limit_ns);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;             // TMEM lane quadrant this warp may access
        const int half = (warp - 2) >> 2;   // which 128 of the 256 columns
        const int row = q * 32 + lane;      // tile row of this thread
        const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16) + half * COLS_PER_THREAD;
        const int etid = threadIdx.x - 64;  // 0..255
        uint32_t acc_it = 0;
        int tile_par = 0;
        bool ok = true;
        // tile_par alternates the two `red` buffers and is the parity of the
        // red_bar phase of this tile.
        for (int64_t t = blockIdx.x; ok && t < total_tiles; t += gridDim.x, tile_par ^= 1) {
            const TileCoord c = tile_coord(a, tile_prefix, t);
            float acc[COLS_PER_THREAD];
#pragma unroll
            for (int j = 0; j < COLS_PER_THREAD; ++j) acc[j] = 0.f;

            for (int h = 0; h < a.H; ++h, ++acc_it) {
                const uint32_t buf = acc_it & 1, aph = (acc_it >> 1) & 1;
                if (!mbar_wait(&sm->acc_full[buf], aph, sm, a.spin_limit_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t base = lane_addr + buf * ACC_COLS;
#pragma unroll
                for (int ch = 0; ch < COLS_PER_THREAD; ch += 32) {
                    uint32_t r0[16], r1[16];
                    tmem_ld16(base + ch, r0);
                    tmem_ld16(base + ch + 16, r1);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        acc[ch + j] += fmaxf(__uint_as_float(r0[j]), 0.f);
                        acc[ch + 16 + j] += fmaxf(__uint_as_float(r1[j]), 0.f);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->acc_empty[buf]);
            }
            if (!ok) break;

            // Causal mask + block maxima.  Valid entries: row i inside the
            // sequence and key column j < i (sequence-local indices).  Every
            // entry of A is >= 0, so starting the maxima at 0 also gives the
            // empty-block score 0.
            const int i_loc = c.qi * BM + row;
            const int col0 = c.kj * BN + half * COLS_PER_THREAD;
            const int jlim = (i_loc < c.L) ? (i_loc - col0) : 0;  // local cols < jlim are valid
            float mx[2] = {0.f, 0.f};
#pragma unroll
            for (int j = 0; j < COLS_PER_THREAD; ++j) {
                const float v = (j < jlim) ? acc[j] : 0.f;
                mx[j / 64] = fmaxf(mx[j / 64], v);
            }
#pragma unroll
            for (int g = 0; g < 2; ++g) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], o));
            }
            if (lane == 0) {
                sm->red[tile_par][q][half * 2 + 0] = mx[0];
                sm->red[tile_par][q][half * 2 + 1] = mx[1];
            }
            // Meet the other epilogue warps on an mbarrier (a bounded wait,
            // unlike a named barrier, cannot hang if a warp gave up).
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->red_bar);
            if (!mbar_wait(&sm->red_bar, (uint32_t)tile_par, sm, a.spin_limit_ns)) {
                ok = false;
                break;
            }
            const int nb = (c.L + a.block - 1) / a.block;
            float* M = a.mblk + m_prefix[c.seq];
            if (a.block == 64) {
                if (etid < 8) {  // 2 query blocks x 4 key blocks of 64
                    const int qb = etid >> 2, kslot = etid & 3;
                    const float v = fmaxf(sm->red[tile_par][2 * qb][kslot],
                                          sm->red[tile_par][2 * qb + 1][kslot]);
                    const int n = c.qi * 2 + qb, m = c.kj * 4 + kslot;
                    if (n < nb && m <= n) M[(int64_t)n * nb + m] = v * a.out_scale;
                }
            } else {  // block == 128: 1 query block x 2 key blocks
                if (etid < 2) {
                    float v = 0.f;
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq)
                        v = fmaxf(v, fmaxf(sm->red[tile_par][qq][etid * 2],
                                           sm->red[tile_par][qq][etid * 2 + 1]));
                    const int n = c.qi, m = c.kj * 2 + etid;
                    if (n < nb && m <= n) M[(int64_t)n * nb + m] = v * a.out_scale;
                }
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(TMEM_COLS));
    }
}

// score[g] = sum_{n = m}^{N_b - 1} M[n][m] for the token block g = (seq, m),
// summed in increasing n (fixed order, deterministic).
__global__ void __launch_bounds__(256) column_sum_kernel(const float* __restrict__ mblk,
                                                         const char* __restrict__ ws, WsLayout lay,
                                                         int batch, float* __restrict__ scores) {
    const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(ws + lay.hdr);
    if (!hdr->valid) return;
    const int32_t* blk_prefix = reinterpret_cast<const int32_t*>(ws + lay.blk_prefix);
    const int64_t* m_prefix = reinterpret_cast<const int64_t*>(ws + lay.m_prefix);
    const int total = hdr->total_blocks;
    for (int g = blockIdx.x * blockDim.x + threadIdx.x; g < total; g += gridDim.x * blockDim.x) {
        const int s = last_le(blk_prefix, batch + 1, g);
        const int m = g - blk_prefix[s];
        const int nb = blk_prefix[s + 1] - blk_prefix[s];
        const float* col = mblk + m_prefix[s] + m;
        float sum = 0.f;
        for (int n = m; n < nb; ++n) sum += col[(int64_t)n * nb];
        scores[g] = sum;
    }
}

}  // namespace score
}  // namespace lemo
