// score.cuh - block-wise token informativeness scores on the tensor cores
// (steps a1-a3; Jenga summary section 4.2.1, Eq. 1, Eq. 2 and Fig. 6).
//
// Persistent, warp-specialised sm_100a kernel launched as clusters of two
// CTAs on neighbouring SMs.  Each pair computes tiles of 256 query rows x 256
// key columns of one sequence with 2-SM tensor-core instructions
// (tcgen05.mma.cta_group::2, M = 256, N = 256): CTA r holds query rows
// [128 r, 128 r + 128) and key rows [128 r, 128 r + 128) of the tile in its
// shared memory, and receives the fp32 scores of its 128 query rows x all
// 256 keys in its own tensor memory.  Per head h:
//
//   TMA (warp 0, both CTAs)  Q[rows, h, :] and K[keys, h, :] (128 rows each,
//                            one 3-D box per operand and head, 128-byte
//                            swizzle) into a 3-stage ring of whole heads;
//                            completion is signalled on the leader's barrier;
//   MMA (warp 1, leader)     S^h = Q_h K_h^T into one of two 256-column fp32
//                            accumulators per CTA, so the MMA of head h+1
//                            overlaps the read-out of head h; commits are
//                            multicast to both CTAs;
//   epilogue (8 warps)       tcgen05.ld pulls S^h into registers and folds it
//                            into the running sum 2A += S^h + |S^h| (128 fp32
//                            per thread; s + |s| is exactly 2 max(s, 0), and
//                            both adds are packed fp32x2, so no instruction
//                            runs on the half-rate min/max unit), then frees
//                            the accumulator on the leader's barrier.
//
// After the last head the epilogue applies the causal mask (j < i, rows
// inside the sequence), takes the maximum of 2A over each b x b block and
// writes M[n][m] = max * (scale / H) / 2.  Doubling every addend doubles
// every rounded partial sum, so M has the same bits as summing max(S^h, 0)
// directly.  S is never written to memory.  A second small kernel sums M's
// columns in a fixed order (deterministic).
//
// Splitting the key operand across the pair cuts the bytes each SM loads per
// head from 96 KB (one-SM 128 x 256 tile) to 64 KB, and loading a whole head
// per TMA operation halves the number of operations; together they keep the
// MMA fed.  Ten warps per CTA (not more) leave 168 registers per thread for
// the 128 running sums.  No TMA load uses multicast.
//
// One 256 x 256 x 16 MMA keeps the tensor pipe busy for ~137 cycles and the
// pipe queues only about two of them, so every cycle between the epilogue
// freeing an accumulator and the next MMA shows up as idle tensor time: the
// issuer prepares head g + 1 before it blocks, and the epilogue frees the
// accumulator as soon as its last tensor-memory load has landed (before the
// arithmetic on that chunk).  Sustained, the kernel runs at the board's power
// limit (the SM clock settles near 1.4-1.6 GHz), so fewer issued
// instructions per score element turn directly into speed.
//
// Every mbarrier wait is bounded in time; a wait that runs out records
// LEMO_ERR_TIMEOUT and makes both CTAs of the pair drain what they issued,
// free their tensor memory and return.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tile_plan.h"

namespace lemo {
namespace score {

constexpr int TM = lemo_plan::TM;  // 256 query rows per pair = MMA M
constexpr int TN = lemo_plan::TN;  // 256 key columns = MMA N
constexpr int ROWS = TM / 2;       // query rows (and key rows) per CTA
constexpr int KB = 64;             // elements per 128-byte swizzle row
constexpr int MAX_DH = 128;        // head dimensions up to this fit a stage
constexpr int UMMA_K = 16;         // K of one tcgen05.mma kind::f16
constexpr int STAGES = 3;          // one stage = one head of Q and K
constexpr int KB_BYTES = ROWS * KB * 2;          // one 64-wide slice of 128 rows: 16 KB
constexpr int A_BYTES = ROWS * MAX_DH * 2;       // 32 KB of Q per CTA per stage
constexpr int B_BYTES = ROWS * MAX_DH * 2;       // 32 KB of K per CTA per stage
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int EPI_WARPS = 8;     // two per TMEM lane quadrant
constexpr int THREADS = 32 * (2 + EPI_WARPS);
constexpr int ACC_COLS = TN;       // fp32 columns of one accumulator
constexpr int TMEM_COLS = 2 * ACC_COLS;
constexpr int COLS_PER_THREAD = TN / 2;  // 128 columns per epilogue thread

struct Smem {
    uint64_t full[STAGES];   // leader: both CTAs' slices of a stage have landed
    uint64_t empty[STAGES];  // each CTA: the pair's MMAs are done with a stage
    uint64_t acc_full[2];    // each CTA: accumulator holds a finished head
    uint64_t acc_empty[2];   // leader: both CTAs' epilogues drained an accumulator
    uint64_t done;           // each CTA: every MMA of the leader has completed
    uint64_t red_bar;        // the epilogue warps of a CTA meet here once per tile
    uint32_t tmem_base;
    int abort_flag;
    float red[2][4][4];      // [tile parity][lane quadrant][64-column slot]
};
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align slack*/ + (int)sizeof(Smem);
static_assert(SMEM_BYTES <= 232448, "exceeds the 227 KB of shared memory per CTA");

// Instruction descriptor of tcgen05.mma kind::f16: D fp32, A and B bf16, both
// K-major, N = TN, M = TM (bit layout of the PTX ISA instruction-descriptor
// table for .kind::f16).
constexpr uint32_t kIdesc = (1u << 4)              // D format: F32
                            | (1u << 7)            // A format: BF16
                            | (1u << 10)           // B format: BF16
                            | ((uint32_t)(TN >> 3) << 17)
                            | ((uint32_t)(TM >> 4) << 24);

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
    int shard, nshards;  // key-tile shard of every sequence computed here (1 shard: all)
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint32_t cta_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// shared::cluster address of the same shared variable in CTA `rank`.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
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

// Arrive on the barrier at cluster address `caddr` (possibly in the peer CTA).
// The tensor-memory reads it publishes are ordered by tcgen05.fence before
// the arrive, so no cluster-scope release fence is needed (it costs
// ~1000 cycles per arrive).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t caddr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
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

// Give up everywhere: this CTA and its peer stop at their next wait.
__device__ __forceinline__ void abort_pair(Smem* sm) {
    *reinterpret_cast<volatile int*>(&sm->abort_flag) = 1;
    const uint32_t peer = map_to_rank(smem_u32(&sm->abort_flag), cta_rank() ^ 1u);
    asm volatile("st.relaxed.cluster.shared::cluster.u32 [%0], %1;" ::"r"(peer), "r"(1)
                 : "memory");
}

// Slow path of mbar_wait: poll until the phase completes, the pair aborted
// or `limit_ns` passed.
__device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, Smem* sm,
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

// Wait for the phase with the given parity to complete (false: gave up).
// The common case - already complete - costs one try_wait and no call.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, Smem* sm,
                                          uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    return mbar_wait_slow(bar, parity, sm, limit_ns);
}

// 3-D tiled TMA load into this CTA's shared memory; completion (bytes) is
// signalled on the barrier at cluster address `bar_caddr` (the leader's).
// The tensor map views a [rows, H*dh] bf16 matrix as (64 elements, rows,
// H*dh/64 slices); one box of (64, 128, dh/64) brings one head of 128 rows as
// dh/64 consecutive 16 KB K-major tiles with 128-byte swizzle.
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* tm, int x, int y,
                                                 int z, uint32_t bar_caddr) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(bar_caddr)
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

__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t da, uint64_t db,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %3, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %4, p;\n\t}\n" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(accumulate), "r"(kIdesc));
}

// Arrive (once) on the barrier at this shared offset in both CTAs of the
// pair when every MMA issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"((uint16_t)0x3)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
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

// a0 += b0, a1 += b1 as one packed fp32x2 add (round to nearest per lane).
__device__ __forceinline__ void add_f32x2(float& a0, float& a1, float b0, float b1) {
    asm("{\n\t.reg .b64 x, y;\n\t"
        "mov.b64 x, {%0, %1};\n\t"
        "mov.b64 y, {%2, %3};\n\t"
        "add.rn.f32x2 x, x, y;\n\t"
        "mov.b64 {%0, %1}, x;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "f"(b0), "f"(b1));
}

// MMAs k = K0 .. K1-1 of one head (16 bf16 of K each): 16 bf16 (32 bytes)
// along K inside a swizzle row, every 4 steps the next 16 KB slice.
template <int K0, int K1>
__device__ __forceinline__ void issue_mmas(uint32_t d_tmem, uint64_t da, uint64_t db) {
#pragma unroll
    for (int k = K0; k < K1; ++k) {
        const uint64_t off = (uint64_t)((k >> 2) * (KB_BYTES >> 4) + (k & 3) * 2);
        umma_bf16_pair(d_tmem, da + off, db + off, k > 0 ? 1u : 0u);
    }
}

// max(a, b, c) in one three-input min/max instruction.
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
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
    // several sequences can share a prefix value (empty ones): last_le picks
    // the last, which is the one whose tiles contain t.
    c.seq = last_le(tile_prefix, a.batch + 1, t);
    c.seq_start = a.cu[c.seq];
    c.L = a.cu[c.seq + 1] - c.seq_start;
    if (a.nshards > 1)
        lemo_plan::decode_tile_shard(c.L, t - tile_prefix[c.seq], a.shard, a.nshards, &c.qi, &c.kj);
    else
        lemo_plan::decode_tile(c.L, t - tile_prefix[c.seq], &c.qi, &c.kj);
    return c;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    score_tiles_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k, const Args a) {
    pdl_entry();
    const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(a.ws + a.lay.hdr);
    const int64_t* tile_prefix = reinterpret_cast<const int64_t*>(a.ws + a.lay.tile_prefix);
    const int64_t* m_prefix = reinterpret_cast<const int64_t*>(a.ws + a.lay.m_prefix);
    const int64_t total_tiles = hdr->total_tiles;
    const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    if (pair >= total_tiles) return;  // both CTAs of the pair leave together

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* tiles = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Smem* sm = reinterpret_cast<Smem*>(tiles + STAGES * STAGE_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cta_rank();
    const bool leader = rank == 0;
    const int kblocks = a.dh / KB;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm->full[s], 1);   // the leader's expect_tx arrival (+ both CTAs' bytes)
            mbar_init(&sm->empty[s], 1);  // one multicast commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm->acc_full[b], 1);
            mbar_init(&sm->acc_empty[b], 2 * EPI_WARPS);  // epilogue warps of both CTAs
        }
        mbar_init(&sm->done, 1);
        mbar_init(&sm->red_bar, EPI_WARPS);
        sm->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {  // the same warp of both CTAs allocates the 512 TMEM columns
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sm->tmem_base)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
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
            for (int64_t t = pair; ok && t < total_tiles; t += npairs) {
                const TileCoord c = tile_coord(a, tile_prefix, t);
                const int qrow = c.seq_start + c.qi * TM + (int)rank * ROWS;
                const int krow = c.seq_start + c.kj * TN + (int)rank * ROWS;
                for (int h = 0; h < a.H; ++h, ++it) {
                    const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
                    if (!mbar_wait(&sm->empty[s], ph ^ 1, sm, a.spin_limit_ns)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = tiles + s * STAGE_BYTES;
                    if (leader) mbar_arrive_expect_tx(&sm->full[s], 2 * 2 * kblocks * KB_BYTES);
                    const uint32_t full_c = map_to_rank(smem_u32(&sm->full[s]), 0);
                    tma_load_3d_pair(sa, &tm_q, 0, qrow, h * kblocks, full_c);
                    tma_load_3d_pair(sa + A_BYTES, &tm_k, 0, krow, h * kblocks, full_c);
                }
            }
            if (!ok && leader) {
                // Drain: every load issued lands before the CTA may exit.
                const uint32_t first = it > STAGES ? it - STAGES : 0;
                for (uint32_t j = first; j < it; ++j)
                    mbar_wait(&sm->full[j % STAGES], (j / STAGES) & 1, sm, a.spin_limit_ns);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Heads are issued back to back over all tiles of the pair (the MMAs
        // need no tile coordinates).  The stage, parities and descriptors of
        // head g + 1 are computed before the thread blocks on its barriers, so
        // that once the epilogue frees the accumulator only a fence stands
        // between the wake-up and the next MMA.
        if (lane == 0 && leader) {
            const int64_t my_tiles = (total_tiles - pair + npairs - 1) / npairs;
            const uint32_t heads = (uint32_t)(my_tiles * a.H);
            const uint32_t sa0 = smem_u32(tiles);
            uint32_t s = 0, fph = 0;  // stage of head g and the parity of its full phase
            uint64_t da = sdesc_sw128(sa0), db = sdesc_sw128(sa0 + A_BYTES);
            bool ok = heads > 0 && mbar_wait(&sm->acc_empty[0], 1, sm, a.spin_limit_ns) &&
                      mbar_wait(&sm->full[0], 0, sm, a.spin_limit_ns);
            for (uint32_t g = 0; ok && g < heads; ++g) {
                const uint32_t buf = g & 1;
                const uint32_t d_tmem = tmem_base + buf * ACC_COLS;
                // head g + 1: its stage, the parities of its two waits
                const uint32_t s1 = s + 1 == STAGES ? 0 : s + 1;
                const uint32_t fph1 = s1 == 0 ? fph ^ 1 : fph;
                const uint32_t aph1 = (((g + 1) >> 1) & 1) ^ 1;
                const bool more = g + 1 < heads;
                tc_fence_after();
                if (a.dh == 128)  // head dimensions 64 and 128 are accepted
                    issue_mmas<0, 8>(d_tmem, da, db);
                else
                    issue_mmas<0, 4>(d_tmem, da, db);
                umma_commit_pair(&sm->empty[s]);       // both CTAs' stage s is free again
                umma_commit_pair(&sm->acc_full[buf]);  // both CTAs' accumulators are ready
                // everything head g + 1 needs except its barriers, before blocking on them
                const uint32_t sa1 = sa0 + s1 * STAGE_BYTES;
                da = sdesc_sw128(sa1);
                db = sdesc_sw128(sa1 + A_BYTES);
                if (more)
                    ok = mbar_wait(&sm->acc_empty[buf ^ 1], aph1, sm, a.spin_limit_ns) &&
                         mbar_wait(&sm->full[s1], fph1, sm, a.spin_limit_ns);
                s = s1;
                fph = fph1;
            }
            // Every MMA completes before either CTA releases its tensor memory.
            umma_commit_pair(&sm->done);
        }
        if (lane == 0) mbar_wait(&sm->done, 0, sm, a.spin_limit_ns);
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                // TMEM lane quadrant this warp may access
        const int colhalf = (warp - 2) >> 2;   // which 128 of the 256 columns
        const int row = q * 32 + lane;         // row of this thread within the CTA's 128
        const uint32_t lane_addr =
            tmem_base + ((uint32_t)(q * 32) << 16) + colhalf * COLS_PER_THREAD;
        const int etid = threadIdx.x - 64;     // 0 .. 32*EPI_WARPS-1
        uint32_t acc_empty_c[2];
        acc_empty_c[0] = map_to_rank(smem_u32(&sm->acc_empty[0]), 0);
        acc_empty_c[1] = map_to_rank(smem_u32(&sm->acc_empty[1]), 0);
        uint32_t acc_it = 0;
        int tile_par = 0;
        bool ok = true;
        // tile_par alternates the two `red` buffers and is the parity of the
        // red_bar phase of this tile.
        for (int64_t t = pair; ok && t < total_tiles; t += npairs, tile_par ^= 1) {
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
                    uint32_t r[32];
                    tmem_ld16(base + ch, &r[0]);
                    tmem_ld16(base + ch + 16, &r[16]);
                    tmem_wait_ld();
                    if (ch + 32 == COLS_PER_THREAD) {
                        // every read of this accumulator has landed: free it
                        // before folding the last chunk
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(acc_empty_c[buf]);
                    }
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        const float s0 = __uint_as_float(r[j]), s1 = __uint_as_float(r[j + 1]);
                        float t0 = s0, t1 = s1;
                        add_f32x2(t0, t1, fabsf(s0), fabsf(s1));  // 2 max(s, 0), exactly
                        add_f32x2(acc[ch + j], acc[ch + j + 1], t0, t1);
                    }
                }
            }
            if (!ok) break;


            // Causal mask + block maxima.  Valid entries: row i inside the
            // sequence and key column j < i (sequence-local indices).  Every
            // entry of A is >= 0, so starting the maximum at 0 also gives the
            // empty-block score 0.  Each warp covers 32 rows x 128 columns,
            // i.e. two 64-column slots.
            const int row0 = c.qi * TM + (int)rank * ROWS;  // first query row of this CTA
            const int i_loc = row0 + row;
            const int col0 = c.kj * TN + colhalf * COLS_PER_THREAD;
            const int jlim = (i_loc < c.L) ? (i_loc - col0) : 0;  // local cols < jlim are valid
            float mx[2] = {0.f, 0.f};
            if (jlim >= COLS_PER_THREAD) {  // every column of this thread's slice is valid
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    float m0 = 0.f, m1 = 0.f;
#pragma unroll
                    for (int j = g * 64; j < g * 64 + 64; j += 4) {
                        m0 = max3(m0, acc[j], acc[j + 1]);
                        m1 = max3(m1, acc[j + 2], acc[j + 3]);
                    }
                    mx[g] = fmaxf(m0, m1);
                }
            } else {
#pragma unroll
                for (int j = 0; j < COLS_PER_THREAD; ++j)
                    mx[j / 64] = fmaxf(mx[j / 64], (j < jlim) ? acc[j] : 0.f);
            }
#pragma unroll
            for (int g = 0; g < 2; ++g)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], o));
            if (lane == 0) { sm->red[tile_par][q][colhalf * 2] = mx[0]; sm->red[tile_par][q][colhalf * 2 + 1] = mx[1]; }
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
                    const int n = row0 / 64 + qb, m = c.kj * (TN / 64) + kslot;
                    if (n < nb && m <= n) M[(int64_t)n * nb + m] = v * (0.5f * a.out_scale);
                }
            } else {  // block == 128: 1 query block x 2 key blocks
                if (etid < 2) {
                    float v = 0.f;
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq)
                        v = fmaxf(v, fmaxf(sm->red[tile_par][qq][etid * 2],
                                           sm->red[tile_par][qq][etid * 2 + 1]));
                    const int n = row0 / 128, m = c.kj * (TN / 128) + etid;
                    if (n < nb && m <= n) M[(int64_t)n * nb + m] = v * (0.5f * a.out_scale);
                }
            }
        }
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

// score[g] = sum_{n = m}^{N_b - 1} M[n][m] for the token block g = (seq, m).
// One warp per token block: lane l adds rows n = m + l, m + l + 32, ... in
// increasing order, then a fixed butterfly combines the 32 partial sums, so
// the result is the same bits on every run (no float atomics).  With key-tile
// shards, blocks whose key tile belongs to another shard get 0.
__global__ void __launch_bounds__(256) column_sum_kernel(const float* __restrict__ mblk,
                                                         const char* __restrict__ ws, WsLayout lay,
                                                         int batch, float* __restrict__ scores,
                                                         int block, int shard, int nshards) {
    pdl_entry();
    const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(ws + lay.hdr);
    if (!hdr->valid) return;
    const int32_t* blk_prefix = reinterpret_cast<const int32_t*>(ws + lay.blk_prefix);
    const int64_t* m_prefix = reinterpret_cast<const int64_t*>(ws + lay.m_prefix);
    const int total = hdr->total_blocks;
    const int lane = threadIdx.x & 31;
    const int warps = (gridDim.x * blockDim.x) >> 5;
    for (int g = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; g < total; g += warps) {
        const int s = last_le(blk_prefix, batch + 1, g);
        const int m = g - blk_prefix[s];
        const int nb = blk_prefix[s + 1] - blk_prefix[s];
        if (nshards > 1 && !lemo_plan::owns_key_tile((int64_t)m * block / TN, shard, nshards)) {
            if (lane == 0) scores[g] = 0.f;
            continue;
        }
        const float* col = mblk + m_prefix[s] + m;
        // rows in batches of 4 per lane (loads in flight together), added in n order
        float sum = 0.f;
        int n = m + lane;
        for (; n + 96 < nb; n += 128) {
            float t[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) t[u] = col[(int64_t)(n + 32 * u) * nb];
#pragma unroll
            for (int u = 0; u < 4; ++u) sum += t[u];
        }
        for (; n < nb; n += 32) sum += col[(int64_t)n * nb];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) scores[g] = sum;
    }
}

}  // namespace score
}  // namespace lemo
