// attn.cuh - permutation-free attention over the kept tokens (Jenga summary,
// section 4.2.3 "Permutation-free Token Movement": selective load and
// in-place addition fused with the attention computation).
//
// For the kept tokens of each sequence (rows kept_idx[cu_kept[s] ..
// cu_kept[s+1]) of Q, K, V, ascending positions) the kernel computes causal
// attention among them and adds the output into the residual rows of the
// same tokens in place:
//
//   x[kept_idx[r], h*dh : (h+1)*dh] += softmax_r'(scale Q_r^h . K_r'^h) V_r'^h
//
// (or writes the output to a compact [K, H*dh] buffer).  No re-permuted copy
// of Q, K, V or of the output exists; eliminated rows are never read or
// written.
//
// Selective load with TMA: the kept set is made of whole token blocks of 64
// or 128 tokens (only a sequence's last block can be short), so every chunk
// of 64 consecutive kept rows, counted from the sequence's first kept row,
// is one contiguous run of original rows.  One 2-D box (64 columns x 64
// rows, 128-byte swizzle) per chunk and 64-column slice brings it from its
// original position; the kernel checks the run is contiguous.
//
// One CTA per (pair of consecutive query tiles of 128 kept rows, head);
// 12 warps in 3 warpgroups:
//   warp 0      TMA producer: both query tiles once, then K_0, V_0, K_1,
//               V_1, ... (key tiles of 64 kept rows, 16 KB each) through a
//               10-slot ring;
//   warps 1, 2  S issuers for query tiles 0 and 1, warps 3, 12 P V issuers
//               for query tiles 0 and 1 (one thread each; tcgen05,
//               cta_group::1, M = 128).  For key tile j:
//                 S_t(j) = Q_t K_j^T      into TMEM columns [128 t + 64 (j%2), +64)
//                 O_t += P_t(j) V_j       into TMEM columns [256 + 128 t, +dh)
//               where P_t(j) is read from TMEM (A operand) and V is the
//               MN-major shared-memory B operand.  S is double-buffered, so
//               S_t(j + 1) is computed while the softmax works on tile j;
//   warp 3      idle (it completes the first warpgroup);
//   warps 4-7   softmax group 0 (query tile 0), warps 8-11 softmax group 1
//               (query tile 1): one thread per query row (its TMEM lane).
//               A thread reads its 64 scores of S_t(j) into registers, keeps
//               an online max / sum in log2 units, and writes the bf16
//               probabilities back over the first 32 columns of the same S
//               buffer, where the P V MMA reads them.  O_t is rescaled in TMEM
//               only when the running max grows by more than 8 (2^8).  At the
//               end O_t / l is added into x.
// S_t(j + 2) overwrites P_t(j), so it is issued only after O_t += P_t(j) V_j
// has completed.  A K or V slot is released when the MMAs of both query
// tiles that read it have completed.  The rows of the last, short key tile
// past the kept set are zeroed by the producer before the tile is handed
// to the MMAs, so that 0-probability keys contribute exactly 0.
//
// Every wait is bounded in time; a wait that runs out records
// LEMO_ERR_TIMEOUT and the CTA drains what it issued, frees its tensor
// memory and returns.  No TMA load uses multicast.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include "common.cuh"
#include "score.cuh"
#include "select.cuh"

namespace lemo {
namespace attn {

using score::mbar_arrive;
using score::mbar_arrive_expect_tx;
using score::mbar_init;
using score::mbar_try_wait;
using score::smem_u32;
using score::tc_fence_after;
using score::tc_fence_before;
using score::tmem_ld16;
using score::tmem_wait_ld;

constexpr int BM = 128;          // kept query rows per query tile (MMA M, TMEM lanes)
constexpr int BN = 64;           // kept keys per key tile (MMA N of S, K of P V)
constexpr int KB = 64;           // elements per 128-byte swizzle row
constexpr int MAX_DH = 128;
constexpr int UMMA_K = 16;
constexpr int Q_SLICE = BM * KB * 2;               // 128 rows x 64 elements: 16 KB
constexpr int Q_CHUNK = 64 * KB * 2;               // one 64-row box: 8 KB
constexpr int Q_TILE = (MAX_DH / KB) * Q_SLICE;    // 32 KB
constexpr int KV_SLICE = BN * KB * 2;              // 64 rows x 64 elements: 8 KB
constexpr int KV_TILE = (MAX_DH / KB) * KV_SLICE;  // 16 KB
constexpr int SOFTMAX_WARPS = 4;                   // per group (one warpgroup)
constexpr int THREADS = 32 * 16;
constexpr int KV_SLOTS = 10;
constexpr int TMEM_COLS = 512;   // S_0 [0,128), S_1 [128,256), O_0 [256,+dh), O_1 [384,+dh)
constexpr int O_COL = 256;
constexpr float kRescaleLog2 = 8.f;  // rescale O only when the max grows by more
constexpr int HEAD_GROUP = 16;       // heads whose query-tile pairs are interleaved

// shared memory: Q_0 | Q_1 | KV ring | barriers
constexpr int OFF_Q = 0;
constexpr int OFF_KV = OFF_Q + 2 * Q_TILE;
constexpr int OFF_BAR = OFF_KV + KV_SLOTS * KV_TILE;

struct Smem {
    uint64_t q_full;
    uint64_t kv_full[KV_SLOTS];
    uint64_t kv_empty[KV_SLOTS];  // two arrivals: both query tiles' MMAs on the slot done
    uint64_t s_full[2][2];        // [tile][buffer] S_t(j) in TMEM
    uint64_t p_full[2][2];        // [tile][buffer] P_t(j) in TMEM (and O_t rescaled)
    uint64_t pv_done[2][2];       // [tile][buffer] O_t += P_t(j) V_j completed
    uint64_t vtail;               // the short last V tile has landed (producer only)
    uint64_t done[4];             // every MMA of issuer i completed
    uint32_t tmem_base;
    int abort_flag;
};
constexpr int SMEM_BYTES = OFF_BAR + (int)sizeof(Smem) + 1024 /*align slack*/;
static_assert(SMEM_BYTES <= 232448, "exceeds the 227 KB of shared memory per CTA");

// Instruction descriptors of tcgen05.mma kind::f16 (D fp32, A and B bf16,
// M = 128): S = Q K^T with both operands K-major, N = 64; O += P V with V
// MN-major (bit 16), N = dh.
__host__ __device__ constexpr uint32_t idesc(int n, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn_major ? (1u << 16) : 0u) |
           ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}
constexpr uint32_t kIdescS = idesc(BN, false);

// Work decomposition written by plan_kernel.
struct WsHeader {
    int valid;
    int total_items;  // query-tile pairs over all sequences
};
constexpr size_t kWsPrefix = 256;  // int32 [batch + 1]: query-tile pairs before sequence s

inline size_t ws_bytes(int batch) { return kWsPrefix + align_up(4 * (size_t)(batch + 1), 256); }

struct Args {
    const int32_t* kept_idx;
    const int32_t* cu_kept;     // [batch + 1]
    const int32_t* cu_seqlens;  // [batch + 1]
    int batch;
    int H;
    int dh;
    float scale_log2;           // softmax scale * log2(e)
    uint16_t* x;                // in-place target [x_rows, ld_x] (or nullptr)
    int64_t ld_x;
    int64_t x_rows;
    uint16_t* o;                // compact output [K, ld_o] (or nullptr)
    int64_t ld_o;
    const char* ws;
    uint64_t spin_limit_ns;
};

// ---------------------------------------------------------------------------
// Plan: query-tile pairs per sequence from cu_kept, their prefix, and
// checks of cu_kept against the shape (1 CTA of 1024 threads).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024)
    plan_kernel(const int32_t* __restrict__ cu_kept, const int32_t* __restrict__ kept_total,
                const int32_t* __restrict__ cu_seqlens, int batch, char* __restrict__ ws) {
    pdl_entry();
    __shared__ int sum32[32];
    __shared__ int bad;
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    int32_t* prefix = reinterpret_cast<int32_t*>(ws + kWsPrefix);
    if (threadIdx.x == 0) bad = (cu_kept[0] != 0 || cu_kept[batch] != *kept_total) ? 1 : 0;
    __syncthreads();
    int carry = 0;
    for (int base = 0; base < batch; base += 1024) {
        const int s = base + threadIdx.x;
        int nq = 0;
        if (s < batch) {
            const int k0 = cu_kept[s], k1 = cu_kept[s + 1];
            const int L = cu_seqlens[s + 1] - cu_seqlens[s];
            if (k1 < k0 || k1 - k0 > L) bad = 1;
            else nq = ((k1 - k0 + BM - 1) / BM + 1) / 2;
        }
        int tot;
        const int incl = block_scan_incl<int>(nq, sum32, &tot);
        if (s < batch) prefix[s] = carry + incl - nq;
        carry += tot;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        prefix[batch] = carry;
        hdr->total_items = carry;
        hdr->valid = bad ? 0 : 1;
        if (bad) raise_error(LEMO_ERR_INVALID_ARG);
    }
}

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void abort_cta(Smem* sm) {
    *reinterpret_cast<volatile int*>(&sm->abort_flag) = 1;
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
                abort_cta(sm);
                return false;
            }
        }
    }
}

// Wait for the phase of the given parity (false: the CTA gave up).
__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, Smem* sm, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_slow(bar, parity, sm, limit_ns);
}

// Wait for the phase of the given parity regardless of the abort flag
// (bounded in time only): used before exit, for copies and MMAs already
// issued, which always complete.
__device__ __noinline__ bool wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > limit_ns) {
            raise_error(LEMO_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// wait() by every lane of the warp, with a warp-uniform result (the warp
// then runs its collective tensor-memory instructions together or not at all).
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, Smem* sm,
                                          uint64_t limit_ns) {
    const bool ok = wait(bar, parity, sm, limit_ns);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int x, int y,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle: start address, leading
// byte offset, stride byte offset (all >> 4), version 1, layout SWIZZLE_128B.
// K-major operand: rows of 128 bytes, 8-row groups SBO = 1024 bytes apart
// (LBO unused).  MN-major operand (V): 64 contiguous elements of the N
// dimension per 128-byte row, one row per K index; 8-row groups along K are
// SBO = 1024 bytes apart and 64-element groups along N are LBO = 16 KB apart.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

__device__ __forceinline__ void umma(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc_v,
                                     uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %3, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p;\n\t}\n" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(accumulate), "r"(idesc_v));
}

// Same with the A operand in tensor memory (M rows in lanes, two 16-bit K
// elements per 32-bit column).
__device__ __forceinline__ void umma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db,
                                        uint32_t idesc_v, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %3, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, p;\n\t}\n" ::"r"(tmem_d),
        "r"(tmem_a), "l"(db), "r"(accumulate), "r"(idesc_v));
}

// Arrive once on `bar` when every MMA issued so far by this thread is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2^x with the hardware approximation (flushes subnormal results to 0;
// exact 0 for x = -inf).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed fp32 pairs (one instruction for two lanes of work) and the
// three-input maximum of sm_100.
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t v;
    asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(lo), "f"(hi));
    return v;
}
__device__ __forceinline__ void unf2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&r);
}

// TMA boxes (64 columns x 64 rows) of one run of up to 64 kept rows that
// starts at compact row c0 (rows at or beyond `end` are not loaded).  The
// run must be contiguous in the original rows and inside the sequence
// [seq0, seq1); one that is not is reported (the load stays in bounds: TMA
// fills rows outside the tensor with zeros).  Slice kc of the run goes to
// dst + kc * slice.  Returns the bytes issued.
__device__ __forceinline__ uint32_t run_bytes(int c0, int end, int kblocks) {
    return c0 < end ? (uint32_t)(kblocks * KV_SLICE) : 0u;
}

__device__ __forceinline__ void load_run(const CUtensorMap* tm, uint8_t* dst, int slice, int c0,
                                         int end, const int32_t* kept_idx, int seq0, int seq1,
                                         int col0, int kblocks, uint64_t* bar) {
    if (c0 >= end) return;
    const int valid = min(64, end - c0);
    const int row = kept_idx[c0];
    if (kept_idx[c0 + valid - 1] != row + valid - 1 || row < seq0 || row + valid > seq1)
        raise_error(LEMO_ERR_INVALID_ARG);
    for (int kc = 0; kc < kblocks; ++kc)
        tma_load_2d(dst + kc * slice, tm, col0 + kc * KB, row, bar);
}

__global__ void __launch_bounds__(THREADS, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const Args a) {
    pdl_entry();
    const WsHeader* hdr = reinterpret_cast<const WsHeader*>(a.ws);
    const int32_t* prefix = reinterpret_cast<const int32_t*>(a.ws + kWsPrefix);
    if (!hdr->valid) return;
    // Order: heads in groups of HEAD_GROUP; inside a group, query-tile pairs
    // heaviest first with the group's heads side by side.  The heavy pairs
    // still start first, and the K / V rows read at a time (one group's
    // heads) fit in L2.
    const int ti = hdr->total_items;
    const int hg = min(a.H, HEAD_GROUP);
    const int64_t per_group = (int64_t)ti * hg;
    if (ti <= 0 || (int64_t)blockIdx.x >= per_group * ((a.H + hg - 1) / hg)) return;
    const int grp = (int)(blockIdx.x / per_group);
    const int rem = (int)(blockIdx.x - grp * per_group);
    const int item = rem / hg, h = grp * hg + rem % hg;
    if (h >= a.H) return;
    const int s = last_le(prefix, a.batch + 1, item);
    const int npairs = prefix[s + 1] - prefix[s];
    const int pair = npairs - 1 - (item - prefix[s]);  // heaviest pairs first
    const int kbeg = a.cu_kept[s], kend = a.cu_kept[s + 1];
    const int seq0 = a.cu_seqlens[s], seq1 = a.cu_seqlens[s + 1];
    const int nq = (kend - kbeg + BM - 1) / BM;      // query tiles of the sequence
    const int nk = (kend - kbeg + BN - 1) / BN;      // key tiles of the sequence
    const int qa = 2 * pair;                         // query tile of group 0; group 1 has qa + 1
    const bool two = qa + 1 < nq;
    // key tiles of query tile t: those up to the end of its rows
    const int ntk[2] = {min(2 * qa + 2, nk), two ? min(2 * qa + 4, nk) : 0};
    const int nt = two ? ntk[1] : ntk[0];            // key tiles loaded for the pair
    const int kblocks = a.dh / KB;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Smem* sm = reinterpret_cast<Smem*>(base + OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&sm->q_full, 1);
        for (int i = 0; i < KV_SLOTS; ++i) {
            mbar_init(&sm->kv_full[i], 1);
            mbar_init(&sm->kv_empty[i], 2);
        }
        for (int t = 0; t < 2; ++t)
            for (int b = 0; b < 2; ++b) {
                mbar_init(&sm->s_full[t][b], 1);
                mbar_init(&sm->p_full[t][b], SOFTMAX_WARPS);
                mbar_init(&sm->pv_done[t][b], 1);
            }
        mbar_init(&sm->vtail, 1);
        for (int i = 0; i < 4; ++i) mbar_init(&sm->done[i], 1);
        sm->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
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
    const uint64_t lim = a.spin_limit_ns;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_q)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_k)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_v)) : "memory");
            const int col0 = h * a.dh;
            const int q0 = kbeg + qa * BM;
            uint32_t qbytes = 0;
            for (int r = 0; r < (two ? 4 : 2); ++r) qbytes += run_bytes(q0 + 64 * r, kend, kblocks);
            mbar_arrive_expect_tx(&sm->q_full, qbytes);
            for (int r = 0; r < (two ? 4 : 2); ++r)   // query tile r / 2, 64-row half r % 2
                load_run(&tm_q, base + OFF_Q + (r >> 1) * Q_TILE + (r & 1) * Q_CHUNK, Q_SLICE,
                         q0 + 64 * r, kend, a.kept_idx, seq0, seq1, col0, kblocks, &sm->q_full);
            // loads n = 0, 1, 2, ...: K_{n/2} (n even) or V_{n/2} (n odd)
            const int nloads = 2 * nt;
            int n = 0;
            for (; n < nloads; ++n) {
                const int slot = n % KV_SLOTS;
                if (!wait(&sm->kv_empty[slot], ((n / KV_SLOTS) & 1) ^ 1, sm, lim)) break;
                const int c0 = kbeg + (n >> 1) * BN;
                uint8_t* dst = base + OFF_KV + slot * KV_TILE;
                const int nvalid = min(BN, kend - c0);
                if ((n & 1) && nvalid < BN) {
                    // the short last V tile: land it, zero the rows past the
                    // kept set, then hand it to the MMAs
                    mbar_arrive_expect_tx(&sm->vtail, run_bytes(c0, kend, kblocks));
                    load_run(&tm_v, dst, KV_SLICE, c0, kend, a.kept_idx, seq0, seq1, col0,
                             kblocks, &sm->vtail);
                    if (!wait_drain(&sm->vtail, 0, lim)) break;
                    for (int kc = 0; kc < kblocks; ++kc) {
                        uint4* z = reinterpret_cast<uint4*>(dst + kc * KV_SLICE + nvalid * 128);
                        for (int i = 0; i < (BN - nvalid) * 8; ++i) z[i] = make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_async_smem();
                    mbar_arrive(&sm->kv_full[slot]);
                    continue;
                }
                mbar_arrive_expect_tx(&sm->kv_full[slot], run_bytes(c0, kend, kblocks));
                load_run((n & 1) ? &tm_v : &tm_k, dst, KV_SLICE, c0, kend, a.kept_idx, seq0, seq1,
                         col0, kblocks, &sm->kv_full[slot]);
            }
            if (n < nloads) {
                // gave up: every load issued lands before the CTA may exit
                wait_drain(&sm->q_full, 0, lim);
                for (int i = n > KV_SLOTS ? n - KV_SLOTS : 0; i < n; ++i)
                    wait_drain(&sm->kv_full[i % KV_SLOTS], (i / KV_SLOTS) & 1, lim);
            }
        }
    } else if ((warp == 1 || warp == 2 || warp == 3 || warp == 12) && lane == 0) {
        // ------------------------------------------------------------ MMA issuers
        // One thread per chain, waiting, issuing and committing alone.
        //   S issuer of tile t:   S(j) needs K_j loaded and, for j >= 2,
        //                         PV(j - 2) completed (it reuses that buffer);
        //   P V issuer of tile t: PV(j) needs V_j loaded and P(j) written.
        // A K slot is released by the S issuers, a V slot by the P V issuers;
        // a chain releases the other tile's share of a key tile that the
        // other tile does not read.
        const bool is_s = warp <= 2;
        const int t = (warp == 1 || warp == 3) ? 0 : 1;
        const int id = is_s ? t : 2 + t;
        const int n = ntk[t];
        const int nko = ntk[t ^ 1];
        bool ok = n > 0;
        if (ok && is_s) ok = wait(&sm->q_full, 0, sm, lim);
        const uint32_t idesc_pv = idesc(a.dh, true);
        const uint32_t sq = smem_u32(base + OFF_Q + t * Q_TILE);
        for (int j = 0; ok && j < n; ++j) {
            const int ld_no = 2 * j + (is_s ? 0 : 1);
            const int slot = ld_no % KV_SLOTS;
            if (!(ok = wait(&sm->kv_full[slot], (ld_no / KV_SLOTS) & 1, sm, lim))) break;
            const uint32_t tile = smem_u32(base + OFF_KV + slot * KV_TILE);
            const uint32_t sbuf = tmem + t * 128 + (j & 1) * BN;
            if (is_s) {
                if (j >= 2 && !(ok = wait(&sm->pv_done[t][j & 1], ((j - 2) >> 1) & 1, sm, lim)))
                    break;
                tc_fence_after();
                for (int k = 0; k < a.dh / UMMA_K; ++k) {
                    const uint32_t qo = (k >> 2) * Q_SLICE + (k & 3) * 32;
                    const uint32_t ko = (k >> 2) * KV_SLICE + (k & 3) * 32;
                    umma(sbuf, sdesc(sq + qo, 16), sdesc(tile + ko, 16), kIdescS, k > 0);
                }
                umma_commit(&sm->s_full[t][j & 1]);
            } else {
                if (!(ok = wait(&sm->p_full[t][j & 1], (j >> 1) & 1, sm, lim))) break;
                tc_fence_after();
                for (int k = 0; k < BN / UMMA_K; ++k)
                    umma_ts(tmem + O_COL + t * 128, sbuf + k * (UMMA_K / 2),
                            sdesc(tile + k * 2048, KV_SLICE), idesc_pv, (j > 0 || k > 0) ? 1u : 0u);
                umma_commit(&sm->pv_done[t][j & 1]);
            }
            umma_commit(&sm->kv_empty[slot]);
            if (j >= nko) umma_commit(&sm->kv_empty[slot]);
        }
        // every MMA completes before the tensor memory is released
        if (n > 0) {
            umma_commit(&sm->done[id]);
            wait_drain(&sm->done[id], 0, lim);
        }
    } else if (warp >= 4 && warp < 12) {
        // ------------------------------------------------------------ softmax + epilogue
        const int t = (warp - 4) / SOFTMAX_WARPS;    // query tile of this group
        const int qd = warp & 3;                     // TMEM lane quadrant of this warp
        const int row = qd * 32 + lane;              // query row of this thread in the tile
        const int qc = kbeg + (qa + t) * BM + row;   // its compact (kept) index
        const int ntt = ntk[t];                      // key tiles of this query tile
        const uint32_t lrow = tmem + ((uint32_t)(qd * 32) << 16);
        const uint32_t o_col = O_COL + t * 128;
        const float sl2 = a.scale_log2;
        float m = -CUDART_INF_F, l = 0.f;            // running max (log2 units) and sum
        bool ok = ntt > 0;
        for (int j = 0; ok && j < ntt; ++j) {
            const int b = j & 1;
            const uint32_t s_col = t * 128 + b * BN;
            if (!(ok = wait_warp(&sm->s_full[t][b], (j >> 1) & 1, sm, lim))) break;
            tc_fence_after();
            uint32_t r[BN];
            tmem_ld32(lrow + s_col, &r[0]);
            tmem_ld32(lrow + s_col + 32, &r[32]);
            tmem_wait_ld();
            // keys past the query (causal) or past the kept set are masked
            const int c0 = kbeg + j * BN;
            const int ncols = min(BN, min(kend, qc + 1) - c0);
            if (__any_sync(0xffffffffu, ncols < BN)) {
#pragma unroll
                for (int c = 0; c < BN; ++c)
                    if (c >= ncols) r[c] = __float_as_uint(-CUDART_INF_F);
            }
            // row maximum: 8 independent chains of three-input maxima, then a tree
            float mx[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mx[i] = __uint_as_float(r[i]);
#pragma unroll
            for (int c = 8; c < BN; c += 16)
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    mx[i] = max3(mx[i], __uint_as_float(r[c + i]), __uint_as_float(r[c + 8 + i]));
            const float mt =
                max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * sl2;
            bool rescale = false;
            float alpha = 1.f;
            if (j == 0) {
                m = mt;
            } else if (mt > m + kRescaleLog2) {  // lazy: otherwise p <= 2^8, harmless
                alpha = ex2(m - mt);
                m = mt;
                rescale = true;
            }
            // probabilities as bf16 pairs; exponent arguments and partial
            // sums on packed fp32 pairs (2 pair sums x 2 lanes)
            const uint64_t sc2 = f2(sl2, sl2), nm2 = f2(-m, -m);
            uint32_t pk[BN / 2];
            uint64_t ps2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
            for (int c = 0; c < BN; c += 2) {
                float x0, x1;
                unf2(fma_f32x2(f2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), sc2, nm2), x0, x1);
                const float p0 = ex2(x0), p1 = ex2(x1);
                ps2[(c >> 1) & 1] = add_f32x2(ps2[(c >> 1) & 1], f2(p0, p1));
                pk[c >> 1] = pack_bf16(p0, p1);
            }
            float a0, a1, b0, b1;
            unf2(ps2[0], a0, a1);
            unf2(ps2[1], b0, b1);
            l = l * alpha + ((a0 + a1) + (b0 + b1));
            // P_t(j) over the first 32 columns of its S buffer (S_t(j) is in
            // registers; that buffer is written again only after P V(j))
            tmem_st32(lrow + s_col, pk);
            if (__any_sync(0xffffffffu, rescale)) {
                // O_t must hold P V up to tile j - 1 before it is scaled
                if (j > 0 && !(ok = wait_warp(&sm->pv_done[t][(j - 1) & 1], ((j - 1) >> 1) & 1,
                                              sm, lim)))
                    break;
                tc_fence_after();
                for (int c = 0; c < a.dh; c += 16) {
                    uint32_t o[16];
                    tmem_ld16(lrow + o_col + c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st16(lrow + o_col + c, o);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->p_full[t][b]);
        }
        // the last P V of the tile (its commit covers every earlier MMA)
        if (ok) ok = wait_warp(&sm->pv_done[t][(ntt - 1) & 1], ((ntt - 1) >> 1) & 1, sm, lim);
        if (ok) {
            tc_fence_after();
            const float inv = 1.f / l;
            bool live = qc < kend;
            const bool add = a.x != nullptr;
            uint16_t* dst = nullptr;
            if (live) {
                if (add) {
                    const int64_t tok = a.kept_idx[qc];
                    if (tok < 0 || tok >= a.x_rows) {
                        raise_error(LEMO_ERR_INVALID_ARG);
                        live = false;
                    } else {
                        dst = a.x + tok * a.ld_x + (int64_t)h * a.dh;
                    }
                } else {
                    dst = a.o + (int64_t)qc * a.ld_o + (int64_t)h * a.dh;
                }
            }
            for (int c = 0; c < a.dh; c += 16) {
                uint32_t o[16];
                tmem_ld16(lrow + o_col + c, o);
                tmem_wait_ld();
                if (!live) continue;
                uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    float f[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(o[8 * u + i]) * inv;
                    if (add) {  // one rounding of x + O
                        const uint4 xv = d4[u];
                        const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            f[2 * i] += __uint_as_float(w[i] << 16);
                            f[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
                        }
                    }
                    d4[u] = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]),
                                       pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(TMEM_COLS));
    }
}

}  // namespace attn
}  // namespace lemo
