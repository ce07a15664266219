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
// One CTA per (query tile of 128 kept rows, head); 6 warps:
//   warp 0      TMA producer: Q once, then K and V of each key tile into a
//               2-stage ring;
//   warp 1      MMA issuer (tcgen05, cta_group::1, M = 128):
//               S_j = Q K_j^T into one of two 128-column TMEM buffers, issued
//               one tile ahead so it overlaps the softmax of tile j-1;
//               O += P_j V_j into a dh-column TMEM accumulator (V is the
//               MN-major B operand: keys are the contraction dimension);
//   warps 2-5   softmax: one thread per query row (its TMEM lane), online
//               max / sum in log2 units; O is rescaled in TMEM only when the
//               running max grows by more than 8 (2^8), P is written to
//               shared memory as bf16 in the canonical 128-byte-swizzled
//               K-major layout; at the end O / l is added into x.
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

constexpr int BM = 128;          // kept query rows per CTA (MMA M, TMEM lanes)
constexpr int BN = 128;          // kept keys per key tile (MMA N of S, K of P V)
constexpr int CHUNK = 64;        // rows of one TMA box (one contiguous run)
constexpr int KB = 64;           // elements per 128-byte swizzle row
constexpr int MAX_DH = 128;
constexpr int UMMA_K = 16;
constexpr int SLICE_BYTES = BM * KB * 2;          // 128 rows x 64 elements: 16 KB
constexpr int CHUNK_BYTES = CHUNK * KB * 2;       // one box: 8 KB
constexpr int TILE_BYTES = (MAX_DH / KB) * SLICE_BYTES;  // 32 KB
constexpr int SOFTMAX_WARPS = 4;
constexpr int THREADS = 32 * (2 + SOFTMAX_WARPS);
constexpr int TMEM_COLS = 512;   // S0 [0,128), S1 [128,256), O [256, 256+dh)
constexpr int O_COL = 256;
constexpr float kRescaleLog2 = 8.f;  // rescale O only when the max grows by more

// shared memory: Q | K0 | K1 | V0 | V1 | P | barriers
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + TILE_BYTES;
constexpr int OFF_V = OFF_K + 2 * TILE_BYTES;
constexpr int OFF_P = OFF_V + 2 * TILE_BYTES;
constexpr int OFF_BAR = OFF_P + (BN / KB) * SLICE_BYTES;

struct Smem {
    uint64_t q_full;
    uint64_t k_full[2];
    uint64_t v_full[2];
    uint64_t kv_empty[2];  // MMA done with stage (both K and V)
    uint64_t s_full[2];    // S_j in TMEM buffer j % 2
    uint64_t p_full;       // P_j in shared memory (and O rescaled)
    uint64_t pv_done;      // O += P_j V_j completed
    uint64_t done;         // every MMA of the CTA completed
    uint32_t tmem_base;
    int abort_flag;
};
constexpr int SMEM_BYTES = OFF_BAR + (int)sizeof(Smem) + 1024 /*align slack*/;
static_assert(SMEM_BYTES <= 232448, "exceeds the 227 KB of shared memory per CTA");

// Instruction descriptors of tcgen05.mma kind::f16 (D fp32, A and B bf16,
// M = 128): S = Q K^T with both operands K-major, N = 128; O += P V with V
// MN-major (bit 16), N = dh.
__host__ __device__ constexpr uint32_t idesc(int n, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn_major ? (1u << 16) : 0u) |
           ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}
constexpr uint32_t kIdescS = idesc(BN, false);

// Work decomposition written by plan_kernel.
struct WsHeader {
    int valid;
    int total_items;  // query tiles over all sequences
};
constexpr size_t kWsPrefix = 256;  // int32 [batch + 1]: query tiles before sequence s

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
// Plan: query tiles per sequence from cu_kept, their prefix, and checks of
// cu_kept against the shape (1 CTA of 1024 threads).
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
            else nq = (k1 - k0 + BM - 1) / BM;
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

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&r);
}

// Issue the TMA boxes of one tile of 128 kept rows starting at compact row
// c0 (rows at or beyond `end` are not loaded); returns the bytes issued.
// Each 64-row chunk must be one contiguous run of original rows inside the
// sequence [seq0, seq1); a chunk that is not is reported (the load stays in
// bounds: TMA fills rows outside the tensor with zeros).
__device__ __forceinline__ uint32_t chunk_bytes(int c0, int end, int kblocks) {
    uint32_t n = 0;
    for (int c = 0; c < BM / CHUNK; ++c)
        if (c0 + c * CHUNK < end) n += kblocks * CHUNK_BYTES;
    return n;
}

__device__ __forceinline__ void load_tile(const CUtensorMap* tm, uint8_t* dst, int c0, int end,
                                          const int32_t* kept_idx, int seq0, int seq1, int col0,
                                          int kblocks, uint64_t* bar) {
    for (int c = 0; c < BM / CHUNK; ++c) {
        const int start = c0 + c * CHUNK;
        if (start >= end) break;
        const int valid = min(CHUNK, end - start);
        const int row = kept_idx[start];
        if (kept_idx[start + valid - 1] != row + valid - 1 || row < seq0 || row + valid > seq1)
            raise_error(LEMO_ERR_INVALID_ARG);
        for (int kc = 0; kc < kblocks; ++kc)
            tma_load_2d(dst + kc * SLICE_BYTES + c * CHUNK_BYTES, tm, col0 + kc * KB, row, bar);
    }
}

__global__ void __launch_bounds__(THREADS, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const Args a) {
    pdl_entry();
    const WsHeader* hdr = reinterpret_cast<const WsHeader*>(a.ws);
    const int32_t* prefix = reinterpret_cast<const int32_t*>(a.ws + kWsPrefix);
    if (!hdr->valid) return;
    const int item = blockIdx.x / a.H, h = blockIdx.x % a.H;
    if (item >= hdr->total_items) return;
    const int s = last_le(prefix, a.batch + 1, item);
    const int nq = prefix[s + 1] - prefix[s];
    const int qt = nq - 1 - (item - prefix[s]);  // heaviest query tiles first
    const int kbeg = a.cu_kept[s], kend = a.cu_kept[s + 1];
    const int seq0 = a.cu_seqlens[s], seq1 = a.cu_seqlens[s + 1];
    const int q0 = kbeg + qt * BM;
    const int ntiles = qt + 1;
    const int kblocks = a.dh / KB;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Smem* sm = reinterpret_cast<Smem*>(base + OFF_BAR);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&sm->q_full, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm->k_full[b], 1);
            mbar_init(&sm->v_full[b], 1);
            mbar_init(&sm->kv_empty[b], 1);
            mbar_init(&sm->s_full[b], 1);
        }
        mbar_init(&sm->p_full, SOFTMAX_WARPS);
        mbar_init(&sm->pv_done, 1);
        mbar_init(&sm->done, 1);
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
            mbar_arrive_expect_tx(&sm->q_full, chunk_bytes(q0, kend, kblocks));
            load_tile(&tm_q, base + OFF_Q, q0, kend, a.kept_idx, seq0, seq1, col0, kblocks,
                      &sm->q_full);
            int j = 0;
            for (; j < ntiles; ++j) {
                const int st = j & 1;
                if (!wait(&sm->kv_empty[st], ((j >> 1) & 1) ^ 1, sm, lim)) break;
                const int c0 = kbeg + j * BN;
                const uint32_t bytes = chunk_bytes(c0, kend, kblocks);
                mbar_arrive_expect_tx(&sm->k_full[st], bytes);
                load_tile(&tm_k, base + OFF_K + st * TILE_BYTES, c0, kend, a.kept_idx, seq0, seq1,
                          col0, kblocks, &sm->k_full[st]);
                mbar_arrive_expect_tx(&sm->v_full[st], bytes);
                load_tile(&tm_v, base + OFF_V + st * TILE_BYTES, c0, kend, a.kept_idx, seq0, seq1,
                          col0, kblocks, &sm->v_full[st]);
            }
            if (j < ntiles) {
                // gave up: every load issued lands before the CTA may exit
                wait(&sm->q_full, 0, sm, lim);
                for (int i = j > 2 ? j - 2 : 0; i < j; ++i) {
                    wait(&sm->k_full[i & 1], (i >> 1) & 1, sm, lim);
                    wait(&sm->v_full[i & 1], (i >> 1) & 1, sm, lim);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t idesc_pv = idesc(a.dh, true);
        const uint32_t sq = smem_u32(base + OFF_Q);
        bool ok = wait_warp(&sm->q_full, 0, sm, lim);
        // S_0
        if (ok) ok = wait_warp(&sm->k_full[0], 0, sm, lim);
        if (ok) {
            tc_fence_after();
            if (lane == 0) {
                const uint32_t sk = smem_u32(base + OFF_K);
                for (int k = 0; k < a.dh / UMMA_K; ++k) {
                    const uint32_t off = (k >> 2) * SLICE_BYTES + (k & 3) * 32;
                    umma(tmem, sdesc(sq + off, 16), sdesc(sk + off, 16), kIdescS, k > 0);
                }
                umma_commit(&sm->s_full[0]);
            }
            __syncwarp();
        }
        for (int j = 0; ok && j < ntiles; ++j) {
            const int st = j & 1;
            if (j + 1 < ntiles) {  // S_{j+1}, overlapping the softmax of tile j
                const int sn = (j + 1) & 1;
                if (!(ok = wait_warp(&sm->k_full[sn], ((j + 1) >> 1) & 1, sm, lim))) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t sk = smem_u32(base + OFF_K + sn * TILE_BYTES);
                    for (int k = 0; k < a.dh / UMMA_K; ++k) {
                        const uint32_t off = (k >> 2) * SLICE_BYTES + (k & 3) * 32;
                        umma(tmem + sn * BN, sdesc(sq + off, 16), sdesc(sk + off, 16), kIdescS,
                             k > 0);
                    }
                    umma_commit(&sm->s_full[sn]);
                }
                __syncwarp();
            }
            if (!(ok = wait_warp(&sm->p_full, j & 1, sm, lim))) break;
            if (!(ok = wait_warp(&sm->v_full[st], (j >> 1) & 1, sm, lim))) break;
            // rows of V past the kept set (a short last chunk) are zeroed so
            // that 0-probability keys contribute exactly 0
            uint8_t* vt = base + OFF_V + st * TILE_BYTES;
            const int c0 = kbeg + j * BN;
            const int nvalid = min(BN, kend - c0);
            if (nvalid < BN) {
                for (int kc = 0; kc < kblocks; ++kc) {
                    uint4* p = reinterpret_cast<uint4*>(vt + kc * SLICE_BYTES + nvalid * 128);
                    const int n16 = (BN - nvalid) * 8;
                    for (int i = lane; i < n16; i += 32) p[i] = make_uint4(0u, 0u, 0u, 0u);
                }
                fence_async_smem();
            }
            __syncwarp();
            tc_fence_after();
            if (lane == 0) {
                const uint32_t sp = smem_u32(base + OFF_P);
                const uint32_t sv = smem_u32(vt);
                for (int k = 0; k < BN / UMMA_K; ++k) {
                    const uint32_t offa = (k >> 2) * SLICE_BYTES + (k & 3) * 32;
                    umma(tmem + O_COL, sdesc(sp + offa, 16), sdesc(sv + k * 2048, SLICE_BYTES),
                         idesc_pv, (j > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit(&sm->kv_empty[st]);
                umma_commit(&sm->pv_done);
            }
            __syncwarp();
        }
        // every MMA completes before the tensor memory is released
        if (lane == 0) umma_commit(&sm->done);
        __syncwarp();
        wait_warp(&sm->done, 0, sm, lim);
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int qd = warp & 3;                  // TMEM lane quadrant of this warp
        const int row = qd * 32 + lane;           // query row of this thread in the tile
        const int qc = q0 + row;                  // its compact (kept) index
        const uint32_t lrow = tmem + ((uint32_t)(qd * 32) << 16);
        uint8_t* prow = base + OFF_P + row * 128; // this row of P in each 64-key slice
        const int sw = row & 7;                   // 128-byte swizzle phase of the row
        float m = -CUDART_INF_F, l = 0.f;         // running max (log2 units) and sum
        bool ok = true;
        for (int j = 0; j < ntiles; ++j) {
            if (!(ok = wait_warp(&sm->s_full[j & 1], (j >> 1) & 1, sm, lim))) break;
            tc_fence_after();
            uint32_t r[BN];
#pragma unroll
            for (int c = 0; c < BN; c += 16) tmem_ld16(lrow + (j & 1) * BN + c, &r[c]);
            tmem_wait_ld();
            // keys past the query (causal) or past the kept set are masked
            const int ncols = min(BN, min(kend, qc + 1) - (kbeg + j * BN));
            float mt = -CUDART_INF_F;
#pragma unroll
            for (int c = 0; c < BN; ++c) {
                const float v = c < ncols ? __uint_as_float(r[c]) * a.scale_log2 : -CUDART_INF_F;
                r[c] = __float_as_uint(v);
                mt = fmaxf(mt, v);
            }
            bool rescale = false;
            float alpha = 1.f;
            if (j == 0) {
                m = mt;
            } else if (mt > m + kRescaleLog2) {  // lazy: otherwise p <= 2^8, harmless
                alpha = exp2f(m - mt);
                m = mt;
                rescale = true;
            }
            float rs = 0.f;
            uint32_t pk[BN / 2];
#pragma unroll
            for (int c = 0; c < BN; c += 2) {
                const float p0 = exp2f(__uint_as_float(r[c]) - m);
                const float p1 = exp2f(__uint_as_float(r[c + 1]) - m);
                rs += p0 + p1;
                pk[c / 2] = pack_bf16(p0, p1);
            }
            l = l * alpha + rs;
            if (j > 0) {  // P buffer free and O complete up to tile j-1
                if (!(ok = wait_warp(&sm->pv_done, (j - 1) & 1, sm, lim))) break;
                tc_fence_after();
            }
            if (__any_sync(0xffffffffu, rescale)) {
                for (int c = 0; c < a.dh; c += 16) {
                    uint32_t o[16];
                    tmem_ld16(lrow + O_COL + c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st16(lrow + O_COL + c, o);
                }
                tmem_wait_st();
            }
#pragma unroll
            for (int kc = 0; kc < BN / KB; ++kc)
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint32_t* v = &pk[kc * 32 + ch * 4];
                    *reinterpret_cast<uint4*>(prow + kc * SLICE_BYTES + ((ch ^ sw) << 4)) =
                        make_uint4(v[0], v[1], v[2], v[3]);
                }
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->p_full);
        }
        if (ok) ok = wait_warp(&sm->pv_done, (ntiles - 1) & 1, sm, lim);
        if (ok) {
            tc_fence_after();
            const float inv = 1.f / l;
            bool live = qc < kend;
            const bool add = a.x != nullptr;
            uint16_t* dst = nullptr;
            if (live) {
                if (add) {
                    const int64_t t = a.kept_idx[qc];
                    if (t < 0 || t >= a.x_rows) {
                        raise_error(LEMO_ERR_INVALID_ARG);
                        live = false;
                    } else {
                        dst = a.x + t * a.ld_x + (int64_t)h * a.dh;
                    }
                } else {
                    dst = a.o + (int64_t)qc * a.ld_o + (int64_t)h * a.dh;
                }
            }
            for (int c = 0; c < a.dh; c += 16) {
                uint32_t o[16];
                tmem_ld16(lrow + O_COL + c, o);
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
