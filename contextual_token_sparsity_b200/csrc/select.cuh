// select.cuh - per-call plan of a packed batch, threshold compare and
// compaction of kept token ids (steps a4-a5).
#pragma once

#include "common.cuh"
#include "tile_plan.h"

namespace lemo {

// Block-wide inclusive scan of one value per thread (blockDim.x multiple of
// 32, at most 1024).  `warp_sums` is shared scratch of 32 entries.  Returns
// the inclusive prefix; *total receives the block total.  Contains
// __syncthreads(): every thread of the block must call it.
template <typename T>
__device__ __forceinline__ T block_scan_incl(T v, T* warp_sums, T* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        T n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) warp_sums[warp] = v;
    __syncthreads();
    if (warp == 0) {
        T w = lane < nwarps ? warp_sums[lane] : T(0);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            T n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += n;
        }
        warp_sums[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    if (warp > 0) v += warp_sums[warp - 1];
    *total = warp_sums[nwarps - 1];
    __syncthreads();  // warp_sums may be reused by the caller
    return v;
}

// ---------------------------------------------------------------------------
// Plan: per-sequence prefix arrays of a packed batch, device-side checks of
// cu_seqlens, and a reset of the compaction look-back state.  One CTA.
// The score-tile prefix counts the tiles of key-tile shard `shard` of
// `nshards` (1 shard: every tile).
// `zero_word` (optional) is set to 0 first, so that a compaction that gives
// up leaves K = 0 behind rather than a stale count.  `zero_blocks` (optional)
// gets its first total_blocks entries cleared (the host only knows an upper
// bound of that count).  plan_body() is the work of one CTA of any size
// (every thread calls it); plan_kernel is that CTA on its own.
// ---------------------------------------------------------------------------
__device__ __noinline__ void plan_body(const int32_t* __restrict__ cu, int batch, int total_L,
                                       int max_seqlen, int block, char* __restrict__ ws,
                                       WsLayout lay, int32_t* zero_word, float* zero_blocks,
                                       int shard, int nshards) {
    PlanHeader* hdr = reinterpret_cast<PlanHeader*>(ws + lay.hdr);
    int64_t* tile_prefix = reinterpret_cast<int64_t*>(ws + lay.tile_prefix);
    int32_t* blk_prefix = reinterpret_cast<int32_t*>(ws + lay.blk_prefix);
    int64_t* m_prefix = reinterpret_cast<int64_t*>(ws + lay.m_prefix);
    uint64_t* lookback = reinterpret_cast<uint64_t*>(ws + lay.lookback);

    __shared__ int bad;
    __shared__ int64_t sum64[32];
    __shared__ int sum32[32];
    const int tid = threadIdx.x;
    if (tid == 0) {
        bad = (cu[0] != 0 || cu[batch] != total_L) ? 1 : 0;
        if (zero_word) *zero_word = 0;  // e.g. kept_total: 0 unless compaction completes
    }
    for (int64_t i = tid; i < lay.n_lookback; i += blockDim.x) lookback[i] = 0ull;
    __syncthreads();

    int64_t carry_t = 0, carry_m = 0;
    int carry_b = 0;
    for (int base = 0; base < batch; base += blockDim.x) {
        const int s = base + tid;
        int64_t t_s = 0, m_s = 0;
        int b_s = 0;
        if (s < batch) {
            const int L = cu[s + 1] - cu[s];
            if (L < 0 || L > max_seqlen) {
                bad = 1;
            } else {
                b_s = (L + block - 1) / block;
                m_s = (int64_t)b_s * b_s;
                t_s = nshards > 1 ? lemo_plan::shard_seq_tiles(L, shard, nshards)
                                  : lemo_plan::seq_tiles(L);
            }
        }
        int64_t tot_t, tot_m;
        int tot_b;
        const int64_t it = block_scan_incl<int64_t>(t_s, sum64, &tot_t);
        const int64_t im = block_scan_incl<int64_t>(m_s, sum64, &tot_m);
        const int ib = block_scan_incl<int>(b_s, sum32, &tot_b);
        if (s < batch) {
            tile_prefix[s] = carry_t + it - t_s;
            m_prefix[s] = carry_m + im - m_s;
            blk_prefix[s] = carry_b + ib - b_s;
        }
        carry_t += tot_t;
        carry_m += tot_m;
        carry_b += tot_b;
    }
    __syncthreads();
    if (zero_blocks && !bad)
        for (int i = tid; i < carry_b; i += blockDim.x) zero_blocks[i] = 0.f;
    if (tid == 0) {
        tile_prefix[batch] = carry_t;
        m_prefix[batch] = carry_m;
        blk_prefix[batch] = carry_b;
        if (carry_m > lay.m_cap) bad = 1;
        hdr->valid = bad ? 0 : 1;
        hdr->total_blocks = bad ? 0 : carry_b;
        hdr->total_tiles = bad ? 0 : carry_t;
        hdr->total_m = carry_m;
        hdr->select_ticket = 0;
        if (bad) raise_error(LEMO_ERR_INVALID_ARG);
    }
}

__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ cu, int batch,
                                                    int total_L, int max_seqlen, int block,
                                                    char* __restrict__ ws, WsLayout lay,
                                                    int32_t* zero_word, float* zero_blocks,
                                                    int shard, int nshards) {
    pdl_entry();
    plan_body(cu, batch, total_L, max_seqlen, block, ws, lay, zero_word, zero_blocks, shard,
              nshards);
}

// ---------------------------------------------------------------------------
// Threshold compare + compaction with a decoupled look-back scan.
// ---------------------------------------------------------------------------
struct SelectArgs {
    const int32_t* cu;
    int batch;
    int total_L;
    int block;
    const float* scores;
    float theta;
    uint8_t* mask;
    int32_t* kept_idx;
    int32_t* cu_kept;
    int32_t* kept_total;
    char* ws;
    WsLayout lay;
    int skip_publish_tile;  // test hook, -1 = off
    uint64_t spin_limit_ns;
};

// Descriptor word of one compaction tile: bits 63..62 = state, 61..0 = value.
constexpr uint64_t kLbEmpty = 0ull, kLbAggregate = 1ull, kLbInclusive = 2ull, kLbError = 3ull;
constexpr uint64_t kLbValueMask = (1ull << 62) - 1;

__device__ __forceinline__ void lb_publish(uint64_t* p, uint64_t state, uint64_t value) {
    const uint64_t w = (state << 62) | (value & kLbValueMask);
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}

__device__ __forceinline__ uint64_t lb_read(const uint64_t* p) {
    uint64_t w;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
    return w;
}

__global__ void __launch_bounds__(kSelectThreads) select_kernel(SelectArgs a) {
    pdl_entry();
    PlanHeader* hdr = reinterpret_cast<PlanHeader*>(a.ws + a.lay.hdr);
    const int32_t* blk_prefix = reinterpret_cast<const int32_t*>(a.ws + a.lay.blk_prefix);
    uint64_t* lookback = reinterpret_cast<uint64_t*>(a.ws + a.lay.lookback);

    __shared__ int s_tile;
    __shared__ int s_cnt[kSelectItems * (kSelectThreads / 32)];
    __shared__ int s_excl;
    __shared__ int s_abort;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int kWarps = kSelectThreads / 32;
    if (!*reinterpret_cast<volatile int32_t*>(&hdr->valid)) return;
    if (tid == 0) {
        s_tile = atomicAdd(&hdr->select_ticket, 1);
        s_abort = 0;
    }
    __syncthreads();
    const int tile = s_tile;
    const int64_t base = (int64_t)tile * kSelectTile;

    // Keep bit of each item (token base + i*256 + tid), ballots per warp.
    unsigned keep_bits = 0;
    int rank[kSelectItems];
#pragma unroll
    for (int i = 0; i < kSelectItems; ++i) {
        const int64_t t = base + (int64_t)i * kSelectThreads + tid;
        bool keep = false;
        if (t < a.total_L) {
            const int s = last_le(a.cu, a.batch + 1, (int)t);
            const int local = (int)t - a.cu[s];
            const int g = blk_prefix[s] + local / a.block;
            keep = a.scores[g] >= a.theta;  // false for NaN
            if (local % a.block == 0) a.mask[g] = keep ? 1 : 0;
        }
        const unsigned bal = __ballot_sync(0xffffffffu, keep);
        rank[i] = __popc(bal & ((1u << lane) - 1u));
        if (lane == 0) s_cnt[i * kWarps + warp] = __popc(bal);
        keep_bits |= (keep ? 1u : 0u) << i;
    }
    __syncthreads();

    // Exclusive scan of the 64 (item, warp) counts in token order, by warp 0.
    if (warp == 0) {
        static_assert(kSelectItems * kWarps == 64, "two counts per lane");
        const int c0 = s_cnt[2 * lane], c1 = s_cnt[2 * lane + 1];
        int v = c0 + c1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += n;
        }
        const int excl = v - c0 - c1;
        const int tile_total = __shfl_sync(0xffffffffu, v, 31);
        s_cnt[2 * lane] = excl;
        s_cnt[2 * lane + 1] = excl + c0;

        // Decoupled look-back (lane 0): publish this tile's aggregate, then
        // walk back over predecessors until an inclusive prefix is found.
        if (lane == 0) {
            const bool publish = tile != a.skip_publish_tile;
            uint64_t prefix = 0;
            bool aborted = false;
            if (tile == 0) {
                if (publish) lb_publish(&lookback[0], kLbInclusive, (uint64_t)tile_total);
            } else {
                if (publish) lb_publish(&lookback[tile], kLbAggregate, (uint64_t)tile_total);
                int j = tile - 1;
                uint64_t t0 = 0;
                unsigned polls = 0;
                while (j >= 0) {
                    const uint64_t w = lb_read(&lookback[j]);
                    const uint64_t st = w >> 62;
                    if (st == kLbInclusive) { prefix += w & kLbValueMask; break; }
                    if (st == kLbAggregate) { prefix += w & kLbValueMask; --j; continue; }
                    if (st == kLbError) { aborted = true; break; }
                    if (polls++ == 0) t0 = globaltimer_ns();
                    if ((polls & 63) == 0 && globaltimer_ns() - t0 > a.spin_limit_ns) {
                        raise_error(LEMO_ERR_TIMEOUT);
                        aborted = true;
                        break;
                    }
                    __nanosleep(64);
                }
                if (publish)
                    lb_publish(&lookback[tile], aborted ? kLbError : kLbInclusive,
                               prefix + (uint64_t)tile_total);
            }
            s_excl = (int)prefix;
            s_abort = aborted ? 1 : 0;
            const bool last_tile = (int64_t)(tile + 1) * kSelectTile >= a.total_L;
            if (last_tile && !aborted) {
                const int K = (int)prefix + tile_total;
                *a.kept_total = K;
                for (int s = a.batch; s >= 0 && a.cu[s] == a.total_L; --s) a.cu_kept[s] = K;
            }
        }
    }
    __syncthreads();
    if (s_abort) return;
    const int excl = s_excl;

#pragma unroll
    for (int i = 0; i < kSelectItems; ++i) {
        const int64_t t = base + (int64_t)i * kSelectThreads + tid;
        if (t >= a.total_L) break;
        const int pos = excl + s_cnt[i * kWarps + warp] + rank[i];
        if (keep_bits & (1u << i)) a.kept_idx[pos] = (int32_t)t;
        // sequences that start at token t (empty ones share the start)
        int s = last_le(a.cu, a.batch + 1, (int)t);
        for (; s >= 0 && a.cu[s] == (int)t; --s) a.cu_kept[s] = pos;
    }
}

}  // namespace lemo
