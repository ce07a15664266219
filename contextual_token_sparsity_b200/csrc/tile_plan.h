// tile_plan.h - lower-triangular tile enumeration of the block-scoring kernel.
//
// Pure integer logic shared by host and device code (and compiled by a host
// C++ test that checks every score block is covered exactly once).
//
// One score tile is BM = 128 query rows x BN = 256 key columns of one
// sequence, aligned to the sequence's first row.  Query tile qi covers rows
// [128 qi, 128 qi + 128); key tile kj covers columns [256 kj, 256 kj + 256).
// Causality (j < i) means key tile kj is needed by query tile qi iff
// 256 kj <= 128 qi + 127, i.e. kj <= floor(qi / 2); this also covers the
// diagonal block of every query block, so blocks without any causal pair
// (a one-token last block) still get their block score 0 written.
//
// Order inside a sequence: query tiles are taken in groups of GROUP; within a
// group key tile kj is the outer loop and the group's query tiles the inner
// one.  Tiles that run at the same time then share a few query bands and a
// few key bands, which keeps the live part of Q and K resident in L2.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define LEMO_HD __host__ __device__ __forceinline__
#else
#define LEMO_HD inline
#endif

namespace lemo_plan {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int GROUP = 16;

// sum_{q=0}^{n-1} floor(q/2) = floor(n/2) * floor((n-1)/2), n >= 0
LEMO_HD int64_t half_floor_sum(int64_t n) {
    return n <= 0 ? 0 : (n / 2) * ((n - 1) / 2);
}

// tiles of query tiles [0, n): sum_{q<n} (floor(q/2) + 1)
LEMO_HD int64_t tiles_below(int64_t n) { return half_floor_sum(n) + (n > 0 ? n : 0); }

LEMO_HD int64_t query_tiles(int64_t L) { return (L + BM - 1) / BM; }

LEMO_HD int64_t seq_tiles(int64_t L) { return tiles_below(query_tiles(L)); }

// Decode local tile index t (0 <= t < seq_tiles(L)) of a sequence of L rows.
LEMO_HD void decode_tile(int64_t L, int64_t t, int* qi_out, int* kj_out) {
    const int64_t nq = query_tiles(L);
    int64_t lo = 0;
    for (;;) {
        int64_t hi = lo + GROUP < nq ? lo + GROUP : nq;
        int64_t cnt = tiles_below(hi) - tiles_below(lo);
        if (t < cnt) {
            const int64_t w = hi - lo;
            const int64_t nfull = lo / 2 + 1;  // key tiles needed by every query tile of the group
            if (t < nfull * w) {
                *kj_out = (int)(t / w);
                *qi_out = (int)(lo + t % w);
                return;
            }
            t -= nfull * w;
            int64_t kj = nfull;
            for (;;) {
                int64_t c = hi - 2 * kj;  // query tiles qi >= 2 kj of the group
                if (t < c) {
                    *kj_out = (int)kj;
                    *qi_out = (int)(2 * kj + t);
                    return;
                }
                t -= c;
                ++kj;
            }
        }
        t -= cnt;
        lo = hi;
    }
}

}  // namespace lemo_plan
