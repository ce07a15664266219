// tile_plan.h - lower-triangular tile enumeration of the block-scoring kernel.
//
// Pure integer logic shared by host and device code (and compiled by a host
// C++ test that checks every score block is covered exactly once).
//
// One score tile is TM = 256 query rows x TN = 256 key columns of one
// sequence, aligned to the sequence's first row; a pair of CTAs computes it
// (each CTA owns 128 of the query rows).  Query tile qi covers rows
// [256 qi, 256 qi + 256); key tile kj covers columns [256 kj, 256 kj + 256).
// Causality (j < i) means key tile kj is needed by query tile qi iff
// 256 kj <= 256 qi + 255, i.e. kj <= qi; this also covers the diagonal block
// of every query block, so blocks without any causal pair (a one-token last
// block) still get their block score 0 written.
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

constexpr int TM = 256;  // query rows of a tile (two CTAs x 128)
constexpr int TN = 256;  // key columns of a tile
constexpr int GROUP = 16;

LEMO_HD int64_t query_tiles(int64_t L) { return (L + TM - 1) / TM; }

// tiles of query tiles [0, n): sum_{q<n} (q + 1)
LEMO_HD int64_t tiles_below(int64_t n) { return n > 0 ? n * (n + 1) / 2 : 0; }

LEMO_HD int64_t seq_tiles(int64_t L) { return tiles_below(query_tiles(L)); }

// Decode local tile index t (0 <= t < seq_tiles(L)) of a sequence of L rows.
LEMO_HD void decode_tile(int64_t L, int64_t t, int* qi_out, int* kj_out) {
    const int64_t nq = query_tiles(L);
    int64_t lo = 0;
    for (;;) {
        const int64_t hi = lo + GROUP < nq ? lo + GROUP : nq;
        const int64_t cnt = tiles_below(hi) - tiles_below(lo);
        if (t < cnt) {
            const int64_t w = hi - lo;
            const int64_t nfull = lo + 1;  // key tiles kj <= lo are needed by the whole group
            if (t < nfull * w) {
                *kj_out = (int)(t / w);
                *qi_out = (int)(lo + t % w);
                return;
            }
            t -= nfull * w;
            for (int64_t kj = nfull;; ++kj) {
                const int64_t c = hi - kj;  // query tiles qi >= kj of the group
                if (t < c) {
                    *kj_out = (int)kj;
                    *qi_out = (int)(kj + t);
                    return;
                }
                t -= c;
            }
        }
        t -= cnt;
        lo = hi;
    }
}

// ---------------------------------------------------------------------------
// One sequence split over `nshards` shards by key tiles (columns kj): shard r
// owns the key tiles of one position in every round of nshards consecutive
// tiles, in snake order (round i gives tile i*nshards + p to shard p when i is
// even, to shard nshards-1-p when i is odd), so that the long early columns
// (key tile kj is needed by nq - kj query tiles) are spread evenly.  A shard
// computes every tile of its own columns, so the column sums of its key
// blocks are complete on that shard.  With nshards = 1 shard 0 owns all.
// ---------------------------------------------------------------------------
LEMO_HD int shard_position(int64_t round, int shard, int nshards) {
    return (round & 1) ? nshards - 1 - shard : shard;
}

LEMO_HD bool owns_key_tile(int64_t kj, int shard, int nshards) {
    return (int)(kj % nshards) == shard_position(kj / nshards, shard, nshards);
}

// key tiles kj < n owned by `shard`
LEMO_HD int64_t owned_below(int64_t n, int shard, int nshards) {
    const int64_t full = n / nshards;
    return full + ((int)(n % nshards) > shard_position(full, shard, nshards) ? 1 : 0);
}

// the j-th key tile (0-based) owned by `shard`
LEMO_HD int64_t owned_key_tile(int64_t j, int shard, int nshards) {
    return j * nshards + shard_position(j, shard, nshards);
}

// tiles of a sequence of L rows that `shard` computes: sum over its key
// tiles kj of (nq - kj)
LEMO_HD int64_t shard_seq_tiles(int64_t L, int shard, int nshards) {
    const int64_t nq = query_tiles(L);
    int64_t n = 0;
    for (int64_t j = 0;; ++j) {
        const int64_t kj = owned_key_tile(j, shard, nshards);
        if (kj >= nq) break;
        n += nq - kj;
    }
    return n;
}

// Decode local tile index t (0 <= t < shard_seq_tiles(L, shard, nshards)) of
// a shard: the same order as decode_tile (query tiles in groups of GROUP,
// key tiles outer within a group) restricted to the shard's key tiles.
LEMO_HD void decode_tile_shard(int64_t L, int64_t t, int shard, int nshards, int* qi_out,
                               int* kj_out) {
    const int64_t nq = query_tiles(L);
    int64_t lo = 0;
    for (;;) {
        const int64_t hi = lo + GROUP < nq ? lo + GROUP : nq;
        const int64_t w = hi - lo;
        const int64_t nfull = owned_below(lo + 1, shard, nshards);  // owned kj <= lo
        int64_t cnt = nfull * w;
        for (int64_t kj = lo + 1; kj < hi; ++kj)
            if (owns_key_tile(kj, shard, nshards)) cnt += hi - kj;
        if (t < cnt) {
            if (t < nfull * w) {
                *kj_out = (int)owned_key_tile(t / w, shard, nshards);
                *qi_out = (int)(lo + t % w);
                return;
            }
            t -= nfull * w;
            for (int64_t kj = lo + 1;; ++kj) {
                if (!owns_key_tile(kj, shard, nshards)) continue;
                const int64_t c = hi - kj;
                if (t < c) {
                    *kj_out = (int)kj;
                    *qi_out = (int)(kj + t);
                    return;
                }
                t -= c;
            }
        }
        t -= cnt;
        lo = hi;
    }
}

}  // namespace lemo_plan
