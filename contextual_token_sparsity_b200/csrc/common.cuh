// common.cuh - device-side helpers shared by the kernels of liblemo.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "lemo.h"

namespace lemo {

// First error recorded on this device since the last lemo_get_error()
// (0 = none).  Kernels never trap: they record a status here and skip work.
__device__ unsigned int g_error;

__device__ __forceinline__ void raise_error(unsigned int code) { atomicCAS(&g_error, 0u, code); }

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Programmatic dependent launch.  The host launches every kernel of the
// library with programmatic stream serialization, so a kernel's CTAs may be
// scheduled before the previous kernel in the stream has finished.  Each
// kernel therefore calls pdl_entry() before anything else: it waits until
// the previous kernel has completed and its memory writes are visible, then
// lets the next kernel be scheduled.  For a plain launch both are no-ops.
__device__ __forceinline__ void pdl_entry() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename T>
__host__ __device__ __forceinline__ T ceil_div(T a, T b) { return (a + b - 1) / b; }

// Index of the last element <= v in the nondecreasing array a[0..n-1]
// (a[0] <= v is required).  Used to find the sequence holding a row or a
// block from a prefix array.
template <typename T, typename V>
__device__ __forceinline__ int last_le(const T* a, int n, V v) {
    int lo = 0, hi = n - 1;  // invariant: a[lo] <= v
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((V)a[mid] <= v) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// ---------------------------------------------------------------------------
// Workspace layout (shared by lemo_score_blocks and lemo_select).
// ---------------------------------------------------------------------------
struct PlanHeader {
    int32_t valid;          // 1 once cu_seqlens passed the device checks
    int32_t total_blocks;   // sum_s ceil(L_s / b)
    int32_t select_ticket;  // tile ticket of the compaction kernel
    int32_t pad0;
    int64_t total_tiles;    // score tiles of the batch
    int64_t total_m;        // sum_s ceil(L_s / b)^2
};

struct WsLayout {
    size_t hdr, tile_prefix, blk_prefix, m_prefix, lookback, mblk, total;
    int64_t n_lookback, m_cap;
};

constexpr int kSelectThreads = 256;
constexpr int kSelectItems = 8;
constexpr int kSelectTile = kSelectThreads * kSelectItems;  // tokens per compaction tile

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline WsLayout ws_layout(int batch, int total_L, int max_seqlen, int block) {
    WsLayout w;
    size_t off = 0;
    w.hdr = off;          off = align_up(off + sizeof(PlanHeader), 256);
    w.tile_prefix = off;  off = align_up(off + sizeof(int64_t) * (size_t)(batch + 1), 256);
    w.blk_prefix = off;   off = align_up(off + sizeof(int32_t) * (size_t)(batch + 1), 256);
    w.m_prefix = off;     off = align_up(off + sizeof(int64_t) * (size_t)(batch + 1), 256);
    w.n_lookback = total_L > 0 ? ((int64_t)total_L + kSelectTile - 1) / kSelectTile : 1;
    w.lookback = off;     off = align_up(off + sizeof(uint64_t) * (size_t)w.n_lookback, 256);
    const int64_t nb_max = ((int64_t)max_seqlen + block - 1) / block;
    const int64_t nb_sum = ((int64_t)total_L + (int64_t)batch * (block - 1)) / block;
    w.m_cap = nb_max * nb_sum;
    w.mblk = off;         off = align_up(off + sizeof(float) * (size_t)w.m_cap, 256);
    w.total = off;
    return w;
}

}  // namespace lemo
