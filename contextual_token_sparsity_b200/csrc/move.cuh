// move.cuh - permutation-free token movement (steps a6-a7): gather of kept
// rows into a zero-padded dense buffer, and scatter-back fused with the
// residual add.  Both are HBM-bound row copies: one warp moves one row at a
// time with 16-byte vector accesses, kUnroll loads in flight per lane, and
// the grid is a whole number of waves over the SMs (persistent, grid-stride
// over rows), so the number of kept rows K can stay on the device.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace lemo {

constexpr int kMoveThreads = 256;
constexpr int kMoveUnroll = 16;  // 16-byte vectors per lane in flight

struct MoveArgs {
    const uint4* src;  // gather: x ; scatter: y
    uint4* dst;        // gather: y ; scatter: x (in place)
    int64_t ld_src;    // in 16-byte vectors
    int64_t ld_dst;
    int64_t x_rows;
    int dvec;          // row width in 16-byte vectors
    const int32_t* kept_idx;
    const int32_t* kept_total;
    int pad_to;
    int64_t cap;       // gather: y capacity in rows
};

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// y[r] = x[kept_idx[r]] for r < K; y[r] = 0 for K <= r < round_up(K, pad_to).
__global__ void __launch_bounds__(kMoveThreads) gather_pad_kernel(MoveArgs a) {
    pdl_entry();
    int64_t K = *a.kept_total;
    if (K < 0) K = 0;
    int64_t K_pad = (K + a.pad_to - 1) / a.pad_to * a.pad_to;
    if (K_pad > a.cap) {
        if (blockIdx.x == 0 && threadIdx.x == 0) raise_error(LEMO_ERR_CAPACITY);
        K_pad = a.cap;
        if (K > K_pad) K = K_pad;
    }
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * kMoveThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kMoveThreads) >> 5;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    for (int64_t r = warp; r < K_pad; r += nwarps) {
        uint4* dst = a.dst + r * a.ld_dst;
        if (r < K) {
            const int64_t t = a.kept_idx[r];
            if (t < 0 || t >= a.x_rows) {
                if (lane == 0) raise_error(LEMO_ERR_INVALID_ARG);
                continue;
            }
            const uint4* src = a.src + t * a.ld_src;
            for (int c0 = 0; c0 < a.dvec; c0 += 32 * kMoveUnroll) {
                uint4 v[kMoveUnroll];
#pragma unroll
                for (int u = 0; u < kMoveUnroll; ++u) {
                    const int c = c0 + u * 32 + lane;
                    if (c < a.dvec) v[u] = ld_stream(src + c);
                }
#pragma unroll
                for (int u = 0; u < kMoveUnroll; ++u) {
                    const int c = c0 + u * 32 + lane;
                    if (c < a.dvec) dst[c] = v[u];
                }
            }
        } else {
            for (int c = lane; c < a.dvec; c += 32) dst[c] = zero;
        }
    }
}

__device__ __forceinline__ uint32_t add_bf16x2_rn(uint32_t a, uint32_t b) {
    // Widen both bf16 pairs to fp32 (exact), add in fp32, round once to bf16
    // (nearest, ties to even); for two bf16 inputs this is the exactly
    // rounded sum.
    const float alo = __uint_as_float(a << 16), ahi = __uint_as_float(a & 0xffff0000u);
    const float blo = __uint_as_float(b << 16), bhi = __uint_as_float(b & 0xffff0000u);
    const __nv_bfloat162 r = __floats2bfloat162_rn(alo + blo, ahi + bhi);
    return *reinterpret_cast<const uint32_t*>(&r);
}

__device__ __forceinline__ uint4 add_bf16x8(uint4 x, uint4 y) {
    return make_uint4(add_bf16x2_rn(x.x, y.x), add_bf16x2_rn(x.y, y.y), add_bf16x2_rn(x.z, y.z),
                      add_bf16x2_rn(x.w, y.w));
}

// x[kept_idx[r]] = bf16(x[kept_idx[r]] + y[r]) for r < K, in place.
__global__ void __launch_bounds__(kMoveThreads) scatter_residual_kernel(MoveArgs a) {
    pdl_entry();
    int64_t K = *a.kept_total;
    if (K < 0) K = 0;
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * kMoveThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kMoveThreads) >> 5;
    constexpr int U = kMoveUnroll / 2;  // two streams (x and y) per vector
    for (int64_t r = warp; r < K; r += nwarps) {
        const int64_t t = a.kept_idx[r];
        if (t < 0 || t >= a.x_rows) {
            if (lane == 0) raise_error(LEMO_ERR_INVALID_ARG);
            continue;
        }
        uint4* xr = a.dst + t * a.ld_dst;
        const uint4* yr = a.src + r * a.ld_src;
        for (int c0 = 0; c0 < a.dvec; c0 += 32 * U) {
            uint4 xv[U], yv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < a.dvec) {
                    xv[u] = xr[c];
                    yv[u] = ld_stream(yr + c);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < a.dvec) xr[c] = add_bf16x8(xv[u], yv[u]);
            }
        }
    }
}

// Backward-pass input recomputation (Jenga summary, section 4.2.3: the
// original inputs are recovered by subtracting the sublayer output):
// x[kept_idx[r]] = bf16(x[kept_idx[r]] - y[r]) for r < K, in place, one
// rounding of the exact difference.
__device__ __forceinline__ uint32_t sub_bf16x2_rn(uint32_t a, uint32_t b) {
    const float alo = __uint_as_float(a << 16), ahi = __uint_as_float(a & 0xffff0000u);
    const float blo = __uint_as_float(b << 16), bhi = __uint_as_float(b & 0xffff0000u);
    const __nv_bfloat162 r = __floats2bfloat162_rn(alo - blo, ahi - bhi);
    return *reinterpret_cast<const uint32_t*>(&r);
}

__global__ void __launch_bounds__(kMoveThreads) recompute_input_kernel(MoveArgs a) {
    pdl_entry();
    int64_t K = *a.kept_total;
    if (K < 0) K = 0;
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * kMoveThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kMoveThreads) >> 5;
    constexpr int U = kMoveUnroll / 2;
    for (int64_t r = warp; r < K; r += nwarps) {
        const int64_t t = a.kept_idx[r];
        if (t < 0 || t >= a.x_rows) {
            if (lane == 0) raise_error(LEMO_ERR_INVALID_ARG);
            continue;
        }
        uint4* xr = a.dst + t * a.ld_dst;
        const uint4* yr = a.src + r * a.ld_src;
        for (int c0 = 0; c0 < a.dvec; c0 += 32 * U) {
            uint4 xv[U], yv[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < a.dvec) {
                    xv[u] = xr[c];
                    yv[u] = ld_stream(yr + c);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < a.dvec)
                    xr[c] = make_uint4(sub_bf16x2_rn(xv[u].x, yv[u].x), sub_bf16x2_rn(xv[u].y, yv[u].y),
                                       sub_bf16x2_rn(xv[u].z, yv[u].z), sub_bf16x2_rn(xv[u].w, yv[u].w));
            }
        }
    }
}

}  // namespace lemo
