// mlp.cuh - token-block scores of the MLP block (Jenga summary, section
// 4.2.1, "Extend to MLP Block"): the intermediate activation of a token - the
// ReLU output, or SiLU(gate) * up - is summed over its positive entries, and
// a token block scores the maximum over its tokens (the block rule of Eq. 2).
// The selection, gather and scatter kernels then apply unchanged.
//
// One warp per token row over a persistent grid (two CTAs of 512 threads per
// SM, 64 registers each), 16-byte loads with eight per operand in flight per
// lane (HBM-bound); per-lane partial sums in a fixed order and a
// fixed butterfly make each token score deterministic, and the block maximum
// does not depend on the order its tokens finish.
#pragma once

#include "common.cuh"

namespace lemo {
namespace mlp {

constexpr int kThreads = 512;
constexpr int kUnroll = 8;

__device__ __forceinline__ float pos_sum8(uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        s += fmaxf(__uint_as_float(w[i] << 16), 0.f);
        s += fmaxf(__uint_as_float(w[i] & 0xffff0000u), 0.f);
    }
    return s;
}

// SiLU(g) * u with the logistic written as (1 + tanh(g / 2)) / 2: one
// hardware tanh (tanh.approx.f32, about 2^-11 relative error) instead of an
// exponential and a division, which keeps this kernel memory-bound.
__device__ __forceinline__ float silu_mul(float g, float u) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * g));
    return g * fmaf(0.5f, t, 0.5f) * u;
}

__device__ __forceinline__ float pos_sum8_gated(uint4 g, uint4 u) {
    const uint32_t gw[4] = {g.x, g.y, g.z, g.w}, uw[4] = {u.x, u.y, u.z, u.w};
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        s += fmaxf(silu_mul(__uint_as_float(gw[i] << 16), __uint_as_float(uw[i] << 16)), 0.f);
        s += fmaxf(silu_mul(__uint_as_float(gw[i] & 0xffff0000u), __uint_as_float(uw[i] & 0xffff0000u)), 0.f);
    }
    return s;
}

struct Args {
    const uint16_t* act;   // ReLU-output mode (or nullptr)
    const uint16_t* gate;  // SiLU-gated mode
    const uint16_t* up;
    int64_t ld;            // row stride in elements
    int dvec;              // d_ff / 8
    const int32_t* cu;
    int batch;
    int block;
    const char* ws;
    WsLayout lay;
    float* token_scores;   // optional [total_L]
    float* block_scores;   // [total_blocks]
};

// One warp per token row, persistent grid over all tokens.  The block score
// is the maximum of its tokens' scores; every score is >= 0, so the maxima
// combine with an integer atomicMax on the float bit patterns (order does
// not change a maximum: deterministic).  block_scores must be zeroed first.
__global__ void __launch_bounds__(kThreads, 2) block_scores_kernel(const Args a) {
    pdl_entry();
    const PlanHeader* hdr = reinterpret_cast<const PlanHeader*>(a.ws + a.lay.hdr);
    if (!hdr->valid) return;
    const int32_t* blk_prefix = reinterpret_cast<const int32_t*>(a.ws + a.lay.blk_prefix);
    const int lane = threadIdx.x & 31;
    const int64_t total_L = a.cu[a.batch];
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
    for (int64_t r = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5; r < total_L; r += nwarps) {
        float part = 0.f;
        if (a.act) {
            const uint4* row = reinterpret_cast<const uint4*>(a.act + r * a.ld);
            for (int c0 = 0; c0 < a.dvec; c0 += 32 * kUnroll) {
                uint4 v[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int c = c0 + u * 32 + lane;
                    v[u] = c < a.dvec ? __ldg(row + c) : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) part += pos_sum8(v[u]);
            }
        } else {
            const uint4* grow = reinterpret_cast<const uint4*>(a.gate + r * a.ld);
            const uint4* urow = reinterpret_cast<const uint4*>(a.up + r * a.ld);
            for (int c0 = 0; c0 < a.dvec; c0 += 32 * kUnroll) {
                uint4 gv[kUnroll], uv[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int c = c0 + u * 32 + lane;
                    gv[u] = c < a.dvec ? __ldg(grow + c) : make_uint4(0u, 0u, 0u, 0u);
                    uv[u] = c < a.dvec ? __ldg(urow + c) : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) part += pos_sum8_gated(gv[u], uv[u]);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == 0) {
            if (a.token_scores) a.token_scores[r] = part;
            const int s = last_le(a.cu, a.batch + 1, (int)r);
            const int g = blk_prefix[s] + ((int)r - a.cu[s]) / a.block;
            atomicMax(reinterpret_cast<int*>(a.block_scores) + g, __float_as_int(part));
        }
    }
}

}  // namespace mlp
}  // namespace lemo
