// segloss.cuh - segment-based peak cutting of the lm-head loss (Jenga summary,
// section 4.2.3 "Segment-based Peak Cutting").
//
// The tokens are processed in segments of S rows.  For one segment the host
// runs, in stream order:
//
//   z   = h_seg W^T                      fp32 [S, V]   (gemm_kernel)
//   dz  = (softmax(z) - onehot(y)) / n   bf16 [S, V]   (row_kernel, here)
//   dh_seg  = dz W                       bf16 [S, d]   (gemm_kernel)
//   dW     += dz^T h_seg                 fp32 [V, d]   (gemm_kernel)
//
// so only one segment's logits exist at a time: the activation peak of the
// loss is S/T of the unsegmented one.  n is the number of valid tokens of
// the whole batch, counted once before the first segment (count_kernel);
// the loss is the fixed-order sum of the per-token terms divided by n
// (loss_kernel), so it does not depend on the segment size.
//
// row_kernel is one CTA per token row: the row's (max, sum of exp) - merged
// from the partial pairs the logits GEMM's epilogue left for every 128-column
// half tile, so the logits are read once - a block reduction, then a pass
// that writes the bf16 gradient row (16-byte loads of the fp32 logits).
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "common.cuh"

namespace lemo {
namespace segloss {

constexpr int kRowThreads = 256;
constexpr int kCountThreads = 1024;

// Number of targets different from `ignore`; a target outside [0, V) that is
// not `ignore` raises LEMO_ERR_INVALID_ARG (and is not counted).
__global__ void __launch_bounds__(kCountThreads)
    count_kernel(const int32_t* __restrict__ y, int64_t T, int V, int ignore,
                 int32_t* __restrict__ n_valid) {
    pdl_entry();
    __shared__ int part[kCountThreads / 32];
    int c = 0;
    bool bad = false;
    for (int64_t t = threadIdx.x; t < T; t += kCountThreads) {
        const int v = y[t];
        if (v == ignore) continue;
        if (v < 0 || v >= V)
            bad = true;
        else
            ++c;
    }
    if (bad) raise_error(LEMO_ERR_INVALID_ARG);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = c;
    __syncthreads();
    if (threadIdx.x < 32) {
        c = part[threadIdx.x];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        if (threadIdx.x == 0) *n_valid = c;
    }
}

struct RowArgs {
    const float* z;        // segment logits, row r at z + r * ldz
    int64_t ldz;
    const float2* stats;   // optional: per row, nstats partial (max, sum of 2^(u - max)) pairs
    int nstats;            // (u = z log2(e)) from the logits GEMM, so pass 1 reads no logits
    uint16_t* g;           // bf16 gradient of the logits, row r at g + r * ldg
    int64_t ldg;
    const int32_t* y;      // targets of the segment's rows
    float* token_loss;     // per-row loss term of the segment's rows
    const int32_t* n_valid;
    int V;
    int ignore;
};

// Merge two (max, sum) pairs of the online log-sum-exp; values are in log2
// units (u = z * log2(e)), sums are sum_v 2^(u_v - max).
__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2) {
    const float mn = fmaxf(m, m2);
    if (mn == -CUDART_INF_F) return;  // both empty
    s = s * exp2f(m - mn) + s2 * exp2f(m2 - mn);
    m = mn;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&r);
}

__global__ void __launch_bounds__(kRowThreads) row_kernel(RowArgs a) {
    pdl_entry();
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr float kLn2 = 0.6931471805599453f;
    const int r = blockIdx.x;
    const float* zr = a.z + (int64_t)r * a.ldz;
    uint16_t* gr = a.g + (int64_t)r * a.ldg;
    const int V = a.V;
    const int nvec = V >> 2;
    const int tgt = a.y[r];
    const int n = *a.n_valid;
    const bool live = tgt != a.ignore && tgt >= 0 && tgt < V && n > 0;
    if (!live) {  // ignored token (or nothing valid): zero gradient row, no loss
        for (int j = threadIdx.x; j < nvec; j += kRowThreads)
            *reinterpret_cast<uint2*>(gr + 4 * j) = make_uint2(0u, 0u);
        for (int v = 4 * nvec + threadIdx.x; v < V; v += kRowThreads) gr[v] = 0;
        if (threadIdx.x == 0) a.token_loss[r] = 0.f;
        return;
    }

    // pass 1: online max and sum of 2^(u - max), from the GEMM's partial pairs
    // of the row when it gave them, else from the logits
    float m = -CUDART_INF_F, s = 0.f;
    const float4* z4 = reinterpret_cast<const float4*>(zr);
    if (a.stats) {
        const float2* sr = a.stats + (int64_t)r * a.nstats;
        for (int j = threadIdx.x; j < a.nstats; j += kRowThreads) {
            const float2 p = sr[j];
            lse_merge(m, s, p.x, p.y);
        }
    } else
    for (int j = threadIdx.x; j < nvec; j += kRowThreads) {
        const float4 v = z4[j];
        const float u0 = v.x * kLog2e, u1 = v.y * kLog2e, u2 = v.z * kLog2e, u3 = v.w * kLog2e;
        const float m4 = fmaxf(fmaxf(u0, u1), fmaxf(u2, u3));
        if (m4 > m) {
            s *= exp2f(m - m4);
            m = m4;
        }
        s += exp2f(u0 - m) + exp2f(u1 - m) + exp2f(u2 - m) + exp2f(u3 - m);
    }
    if (!a.stats)
    for (int v = 4 * nvec + threadIdx.x; v < V; v += kRowThreads) {
        const float u = zr[v] * kLog2e;
        if (u > m) {
            s *= exp2f(m - u);
            m = u;
        }
        s += exp2f(u - m);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
        lse_merge(m, s, m2, s2);
    }
    __shared__ float sm[kRowThreads / 32], ss[kRowThreads / 32];
    __shared__ float lse2_sh;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        sm[warp] = m;
        ss[warp] = s;
    }
    __syncthreads();
    if (warp == 0) {
        m = lane < kRowThreads / 32 ? sm[lane] : -CUDART_INF_F;
        s = lane < kRowThreads / 32 ? ss[lane] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
            lse_merge(m, s, m2, s2);
        }
        if (lane == 0) {
            const float lse2 = m + log2f(s);
            lse2_sh = lse2;
            a.token_loss[r] = lse2 * kLn2 - zr[tgt];
        }
    }
    __syncthreads();
    const float lse2 = lse2_sh;

    // pass 2: g = (2^(u - lse2) - [v == tgt]) / n, rounded to bf16
    const float inv_n = 1.f / (float)n;
    const int tj = tgt >> 2, tl = tgt & 3;
    for (int j = threadIdx.x; j < nvec; j += kRowThreads) {
        const float4 v = z4[j];
        float p0 = exp2f(fmaf(v.x, kLog2e, -lse2)) * inv_n;
        float p1 = exp2f(fmaf(v.y, kLog2e, -lse2)) * inv_n;
        float p2 = exp2f(fmaf(v.z, kLog2e, -lse2)) * inv_n;
        float p3 = exp2f(fmaf(v.w, kLog2e, -lse2)) * inv_n;
        if (j == tj) {
            p0 -= tl == 0 ? inv_n : 0.f;
            p1 -= tl == 1 ? inv_n : 0.f;
            p2 -= tl == 2 ? inv_n : 0.f;
            p3 -= tl == 3 ? inv_n : 0.f;
        }
        *reinterpret_cast<uint2*>(gr + 4 * j) = make_uint2(pack_bf16x2(p0, p1), pack_bf16x2(p2, p3));
    }
    for (int v = 4 * nvec + threadIdx.x; v < V; v += kRowThreads) {
        float p = exp2f(fmaf(zr[v], kLog2e, -lse2)) * inv_n;
        if (v == tgt) p -= inv_n;
        const __nv_bfloat16 b = __float2bfloat16_rn(p);
        gr[v] = *reinterpret_cast<const uint16_t*>(&b);
    }
}

// loss = (sum of the per-token terms, fixed order, in double) / n; 0 if n = 0.
__global__ void __launch_bounds__(kCountThreads)
    loss_kernel(const float* __restrict__ token_loss, int64_t T, const int32_t* __restrict__ n_valid,
                float* __restrict__ loss) {
    pdl_entry();
    __shared__ double part[kCountThreads / 32];
    double acc = 0.0;
    for (int64_t t = threadIdx.x; t < T; t += kCountThreads) acc += (double)token_loss[t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x < 32) {
        acc = part[threadIdx.x];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (threadIdx.x == 0) {
            const int n = *n_valid;
            *loss = n > 0 ? (float)(acc / (double)n) : 0.f;
        }
    }
}

}  // namespace segloss
}  // namespace lemo
