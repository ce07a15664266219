// lemo.cu - host side of liblemo.so: argument checks, workspace layout,
// tensor-map encoding and launches.  The kernels live in the included .cuh
// files; everything is one translation unit so that the device error word is
// a single symbol per device.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <climits>
#include <mutex>
#include <utility>

#include "lemo.h"
#include "attn.cuh"
#include "common.cuh"
#include "gemm.cuh"
#include "mlp.cuh"
#include "move.cuh"
#include "predict.cuh"
#include "score.cuh"
#include "segloss.cuh"
#include "select.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int32_t kMaxSeqlen = 1 << 22;
constexpr int64_t kDefaultSpinNs = 2000000000LL;

std::mutex g_mu;
int g_sms[kMaxDevices];              // 0 = not queried yet
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
int g_skip_publish_tile = -1;
int g_predict_skip_cta = -1;
int64_t g_spin_ns = kDefaultSpinNs;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Number of SMs of the current device (cached).  Returns 0 on failure.
int device_sms(int* dev_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    *dev_out = dev;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        g_sms[dev] = n;
    }
    return g_sms[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    return g_encode;
}

// Every kernel of the library starts with griddepcontrol.wait (pdl_wait),
// so each one may be launched with programmatic stream serialization: its
// CTAs can be scheduled while the previous kernel in the stream drains, and
// they touch no memory before that kernel has completed.  Launch errors are
// kept for the next launch_status().
thread_local cudaError_t t_launch_error = cudaSuccess;

template <typename... P, typename... A>
void launch(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
            A&&... args) {
    cudaLaunchConfig_t c = {};
    c.gridDim = grid;
    c.blockDim = block;
    c.dynamicSmemBytes = smem;
    c.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    c.attrs = at;
    c.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&c, kernel, std::forward<A>(args)...);
    if (e != cudaSuccess && t_launch_error == cudaSuccess) t_launch_error = e;
}

lemo_status launch_status() {
    const cudaError_t launch_e = t_launch_error;
    t_launch_error = cudaSuccess;
    return (cudaGetLastError() == cudaSuccess && launch_e == cudaSuccess) ? LEMO_OK : LEMO_ERR_CUDA;
}

// Shape checks common to scoring and selection.
lemo_status check_shape(const lemo_shape* s, bool scoring) {
    if (!s || !s->cu_seqlens) return LEMO_ERR_INVALID_ARG;
    if (s->batch < 1 || s->total_L < 0 || s->max_seqlen < 0) return LEMO_ERR_INVALID_ARG;
    if (s->max_seqlen > kMaxSeqlen) return LEMO_ERR_UNSUPPORTED;
    if (s->total_L > 0 && s->max_seqlen == 0) return LEMO_ERR_INVALID_ARG;
    if (s->block <= 0) return LEMO_ERR_INVALID_ARG;
    if (s->block != 64 && s->block != 128) return LEMO_ERR_UNSUPPORTED;
    if (!aligned(s->cu_seqlens, 4)) return LEMO_ERR_INVALID_ARG;
    if (scoring) {
        if (s->H < 1 || s->dh < 1) return LEMO_ERR_INVALID_ARG;
        if (s->dh != 64 && s->dh != 128) return LEMO_ERR_UNSUPPORTED;
        if ((int64_t)s->H * s->dh > (1 << 20)) return LEMO_ERR_UNSUPPORTED;
    }
    return LEMO_OK;
}

lemo::WsLayout layout_of(const lemo_shape* s) {
    return lemo::ws_layout(s->batch, s->total_L, s->max_seqlen, s->block);
}

lemo_status check_ws(const lemo_shape* s, const void* ws, size_t ws_bytes) {
    if (!ws || !aligned(ws, 256)) return LEMO_ERR_INVALID_ARG;
    if (ws_bytes < layout_of(s).total) return LEMO_ERR_INVALID_ARG;
    return LEMO_OK;
}

void launch_plan(const lemo_shape* s, char* ws, const lemo::WsLayout& lay, int32_t* zero_word,
                 cudaStream_t st, float* zero_blocks = nullptr, int shard = 0, int nshards = 1) {
    launch(lemo::plan_kernel, 1, 1024, 0, st, s->cu_seqlens, s->batch, s->total_L, s->max_seqlen,
           s->block, ws, lay, zero_word, zero_blocks, shard, nshards);
}

// 3-D view of a [rows, H*dh] bf16 matrix as (64 elements, rows, H*dh/64
// slices of 64), so that one box (64, box_rows, dh/64) fetches one head of
// box_rows rows as dh/64 consecutive 128-byte-swizzled K-major tiles.
bool encode_heads(CUtensorMap* tm, const uint16_t* base, int64_t rows, int64_t width, int dh,
                  uint32_t box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)lemo::score::KB, (cuuint64_t)rows,
                                (cuuint64_t)(width / lemo::score::KB)};
    const cuuint64_t strides[2] = {(cuuint64_t)(width * 2), (cuuint64_t)(lemo::score::KB * 2)};
    const cuuint32_t box[3] = {(cuuint32_t)lemo::score::KB, box_rows,
                               (cuuint32_t)(dh / lemo::score::KB)};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(base), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// 2-D view of a [rows, width] bf16 matrix with row stride ld (elements);
// one box is 64 columns x 64 rows with 128-byte swizzle.
bool encode_rows(CUtensorMap* tm, const uint16_t* base, int64_t rows, int64_t width, int64_t ld) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)width, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
    const cuuint32_t box[2] = {(cuuint32_t)lemo::attn::KB, 64u};
    const cuuint32_t estr[2] = {1, 1};
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(base), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

bool g_attn_smem_set[kMaxDevices];
bool g_prod_smem_set[kMaxDevices];

// CTA pairs of the scoring kernel that fit on the device at once (one
// persistent wave).  Sets the kernel's shared-memory limit on first use.
int g_score_pairs[kMaxDevices];

int score_pairs(int dev, int sms) {
    namespace sc = lemo::score;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_score_pairs[dev] == 0) {
        if (cudaFuncSetAttribute(sc::score_tiles_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 sc::SMEM_BYTES) != cudaSuccess)
            return 0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
        cfg.blockDim = dim3(sc::THREADS, 1, 1);
        cfg.dynamicSmemBytes = sc::SMEM_BYTES;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 2;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, sc::score_tiles_kernel, &cfg) !=
                cudaSuccess ||
            clusters < 1) {
            cudaGetLastError();
            clusters = sms / 2;
        }
        g_score_pairs[dev] = clusters < sms / 2 ? clusters : sms / 2;
    }
    return g_score_pairs[dev];
}

// Persistent grid of the row-copy kernels: as many CTAs as fit on the SMs
// at once (one full wave), so no CTA waits for a second wave.
int g_move_ctas[kMaxDevices][3];

template <typename Kernel>
int move_grid(int dev, int sms, int which, Kernel kernel) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_move_ctas[dev][which] == 0) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, lemo::kMoveThreads, 0) !=
                cudaSuccess ||
            per_sm < 1)
            per_sm = 1;
        g_move_ctas[dev][which] = per_sm;
    }
    return sms * g_move_ctas[dev][which];
}

lemo_status check_move(const void* x, int64_t ld_x, int64_t x_rows, int32_t d, const void* y,
                       int64_t ld_y, const int32_t* kept_idx, const int32_t* kept_total) {
    if (!x || !y || !kept_idx || !kept_total) return LEMO_ERR_INVALID_ARG;
    if (d <= 0 || x_rows < 0) return LEMO_ERR_INVALID_ARG;
    if (d % 8 != 0) return LEMO_ERR_UNSUPPORTED;
    if (ld_x < d || ld_y < d || ld_x % 8 != 0 || ld_y % 8 != 0) return LEMO_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(kept_idx, 4) || !aligned(kept_total, 4))
        return LEMO_ERR_INVALID_ARG;
    return LEMO_OK;
}

// Workspace of lemo_predict_scores: the plan/score layout (its block-score
// region holds the block products P) followed by the predictor buffers.
struct PredictLayout {
    lemo::WsLayout base;
    // byte offsets: block-mean images, split-K partials, hidden-activation
    // images, Qhat / Khat images, head-group partial products, barrier words,
    // padded weight planes
    size_t xb, part, hid, qk, ppart, sync, w1p, w2p, total;
    int ldw1;        // row length of the padded W1 planes (rank rounded up to 8)
    int64_t tb;      // upper bound of the number of token blocks
    int rt, tba;     // row tiles of 128 token blocks
    int kc, kc2;     // 64-column chunks of d and of the rank
    int ldr, nj, nt; // rank padded to 32, n tiles of the first GEMM and their width
    int zk, cps;     // K splits of the first GEMM, chunks per split
    int dhp, dc;     // head dimension padded to 64, its chunks
    int np, nc, nj2; // H * dhp, the second GEMM's unit width, its units per row tile
    int pt, groups, hpg;
    bool fits;       // every unit count fits in 32 bits
};

// The launch shapes depend only on the shape (not on the device), so the
// workspace size query and the call agree.  The first GEMM is split along K
// so that about one unit per SM of a B200 (148 SMs) is busy; the block
// products take one head group per unit, as many groups as keep the SMs busy.
PredictLayout predict_layout(const lemo_shape* s, int d, int rank) {
    namespace pr = lemo::predict;
    constexpr int64_t kTarget = 148;
    PredictLayout p;
    p.base = layout_of(s);
    p.tb = ((int64_t)s->total_L + (int64_t)s->batch * (s->block - 1)) / s->block;
    if (p.tb < 1) p.tb = 1;
    const int64_t rt = (p.tb + pr::TILE - 1) / pr::TILE;
    p.rt = (int)rt;
    p.tba = (int)(rt * pr::TILE);
    p.kc = (d + pr::KCH - 1) / pr::KCH;
    p.kc2 = (rank + pr::KCH - 1) / pr::KCH;
    p.ldr = (rank + 31) / 32 * 32;
    p.nj = (p.ldr + pr::MAX_NT - 1) / pr::MAX_NT;
    p.nt = ((p.ldr + p.nj - 1) / p.nj + 31) / 32 * 32;
    const int64_t base_units = 2 * rt * p.nj;
    int64_t cps = (p.kc * base_units + kTarget - 1) / kTarget;
    if (cps < 1) cps = 1;
    p.cps = (int)cps;
    p.zk = (int)((p.kc + cps - 1) / cps);
    p.dhp = (s->dh + pr::KCH - 1) / pr::KCH * pr::KCH;
    p.dc = p.dhp / pr::KCH;
    p.np = s->H * p.dhp;
    // second GEMM: units of nc columns, about one per SM of a B200
    {
        const int64_t cols = 2 * rt * (int64_t)p.np;
        int64_t nc = ((cols + kTarget - 1) / kTarget + 15) / 16 * 16;
        if (nc < 64) nc = 64;
        if (nc > pr::MAX_NT) nc = pr::MAX_NT;
        p.nc = (int)nc;
    }
    p.nj2 = (p.np + p.nc - 1) / p.nc;
    const int64_t pt = rt * (rt + 1) / 2;
    p.pt = (int)(pt < INT_MAX ? pt : INT_MAX);
    int64_t groups = (kTarget + pt - 1) / pt;
    if (groups > s->H) groups = s->H;
    while (groups > 1 && groups * (int64_t)p.tba * p.tba * 4 > ((int64_t)256 << 20)) --groups;
    if (groups < 1) groups = 1;
    p.hpg = (int)((s->H + groups - 1) / groups);
    p.groups = (s->H + p.hpg - 1) / p.hpg;
    p.fits = base_units * p.zk < INT_MAX && 2 * rt * p.nj2 < INT_MAX &&
             pt * p.groups < INT_MAX && (int64_t)p.tba * p.tba < ((int64_t)1 << 40);
    size_t off = p.base.total;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = lemo::align_up(off + bytes, 256);
        return o;
    };
    p.sync = take(4 * pr::kSyncWords);
    p.xb = take((size_t)rt * p.kc * 2 * pr::IMG);
    p.part = take(4 * (size_t)2 * p.zk * p.tba * p.ldr);
    p.hid = take((size_t)2 * rt * p.kc2 * 2 * pr::IMG);
    p.qk = take((size_t)2 * rt * s->H * p.dc * 2 * pr::IMG);
    p.ppart = take(4 * (size_t)p.groups * p.tba * p.tba);
    p.ldw1 = (rank + 7) / 8 * 8;
    p.w1p = take((size_t)2 * d * p.ldw1 * 2);
    p.w2p = take((size_t)2 * rank * p.np * 2);
    p.total = off;
    return p;
}

lemo_status check_predict(const lemo_shape* s, int d, int rank) {
    lemo_status e = check_shape(s, false);
    if (e != LEMO_OK) return e;
    if (s->H < 1 || s->dh < 1 || d < 1 || rank < 1) return LEMO_ERR_INVALID_ARG;
    if (d % 8 != 0) return LEMO_ERR_UNSUPPORTED;
    if (s->dh > 1024 || (int64_t)s->H * s->dh > (1 << 20) || d > (1 << 20) || rank > (1 << 16))
        return LEMO_ERR_UNSUPPORTED;
    return LEMO_OK;
}

// Workspace of lemo_segment_loss.
struct SegLayout {
    size_t n_valid, token_loss, z, g, stats, total;
    int64_t nstats;   // partial (max, sum) pairs per logit row (two per 256-column tile)
    int64_t ld;    // row stride of the segment's logits and gradient
    int64_t rows;  // rows of one segment buffer
    int64_t dz_segs;  // segments of dz held (dW is accumulated once per that many)
};

constexpr int64_t kDwSegs = 4;  // segments per dW GEMM

SegLayout seg_layout(int64_t T, int V, int seg_rows) {
    SegLayout l;
    l.ld = ((int64_t)V + 7) / 8 * 8;
    l.rows = T < seg_rows ? (T > 0 ? T : 1) : seg_rows;
    {
        const int64_t nseg = T > 0 ? (T + seg_rows - 1) / seg_rows : 1;
        l.dz_segs = nseg < kDwSegs ? nseg : kDwSegs;
    }
    size_t off = 0;
    l.n_valid = off; off = lemo::align_up(off + 4, 256);
    l.token_loss = off; off = lemo::align_up(off + 4 * (size_t)(T > 0 ? T : 1), 256);
    l.z = off; off = lemo::align_up(off + 4 * (size_t)l.rows * l.ld, 256);
    // up to kDwSegs segments of dz: dW is accumulated once per kDwSegs
    // segments (K = kDwSegs segment rows), which divides its fp32
    // read-add-write of the weight gradient by kDwSegs
    l.g = off; off = lemo::align_up(off + 2 * (size_t)l.dz_segs * l.rows * l.ld, 256);
    l.nstats = 2 * (((int64_t)V + lemo::gemm::TN - 1) / lemo::gemm::TN);
    l.stats = off; off = lemo::align_up(off + 8 * (size_t)l.rows * l.nstats, 256);
    l.total = off;
    return l;
}

bool seg_args_ok(int64_t T, int V, int seg_rows) {
    return T >= 0 && T <= INT_MAX && V >= 1 && seg_rows >= 1 && (int64_t)V + 7 <= INT_MAX;
}

// 2-D tensor map of a bf16 matrix [rows, cols] with row stride ld elements,
// 128-byte swizzle: K-major operands (cols = K) take boxes of 64 x 128,
// MN-major operands (rows = K, cols = M or N) boxes of 64 x 64.
bool encode_operand(CUtensorMap* tm, const uint16_t* base, int64_t rows, int64_t cols, int64_t ld,
                    bool mn_major) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
    const cuuint32_t box[2] = {(cuuint32_t)lemo::gemm::KB,
                               (cuuint32_t)(mn_major ? lemo::gemm::KB : lemo::gemm::ROWS)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// 2-D tensor map of a GEMM output [rows, cols] (fp32 or bf16, row stride ld
// elements), boxes of 32 rows x 128 bytes with 128-byte swizzle, for the
// epilogue's TMA stores and reduce-adds.
bool encode_output(CUtensorMap* tm, void* base, int64_t rows, int64_t cols, int64_t ld, bool f32) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const int esz = f32 ? 4 : 2;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(ld * esz)};
    const cuuint32_t box[2] = {(cuuint32_t)(128 / esz), 32u};
    const cuuint32_t estr[2] = {1, 1};
    return enc(tm, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base,
               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// 2-D tensor map of a bf16 weight matrix [rows, cols] (row stride ld
// elements, 16-byte aligned rows), boxes of 64 columns x 64 rows with
// 128-byte swizzle: the MN-major operand tiles of the predictor GEMMs.
bool encode_weight(CUtensorMap* tm, const uint16_t* base, int64_t rows, int64_t cols, int64_t ld) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
    const cuuint32_t box[2] = {64u, 64u};
    const cuuint32_t estr[2] = {1, 1};
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// CTA pairs of the GEMM kernel that fit at once (sets its shared-memory
// limit on first use).
int g_gemm_pairs[kMaxDevices];

int gemm_pairs(int dev, int sms) {
    namespace gm = lemo::gemm;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_gemm_pairs[dev] == 0) {
        if (cudaFuncSetAttribute(gm::gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 gm::SMEM_BYTES) != cudaSuccess)
            return 0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
        cfg.blockDim = dim3(gm::THREADS, 1, 1);
        cfg.dynamicSmemBytes = gm::SMEM_BYTES;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 2;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, gm::gemm_kernel, &cfg) != cudaSuccess ||
            clusters < 1) {
            cudaGetLastError();
            clusters = sms / 2;
        }
        g_gemm_pairs[dev] = clusters < sms / 2 ? clusters : sms / 2;
    }
    return g_gemm_pairs[dev];
}

// C[M, N] (=, or += for kAddF32) A[M, K] B[K, N] on the tensor cores.
// a_mn / b_mn: the operand's M / N index is the contiguous one in memory.
lemo_status run_gemm(int dev, int sms, cudaStream_t st, const uint16_t* A, int64_t lda, bool a_mn,
                     const uint16_t* B, int64_t ldb, bool b_mn, int M, int N, int K, int epi,
                     void* out, int64_t ld_out, bool m_fastest, float2* stats = nullptr) {
    namespace gm = lemo::gemm;
    if (M <= 0 || N <= 0) return LEMO_OK;
    CUtensorMap ta, tb, tc;
    if (!encode_operand(&ta, A, a_mn ? K : M, a_mn ? M : K, lda, a_mn) ||
        !encode_operand(&tb, B, b_mn ? K : N, b_mn ? N : K, ldb, b_mn) ||
        !encode_output(&tc, out, M, N, ld_out, epi != gm::kStoreBF16))
        return LEMO_ERR_CUDA;
    const int pairs = gemm_pairs(dev, sms);
    if (pairs <= 0) return LEMO_ERR_CUDA;
    gm::Args a;
    a.M = M;
    a.N = N;
    a.K = K;
    a.a_mn = a_mn ? 1 : 0;
    a.b_mn = b_mn ? 1 : 0;
    a.epi = epi;
    a.stats = stats;
    a.ld_stats = 2 * (int64_t)((N + gm::TN - 1) / gm::TN);
    a.tiles_m = (M + gm::TM - 1) / gm::TM;
    a.tiles_n = (N + gm::TN - 1) / gm::TN;
    a.m_fastest = m_fastest ? 1 : 0;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        a.spin_limit_ns = (uint64_t)g_spin_ns;
    }
    const int64_t tiles = (int64_t)a.tiles_m * a.tiles_n;
    const int64_t use = tiles < pairs ? tiles : pairs;
    launch(gm::gemm_kernel, (unsigned)(2 * use), gm::THREADS, gm::SMEM_BYTES, st, ta, tb, tc, a);
    return launch_status();
}

}  // namespace

extern "C" {

const char* lemo_status_string(lemo_status st) {
    switch (st) {
        case LEMO_OK: return "LEMO_OK";
        case LEMO_ERR_INVALID_ARG: return "LEMO_ERR_INVALID_ARG";
        case LEMO_ERR_UNSUPPORTED: return "LEMO_ERR_UNSUPPORTED";
        case LEMO_ERR_CUDA: return "LEMO_ERR_CUDA";
        case LEMO_ERR_CAPACITY: return "LEMO_ERR_CAPACITY";
        case LEMO_ERR_TIMEOUT: return "LEMO_ERR_TIMEOUT";
    }
    return "LEMO_ERR_UNKNOWN";
}

size_t lemo_workspace_size(const lemo_shape* shape) {
    if (check_shape(shape, false) != LEMO_OK) return 0;
    return layout_of(shape).total;
}

int64_t lemo_block_max_elems(int32_t batch, const int32_t* lengths_host, int32_t block) {
    if (batch < 1 || !lengths_host || block <= 0) return 0;
    int64_t n = 0;
    for (int s = 0; s < batch; ++s) {
        if (lengths_host[s] < 0) return 0;
        const int64_t nb = (lengths_host[s] + (int64_t)block - 1) / block;
        n += nb * nb;
    }
    return n;
}

}  // extern "C"

namespace {

lemo_status score_blocks(const lemo_shape* shape, const uint16_t* q, const uint16_t* k, float scale,
                         int shard, int nshards, float* block_max, float* block_scores, void* ws,
                         size_t ws_bytes, lemo_stream stream) {
    lemo_status e = check_shape(shape, true);
    if (e != LEMO_OK) return e;
    if (!q || !k || !block_scores) return LEMO_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(block_scores, 4) ||
        (block_max && !aligned(block_max, 4)))
        return LEMO_ERR_INVALID_ARG;
    if (!(scale > 0.f) || scale == __builtin_inff()) return LEMO_ERR_INVALID_ARG;
    if (nshards < 1 || nshards > 4096 || shard < 0 || shard >= nshards) return LEMO_ERR_INVALID_ARG;
    if ((e = check_ws(shape, ws, ws_bytes)) != LEMO_OK) return e;
    int dev = 0;
    const int sms = device_sms(&dev);
    if (sms <= 0) return LEMO_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const lemo::WsLayout lay = layout_of(shape);
    char* w = static_cast<char*>(ws);
    float* mblk = block_max ? block_max : reinterpret_cast<float*>(w + lay.mblk);

    launch_plan(shape, w, lay, nullptr, st, nullptr, shard, nshards);
    if ((e = launch_status()) != LEMO_OK) return e;
    if (shape->total_L > 0) {
        namespace sc = lemo::score;
        CUtensorMap tm_q, tm_k;
        const int64_t width = (int64_t)shape->H * shape->dh;
        if (!encode_heads(&tm_q, q, shape->total_L, width, shape->dh, sc::ROWS) ||
            !encode_heads(&tm_k, k, shape->total_L, width, shape->dh, sc::ROWS))
            return LEMO_ERR_CUDA;
        const int pairs = score_pairs(dev, sms);
        if (pairs <= 0) return LEMO_ERR_CUDA;
        sc::Args a;
        a.cu = shape->cu_seqlens;
        a.batch = shape->batch;
        a.H = shape->H;
        a.dh = shape->dh;
        a.block = shape->block;
        a.out_scale = scale / (float)shape->H;
        a.mblk = mblk;
        a.ws = w;
        a.lay = lay;
        a.spin_limit_ns = (uint64_t)g_spin_ns;
        a.shard = shard;
        a.nshards = nshards;
        launch(sc::score_tiles_kernel, 2 * pairs, sc::THREADS, sc::SMEM_BYTES, st, tm_q, tm_k, a);
        if ((e = launch_status()) != LEMO_OK) return e;
        // one warp per token block; the host knows an upper bound of their number
        const int64_t nb_bound =
            ((int64_t)shape->total_L + (int64_t)shape->batch * (shape->block - 1)) / shape->block;
        const int64_t cs_ctas = (nb_bound + 7) / 8;
        const int cs_grid = (int)(cs_ctas < (int64_t)sms * 8 ? (cs_ctas > 0 ? cs_ctas : 1) : sms * 8);
        launch(sc::column_sum_kernel, cs_grid, 256, 0, st, mblk, w, lay, shape->batch,
               block_scores, shape->block, shard, nshards);
        if ((e = launch_status()) != LEMO_OK) return e;
    }
    return LEMO_OK;
}

}  // namespace

extern "C" {

lemo_status lemo_score_blocks(const lemo_shape* shape, const uint16_t* q, const uint16_t* k,
                              float scale, float* block_max, float* block_scores, void* ws,
                              size_t ws_bytes, lemo_stream stream) {
    return score_blocks(shape, q, k, scale, 0, 1, block_max, block_scores, ws, ws_bytes, stream);
}

lemo_status lemo_score_blocks_shard(const lemo_shape* shape, const uint16_t* q, const uint16_t* k,
                                    float scale, int32_t shard, int32_t nshards, float* block_max,
                                    float* block_scores, void* ws, size_t ws_bytes,
                                    lemo_stream stream) {
    return score_blocks(shape, q, k, scale, shard, nshards, block_max, block_scores, ws, ws_bytes,
                        stream);
}

lemo_status lemo_select(const lemo_shape* shape, const float* block_scores, float threshold,
                        uint8_t* block_mask, int32_t* kept_idx, int32_t* cu_kept,
                        int32_t* kept_total, void* ws, size_t ws_bytes, lemo_stream stream) {
    lemo_status e = check_shape(shape, false);
    if (e != LEMO_OK) return e;
    if (!block_scores || !block_mask || !kept_idx || !cu_kept || !kept_total)
        return LEMO_ERR_INVALID_ARG;
    if (!aligned(block_scores, 4) || !aligned(kept_idx, 4) || !aligned(cu_kept, 4) ||
        !aligned(kept_total, 4))
        return LEMO_ERR_INVALID_ARG;
    if ((e = check_ws(shape, ws, ws_bytes)) != LEMO_OK) return e;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const lemo::WsLayout lay = layout_of(shape);
    char* w = static_cast<char*>(ws);
    launch_plan(shape, w, lay, kept_total, st);
    if ((e = launch_status()) != LEMO_OK) return e;
    lemo::SelectArgs a;
    a.cu = shape->cu_seqlens;
    a.batch = shape->batch;
    a.total_L = shape->total_L;
    a.block = shape->block;
    a.scores = block_scores;
    a.theta = threshold;
    a.mask = block_mask;
    a.kept_idx = kept_idx;
    a.cu_kept = cu_kept;
    a.kept_total = kept_total;
    a.ws = w;
    a.lay = lay;
    a.skip_publish_tile = g_skip_publish_tile;
    a.spin_limit_ns = (uint64_t)g_spin_ns;
    launch(lemo::select_kernel, (unsigned)lay.n_lookback, lemo::kSelectThreads, 0, st, a);
    return launch_status();
}

// ---------------------------------------------------------------------------
// lemo_select with its scratch in a device array owned by the library (for
// callers that cannot allocate).  The array is reserved in every GPU's memory
// when the library is loaded.  Host code must not pass the symbol itself to a
// kernel - on the host it names a host-side stand-in - so every call looks up
// its device address on the current device (a host-side query that
// allocates nothing); nothing is cached, so a device that was reset and
// re-initialised gets the array's new address.
// ---------------------------------------------------------------------------
}  // extern "C"

namespace {
constexpr int32_t kStaticMaxBatch = 4096;
constexpr int32_t kStaticMaxTokens = 1 << 24;
constexpr size_t kStaticScratchBytes = 160 * 1024;
}  // namespace

static __device__ __align__(256) char g_select_scratch[kStaticScratchBytes];

extern "C" {

lemo_status lemo_select_static_ws(const lemo_shape* shape, const float* block_scores,
                                  float threshold, uint8_t* block_mask, int32_t* kept_idx,
                                  int32_t* cu_kept, int32_t* kept_total, lemo_stream stream) {
    lemo_status e = check_shape(shape, false);
    if (e != LEMO_OK) return e;
    if (!block_scores || !block_mask || !kept_idx || !cu_kept || !kept_total)
        return LEMO_ERR_INVALID_ARG;
    if (!aligned(block_scores, 4) || !aligned(kept_idx, 4) || !aligned(cu_kept, 4) ||
        !aligned(kept_total, 4))
        return LEMO_ERR_INVALID_ARG;
    if (shape->batch > kStaticMaxBatch || shape->total_L > kStaticMaxTokens)
        return LEMO_ERR_CAPACITY;
    const lemo::WsLayout lay = layout_of(shape);
    if (lay.mblk > kStaticScratchBytes) return LEMO_ERR_CAPACITY;  // selection stops before M
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return LEMO_ERR_CUDA;
    }
    char* w = static_cast<char*>(p);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // The plan kernel re-initialises the look-back descriptors, the ticket and
    // kept_total at the start of every call.
    launch_plan(shape, w, lay, kept_total, st);
    if ((e = launch_status()) != LEMO_OK) return e;
    lemo::SelectArgs a;
    a.cu = shape->cu_seqlens;
    a.batch = shape->batch;
    a.total_L = shape->total_L;
    a.block = shape->block;
    a.scores = block_scores;
    a.theta = threshold;
    a.mask = block_mask;
    a.kept_idx = kept_idx;
    a.cu_kept = cu_kept;
    a.kept_total = kept_total;
    a.ws = w;
    a.lay = lay;
    a.skip_publish_tile = g_skip_publish_tile;
    a.spin_limit_ns = (uint64_t)g_spin_ns;
    launch(lemo::select_kernel, (unsigned)lay.n_lookback, lemo::kSelectThreads, 0, st, a);
    return launch_status();
}

lemo_status lemo_gather_pad(const uint16_t* x, int64_t ld_x, int64_t x_rows, int32_t d,
                            const int32_t* kept_idx, const int32_t* kept_total, int32_t pad_to,
                            uint16_t* y, int64_t ld_y, int64_t y_rows_capacity,
                            lemo_stream stream) {
    lemo_status e = check_move(x, ld_x, x_rows, d, y, ld_y, kept_idx, kept_total);
    if (e != LEMO_OK) return e;
    if (pad_to < 1 || y_rows_capacity < 0) return LEMO_ERR_INVALID_ARG;
    int dev = 0;
    const int sms = device_sms(&dev);
    if (sms <= 0) return LEMO_ERR_CUDA;
    lemo::MoveArgs a;
    a.src = reinterpret_cast<const uint4*>(x);
    a.dst = reinterpret_cast<uint4*>(y);
    a.ld_src = ld_x / 8;
    a.ld_dst = ld_y / 8;
    a.x_rows = x_rows;
    a.dvec = d / 8;
    a.kept_idx = kept_idx;
    a.kept_total = kept_total;
    a.pad_to = pad_to;
    a.cap = y_rows_capacity;
    launch(lemo::gather_pad_kernel, move_grid(dev, sms, 0, lemo::gather_pad_kernel),
           lemo::kMoveThreads, 0, reinterpret_cast<cudaStream_t>(stream), a);
    return launch_status();
}

lemo_status lemo_scatter_residual(uint16_t* x, int64_t ld_x, int64_t x_rows, int32_t d,
                                  const uint16_t* y, int64_t ld_y, const int32_t* kept_idx,
                                  const int32_t* kept_total, lemo_stream stream) {
    lemo_status e = check_move(x, ld_x, x_rows, d, y, ld_y, kept_idx, kept_total);
    if (e != LEMO_OK) return e;
    int dev = 0;
    const int sms = device_sms(&dev);
    if (sms <= 0) return LEMO_ERR_CUDA;
    lemo::MoveArgs a;
    a.src = reinterpret_cast<const uint4*>(y);
    a.dst = reinterpret_cast<uint4*>(x);
    a.ld_src = ld_y / 8;
    a.ld_dst = ld_x / 8;
    a.x_rows = x_rows;
    a.dvec = d / 8;
    a.kept_idx = kept_idx;
    a.kept_total = kept_total;
    a.pad_to = 1;
    a.cap = 0;
    launch(lemo::scatter_residual_kernel, move_grid(dev, sms, 1, lemo::scatter_residual_kernel),
           lemo::kMoveThreads, 0, reinterpret_cast<cudaStream_t>(stream), a);
    return launch_status();
}

lemo_status lemo_recompute_input(uint16_t* x, int64_t ld_x, int64_t x_rows, int32_t d,
                                 const uint16_t* y, int64_t ld_y, const int32_t* kept_idx,
                                 const int32_t* kept_total, lemo_stream stream) {
    lemo_status e = check_move(x, ld_x, x_rows, d, y, ld_y, kept_idx, kept_total);
    if (e != LEMO_OK) return e;
    int dev = 0;
    const int sms = device_sms(&dev);
    if (sms <= 0) return LEMO_ERR_CUDA;
    lemo::MoveArgs a;
    a.src = reinterpret_cast<const uint4*>(y);
    a.dst = reinterpret_cast<uint4*>(x);
    a.ld_src = ld_y / 8;
    a.ld_dst = ld_x / 8;
    a.x_rows = x_rows;
    a.dvec = d / 8;
    a.kept_idx = kept_idx;
    a.kept_total = kept_total;
    a.pad_to = 1;
    a.cap = 0;
    launch(lemo::recompute_input_kernel, move_grid(dev, sms, 2, lemo::recompute_input_kernel),
           lemo::kMoveThreads, 0, reinterpret_cast<cudaStream_t>(stream), a);
    return launch_status();
}

lemo_status lemo_mlp_block_scores(const lemo_shape* shape, int32_t d_ff, const uint16_t* act,
                                  const uint16_t* gate, const uint16_t* up, int64_t ld,
                                  float* token_scores, float* block_scores, void* ws,
                                  size_t ws_bytes, lemo_stream stream) {
    lemo_status e = check_shape(shape, false);
    if (e != LEMO_OK) return e;
    const bool relu_mode = act != nullptr;
    if (relu_mode ? (gate || up) : (!gate || !up)) return LEMO_ERR_INVALID_ARG;
    if (!block_scores || d_ff < 1 || ld < d_ff) return LEMO_ERR_INVALID_ARG;
    if (d_ff % 8 != 0 || ld % 8 != 0) return LEMO_ERR_UNSUPPORTED;
    if ((act && !aligned(act, 16)) || (gate && !aligned(gate, 16)) || (up && !aligned(up, 16)) ||
        !aligned(block_scores, 4) || (token_scores && !aligned(token_scores, 4)))
        return LEMO_ERR_INVALID_ARG;
    if ((e = check_ws(shape, ws, ws_bytes)) != LEMO_OK) return e;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const lemo::WsLayout lay = layout_of(shape);
    char* w = static_cast<char*>(ws);
    launch_plan(shape, w, lay, nullptr, st, block_scores);  // also clears block_scores
    if ((e = launch_status()) != LEMO_OK) return e;
    if (shape->total_L == 0) return LEMO_OK;
    lemo::mlp::Args a;
    a.act = act;
    a.gate = gate;
    a.up = up;
    a.ld = ld;
    a.dvec = d_ff / 8;
    a.cu = shape->cu_seqlens;
    a.batch = shape->batch;
    a.block = shape->block;
    a.ws = w;
    a.lay = lay;
    a.token_scores = token_scores;
    a.block_scores = block_scores;
    int dev = 0;
    const int sms = device_sms(&dev);
    if (sms <= 0) return LEMO_ERR_CUDA;
    const int64_t ctas_needed =
        ((int64_t)shape->total_L + lemo::mlp::kThreads / 32 - 1) / (lemo::mlp::kThreads / 32);
    const int64_t grid = ctas_needed < (int64_t)sms * 2 ? ctas_needed : (int64_t)sms * 2;
    launch(lemo::mlp::block_scores_kernel, (unsigned)grid, lemo::mlp::kThreads, 0, st, a);
    return launch_status();
}

size_t lemo_predict_workspace_size(const lemo_shape* shape, int32_t d, int32_t rank) {
    if (check_predict(shape, d, rank) != LEMO_OK) return 0;
    return predict_layout(shape, d, rank).total;
}

lemo_status lemo_predict_scores(const lemo_shape* shape, int32_t d, const uint16_t* x,
                                int64_t ld_x, const uint16_t* w1q, const uint16_t* w2q,
                                const uint16_t* w1k, const uint16_t* w2k, int32_t rank,
                                float* block_scores, void* ws, size_t ws_bytes,
                                lemo_stream stream) {
    namespace pr = lemo::predict;
    lemo_status e = check_predict(shape, d, rank);
    if (e != LEMO_OK) return e;
    if (!x || !w1q || !w2q || !w1k || !w2k || !block_scores || !ws) return LEMO_ERR_INVALID_ARG;
    if (!aligned(x, 16) || ld_x < d || ld_x % 8 != 0 || !aligned(w1q, 2) || !aligned(w2q, 2) ||
        !aligned(w1k, 2) || !aligned(w2k, 2) || !aligned(block_scores, 4) || !aligned(ws, 256))
        return LEMO_ERR_INVALID_ARG;
    const PredictLayout p = predict_layout(shape, d, rank);
    if (!p.fits) return LEMO_ERR_UNSUPPORTED;
    if (ws_bytes < p.total) return LEMO_ERR_INVALID_ARG;
    int dev = 0;
    const int sms = device_sms(&dev);
    if (sms <= 0) return LEMO_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* w = static_cast<char*>(ws);
    const lemo::WsLayout& lay = p.base;
    uint32_t* sync = reinterpret_cast<uint32_t*>(w + p.sync);

    // one sequence: the pooling pass writes the plan itself (one launch less)
    const bool own_plan = shape->batch == 1 && shape->total_L > 0;
    if (!own_plan) {
        launch_plan(shape, w, lay, nullptr, st);
        if ((e = launch_status()) != LEMO_OK) return e;
    }
    if (shape->total_L == 0) return LEMO_OK;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_prod_smem_set[dev]) {
            if (cudaFuncSetAttribute(pr::predict_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     pr::SMEM_BYTES) != cudaSuccess)
                return LEMO_ERR_CUDA;
            int per_sm = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pr::predict_kernel,
                                                              pr::THREADS, pr::SMEM_BYTES) !=
                    cudaSuccess ||
                per_sm < 1)
                return LEMO_ERR_CUDA;
            g_prod_smem_set[dev] = true;
        }
    }
    // weights that TMA cannot read in place go through padded planes
    const bool pad_w1 = !(rank % 8 == 0 && aligned(w1q, 16) && aligned(w1k, 16));
    const bool pad_w2 = !(shape->dh % pr::KCH == 0 && aligned(w2q, 16) && aligned(w2k, 16));
    uint16_t* w1p = reinterpret_cast<uint16_t*>(w + p.w1p);
    uint16_t* w2p = reinterpret_cast<uint16_t*>(w + p.w2p);
    pr::PadArgs pa = {};
    pa.w1[0] = w1q;
    pa.w1[1] = w1k;
    pa.w2[0] = w2q;
    pa.w2[1] = w2k;
    if (pad_w1) {
        pa.w1p[0] = w1p;
        pa.w1p[1] = w1p + (size_t)d * p.ldw1;
    }
    if (pad_w2) {
        pa.w2p[0] = w2p;
        pa.w2p[1] = w2p + (size_t)rank * p.np;
    }
    pa.d = d;
    pa.rank = rank;
    pa.ldw1 = p.ldw1;
    pa.H = shape->H;
    pa.dh = shape->dh;
    pa.dhp = p.dhp;
    pa.w2_vec4 = shape->dh % 2 == 0 && aligned(w2q, 4) && aligned(w2k, 4);
    pr::Maps maps;
    for (int i = 0; i < 2; ++i) {
        const bool ok1 = pad_w1 ? encode_weight(&maps.w1[i], pa.w1p[i], d, p.ldw1, p.ldw1)
                                : encode_weight(&maps.w1[i], pa.w1[i], d, rank, rank);
        const bool ok2 = pad_w2 ? encode_weight(&maps.w2[i], pa.w2p[i], rank, p.np, p.np)
                                : encode_weight(&maps.w2[i], pa.w2[i], rank,
                                                (int64_t)shape->H * shape->dh,
                                                (int64_t)shape->H * shape->dh);
        if (!ok1 || !ok2) return LEMO_ERR_CUDA;
    }
    // block means, as hi / lo operand images (and the barrier words cleared,
    // the weight planes padded)
    const int npad = (pad_w1 || pad_w2) ? pr::kPadCtas : 0;
    const int64_t pool_ctas =
        (int64_t)p.tba * ((p.kc * pr::KCH + pr::kPoolCols - 1) / pr::kPoolCols);
    if (npad + pool_ctas > INT_MAX) return LEMO_ERR_UNSUPPORTED;
    launch(pr::pool_kernel, (unsigned)(npad + pool_ctas), pr::kPoolThreads, 0, st, x, ld_x, d, p.kc,
           npad, shape->cu_seqlens, shape->batch, shape->total_L, shape->max_seqlen,
           shape->block, w, lay, reinterpret_cast<uint8_t*>(w + p.xb), sync, pa,
           own_plan ? 1 : 0);
    if ((e = launch_status()) != LEMO_OK) return e;
    pr::Args a;
    a.ws = w;
    a.lay = lay;
    a.batch = shape->batch;
    a.d = d;
    a.rank = rank;
    a.H = shape->H;
    a.dh = shape->dh;
    a.dhp = p.dhp;
    a.dc = p.dc;
    a.rt = p.rt;
    a.tba = p.tba;
    a.kc = p.kc;
    a.kc2 = p.kc2;
    a.ldr = p.ldr;
    a.nj = p.nj;
    a.nt = p.nt;
    a.zk = p.zk;
    a.cps = p.cps;
    a.np = p.np;
    a.nc = p.nc;
    a.nj2 = p.nj2;
    a.pt = p.pt;
    a.groups = p.groups;
    a.hpg = p.hpg;
    a.inv_h = 1.f / (float)shape->H;
    a.xb = reinterpret_cast<const uint8_t*>(w + p.xb);
    a.part = reinterpret_cast<float*>(w + p.part);
    a.hid = reinterpret_cast<uint8_t*>(w + p.hid);
    a.qk = reinterpret_cast<uint8_t*>(w + p.qk);
    a.ppart = reinterpret_cast<float*>(w + p.ppart);
    a.sync = sync;
    a.scores = block_scores;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        a.spin_limit_ns = (uint64_t)g_spin_ns;
        a.skip_cta = g_predict_skip_cta;
    }
    // one persistent CTA per SM (the grid barriers need every CTA resident)
    launch(pr::predict_kernel, (unsigned)sms, pr::THREADS, pr::SMEM_BYTES, st, maps, a);
    return launch_status();
}

size_t lemo_attention_workspace_size(int32_t batch) {
    if (batch < 1) return 0;
    return lemo::attn::ws_bytes(batch);
}

lemo_status lemo_attention_kept(const lemo_shape* shape, const uint16_t* q, const uint16_t* k,
                                const uint16_t* v, int64_t ld_qkv, const int32_t* kept_idx,
                                const int32_t* cu_kept, const int32_t* kept_total, float scale,
                                uint16_t* x, int64_t ld_x, uint16_t* o, int64_t ld_o, void* ws,
                                size_t ws_bytes, lemo_stream stream) {
    namespace at = lemo::attn;
    lemo_status e = check_shape(shape, true);
    if (e != LEMO_OK) return e;
    if (!q || !k || !v || !kept_idx || !cu_kept || !kept_total || !ws) return LEMO_ERR_INVALID_ARG;
    if ((x == nullptr) == (o == nullptr)) return LEMO_ERR_INVALID_ARG;  // exactly one output
    if (!(scale > 0.f) || !(scale < 3.0e38f)) return LEMO_ERR_INVALID_ARG;
    const int64_t hd = (int64_t)shape->H * shape->dh;
    if (ld_qkv < hd || ld_qkv % 8 != 0 || (x && (ld_x < hd || ld_x % 8 != 0)) ||
        (o && (ld_o < hd || ld_o % 8 != 0)))
        return LEMO_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || (x && !aligned(x, 16)) ||
        (o && !aligned(o, 16)) || !aligned(kept_idx, 4) || !aligned(cu_kept, 4) ||
        !aligned(kept_total, 4) || !aligned(ws, 256))
        return LEMO_ERR_INVALID_ARG;
    if (ws_bytes < at::ws_bytes(shape->batch)) return LEMO_ERR_INVALID_ARG;
    // query-tile pairs: sequence s has ceil(ceil(K_s / BM) / 2) of them
    const int64_t tiles = ((int64_t)shape->total_L + (int64_t)shape->batch * (at::BM - 1)) / at::BM;
    const int64_t items = (tiles + shape->batch) / 2;
    if (items * shape->H >= (int64_t)1 << 31) return LEMO_ERR_UNSUPPORTED;
    int dev = 0;
    if (device_sms(&dev) <= 0) return LEMO_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* w = static_cast<char*>(ws);
    launch(at::plan_kernel, 1, 1024, 0, st, cu_kept, kept_total, shape->cu_seqlens, shape->batch,
           w);
    if ((e = launch_status()) != LEMO_OK) return e;
    if (shape->total_L == 0 || items == 0) return LEMO_OK;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_attn_smem_set[dev]) {
            if (cudaFuncSetAttribute(at::attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     at::SMEM_BYTES) != cudaSuccess)
                return LEMO_ERR_CUDA;
            g_attn_smem_set[dev] = true;
        }
    }
    CUtensorMap tq, tk, tv;
    if (!encode_rows(&tq, q, shape->total_L, hd, ld_qkv) ||
        !encode_rows(&tk, k, shape->total_L, hd, ld_qkv) ||
        !encode_rows(&tv, v, shape->total_L, hd, ld_qkv))
        return LEMO_ERR_CUDA;
    at::Args a;
    a.kept_idx = kept_idx;
    a.cu_kept = cu_kept;
    a.cu_seqlens = shape->cu_seqlens;
    a.batch = shape->batch;
    a.H = shape->H;
    a.dh = shape->dh;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.x = x;
    a.ld_x = ld_x;
    a.x_rows = shape->total_L;
    a.o = o;
    a.ld_o = ld_o;
    a.ws = w;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        a.spin_limit_ns = (uint64_t)g_spin_ns;
    }
    // heads are taken in groups of HEAD_GROUP: the grid covers whole groups
    const int hg = shape->H < at::HEAD_GROUP ? shape->H : at::HEAD_GROUP;
    const int64_t heads = (int64_t)(shape->H + hg - 1) / hg * hg;
    if (items * heads > INT_MAX) return LEMO_ERR_UNSUPPORTED;
    launch(at::attn_kernel, (unsigned)(items * heads), at::THREADS, at::SMEM_BYTES, st, tq, tk,
           tv, a);
    return launch_status();
}

size_t lemo_segment_loss_workspace_size(int64_t T, int32_t V, int32_t seg_rows) {
    if (!seg_args_ok(T, V, seg_rows)) return 0;
    return seg_layout(T, V, seg_rows).total;
}

lemo_status lemo_segment_loss(const uint16_t* h, int64_t ld_h, int64_t T, int32_t d,
                              const uint16_t* w, int64_t ld_w, int32_t V, const int32_t* targets,
                              int32_t ignore_index, int32_t seg_rows, float* loss,
                              float* token_loss, uint16_t* dh, int64_t ld_dh, float* dw,
                              int64_t ld_dw, void* ws, size_t ws_bytes, lemo_stream stream) {
    namespace sl = lemo::segloss;
    if (!seg_args_ok(T, V, seg_rows) || d < 1) return LEMO_ERR_INVALID_ARG;
    if (!loss || !ws || (T > 0 && (!h || !w || !targets))) return LEMO_ERR_INVALID_ARG;
    if (d % 8 != 0) return LEMO_ERR_UNSUPPORTED;
    auto stride_ok = [d](int64_t ld) { return ld >= d && ld % 8 == 0 && ld <= INT_MAX; };
    if (!stride_ok(ld_h) || !stride_ok(ld_w) || (dh && !stride_ok(ld_dh)) || (dw && !stride_ok(ld_dw)))
        return LEMO_ERR_INVALID_ARG;
    if (!aligned(h, 16) || !aligned(w, 16) || !aligned(targets, 4) || !aligned(loss, 4) ||
        (token_loss && !aligned(token_loss, 4)) || (dh && !aligned(dh, 16)) ||
        (dw && !aligned(dw, 16)) || !aligned(ws, 256))
        return LEMO_ERR_INVALID_ARG;
    const SegLayout l = seg_layout(T, V, seg_rows);
    if (ws_bytes < l.total) return LEMO_ERR_INVALID_ARG;
    int dev = 0;
    const int sms = device_sms(&dev);
    if (sms <= 0) return LEMO_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* wsp = static_cast<char*>(ws);
    int32_t* n_valid = reinterpret_cast<int32_t*>(wsp + l.n_valid);
    float* tl = token_loss ? token_loss : reinterpret_cast<float*>(wsp + l.token_loss);
    float* z = reinterpret_cast<float*>(wsp + l.z);
    uint16_t* g = reinterpret_cast<uint16_t*>(wsp + l.g);

    launch(sl::count_kernel, 1, sl::kCountThreads, 0, st, targets, T, V, ignore_index, n_valid);
    lemo_status e = launch_status();
    if (e != LEMO_OK) return e;
    namespace gm = lemo::gemm;
    for (int64_t s0 = 0, si = 0; s0 < T; s0 += seg_rows, ++si) {
        const int S = (int)(T - s0 < seg_rows ? T - s0 : seg_rows);
        const uint16_t* hs = h + s0 * ld_h;
        const int hb = (int)(si % l.dz_segs);             // which dz slot this segment uses
        uint16_t* gs = g + (size_t)hb * l.rows * l.ld;
        // z [S, V] = h_seg [S, d] . W [V, d]^T  (fp32, row stride l.ld)
        float2* stats = reinterpret_cast<float2*>(wsp + l.stats);
        if ((e = run_gemm(dev, sms, st, hs, ld_h, false, w, ld_w, false, S, V, d, gm::kStoreF32, z,
                          l.ld, true, stats)) != LEMO_OK)
            return e;
        sl::RowArgs a;
        a.z = z;
        a.ldz = l.ld;
        a.stats = stats;
        a.nstats = (int)l.nstats;
        a.g = gs;
        a.ldg = l.ld;
        a.y = targets + s0;
        a.token_loss = tl + s0;
        a.n_valid = n_valid;
        a.V = V;
        a.ignore = ignore_index;
        launch(sl::row_kernel, S, sl::kRowThreads, 0, st, a);
        if ((e = launch_status()) != LEMO_OK) return e;
        // dh_seg [S, d] = dz [S, V] . W [V, d]  (W read N-contiguous: MN-major B)
        if (dh && (e = run_gemm(dev, sms, st, gs, l.ld, false, w, ld_w, true, S, d, V,
                                gm::kStoreBF16, dh + s0 * ld_dh, ld_dh, true)) != LEMO_OK)
            return e;
        // dW [V, d] += dz^T [V, K] . h [K, d] over the rows of this segment and
        // the ones before it since the last dW GEMM (the dz slots hold
        // consecutive rows), both read MN-major; after every kDwSegs-th
        // segment and after the last one
        const bool last = s0 + seg_rows >= T;
        if (dw && (hb == l.dz_segs - 1 || last)) {
            const int64_t p0 = s0 - (int64_t)hb * seg_rows;
            const int K = (int)(s0 + S - p0);
            if ((e = run_gemm(dev, sms, st, g, l.ld, true, h + p0 * ld_h, ld_h, true, V, d, K,
                              gm::kAddF32, dw, ld_dw, false)) != LEMO_OK)
                return e;
        }
    }
    launch(sl::loss_kernel, 1, sl::kCountThreads, 0, st, tl, T, n_valid, loss);
    return launch_status();
}

lemo_status lemo_get_error(lemo_stream stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return LEMO_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, lemo::g_error, sizeof(v)) != cudaSuccess) return LEMO_ERR_CUDA;
    if (v != 0) {
        const unsigned int z = 0;
        if (cudaMemcpyToSymbol(lemo::g_error, &z, sizeof(z)) != cudaSuccess) return LEMO_ERR_CUDA;
    }
    return static_cast<lemo_status>(v);
}

void lemo_set_predict_test_hook(int32_t skip_cta) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_predict_skip_cta = skip_cta < 0 ? -1 : skip_cta;
}

void lemo_set_test_hooks(int32_t select_skip_publish_tile, int64_t spin_limit_ns) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_skip_publish_tile = select_skip_publish_tile < 0 ? -1 : select_skip_publish_tile;
    g_spin_ns = spin_limit_ns > 0 ? spin_limit_ns : kDefaultSpinNs;
}

}  // extern "C"
