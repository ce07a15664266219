// lemo.cu - host side of liblemo.so: argument checks, workspace layout,
// tensor-map encoding and launches.  The kernels live in the included .cuh
// files; everything is one translation unit so that the device error word is
// a single symbol per device.
#include <cublas_v2.h>  // types only: cuBLAS itself is opened with dlopen on first use
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <dlfcn.h>

#include <climits>
#include <mutex>
#include <utility>

#include "lemo.h"
#include "attn.cuh"
#include "common.cuh"
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
                 cudaStream_t st, float* zero_blocks = nullptr) {
    launch(lemo::plan_kernel, 1, 1024, 0, st, s->cu_seqlens, s->batch, s->total_L, s->max_seqlen,
           s->block, ws, lay, zero_word, zero_blocks);
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
    // byte offsets: block-mean planes, padded weight planes, split-K
    // partials, hidden-activation planes, Qhat / Khat planes, partial products
    size_t xb_hi, xb_lo, w1p[2], w2p[2], part, hid_hi, hid_lo, q_hi, q_lo, k_hi, k_lo, ppart, total;
    int ldr;         // rank padded to a multiple of 8
    int ldh;         // head dimension padded to a multiple of 8
    int64_t tb;      // upper bound of the number of token blocks
    int splits;      // split-K factor of the first predictor GEMM
    int k_chunk;     // K range of one split
    int hpg;         // heads per group of the block products
    int groups;      // head groups (partial planes when > 1)
    int64_t ptiles;  // lower-triangular 64 x 64 tiles of block pairs
};

// The launch shapes depend only on the shape (not on the device), so the
// workspace size query and the call agree.  The first GEMM is split along K
// until about four CTAs per SM of a B200 (148 SMs) are busy, with at least
// four K stages each: its loop is latency-bound, so shorter loops on more
// SMs finish sooner.  The block products aim at two CTAs per SM.
PredictLayout predict_layout(const lemo_shape* s, int d, int rank) {
    namespace pr = lemo::predict;
    constexpr int64_t kGemmCtas = 592, kTargetCtas = 296;
    PredictLayout p;
    p.base = layout_of(s);
    p.tb = ((int64_t)s->total_L + (int64_t)s->batch * (s->block - 1)) / s->block;
    if (p.tb < 1) p.tb = 1;
    p.ldr = (rank + 7) / 8 * 8;
    p.ldh = (s->dh + 7) / 8 * 8;
    const int64_t hdp = (int64_t)s->H * p.ldh;
    const int64_t mt = (p.tb + pr::TM - 1) / pr::TM;
    const int64_t tiles = 2 * ((p.ldr + pr::TN - 1) / pr::TN) * mt;
    const int64_t kst = (d + pr::TK - 1) / pr::TK;        // K stages of the first GEMM
    int64_t splits = (kGemmCtas + tiles - 1) / tiles;
    const int64_t max_splits = (kst + 3) / 4;              // at least 4 stages per split
    if (splits > max_splits) splits = max_splits;
    if (splits < 1) splits = 1;
    p.k_chunk = (int)((kst + splits - 1) / splits * pr::TK);
    p.splits = (int)((d + p.k_chunk - 1) / p.k_chunk);
    p.ptiles = mt * (mt + 1) / 2;
    int64_t groups = (kTargetCtas + p.ptiles - 1) / p.ptiles;
    if (groups > s->H) groups = s->H;
    while (groups > 1 && groups * p.tb * p.tb * 4 > ((int64_t)64 << 20)) --groups;
    if (groups < 1) groups = 1;
    p.hpg = (int)((s->H + groups - 1) / groups);
    p.groups = (s->H + p.hpg - 1) / p.hpg;
    size_t off = p.base.total;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = lemo::align_up(off + bytes, 256);
        return o;
    };
    p.xb_hi = take(2 * (size_t)p.tb * d);
    p.xb_lo = take(2 * (size_t)p.tb * d);
    for (int i = 0; i < 2; ++i) p.w1p[i] = take(2 * (size_t)d * p.ldr);
    for (int i = 0; i < 2; ++i) p.w2p[i] = take(2 * (size_t)p.ldr * hdp);
    p.part = take(4 * (size_t)2 * p.splits * p.tb * p.ldr);
    p.hid_hi = take(2 * (size_t)2 * p.tb * p.ldr);
    p.hid_lo = take(2 * (size_t)2 * p.tb * p.ldr);
    p.q_hi = take(2 * (size_t)p.tb * hdp);
    p.q_lo = take(2 * (size_t)p.tb * hdp);
    p.k_hi = take(2 * (size_t)p.tb * hdp);
    p.k_lo = take(2 * (size_t)p.tb * hdp);
    p.ppart = off;
    if (p.groups > 1) off = lemo::align_up(off + 4 * (size_t)p.groups * p.tb * p.tb, 256);
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

// ---------------------------------------------------------------------------
// cuBLAS for the plain GEMMs of the segmented loss, opened on first use so
// that the rest of the library does not depend on it.
// ---------------------------------------------------------------------------
struct Blas {
    using Create = cublasStatus_t (*)(cublasHandle_t*);
    using SetStream = cublasStatus_t (*)(cublasHandle_t, cudaStream_t);
    using SetWorkspace = cublasStatus_t (*)(cublasHandle_t, void*, size_t);
    using GemmEx = cublasStatus_t (*)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int,
                                      int, const void*, const void*, cudaDataType, int, const void*,
                                      cudaDataType, int, const void*, void*, cudaDataType, int,
                                      cublasComputeType_t, cublasGemmAlgo_t);
    bool tried = false;
    Create create = nullptr;
    SetStream set_stream = nullptr;
    SetWorkspace set_workspace = nullptr;
    GemmEx gemm = nullptr;
    cublasHandle_t handle[kMaxDevices] = {};
};
Blas g_blas;
constexpr size_t kBlasWorkspace = 32u << 20;

// Handle of device `dev` (created on first use), or nullptr if cuBLAS is
// unavailable.  Caller holds g_mu.
cublasHandle_t blas_handle(int dev) {
    Blas& b = g_blas;
    if (!b.tried) {
        b.tried = true;
        void* lib = dlopen("libcublas.so.12", RTLD_NOW | RTLD_GLOBAL);
        if (lib) {
            b.create = reinterpret_cast<Blas::Create>(dlsym(lib, "cublasCreate_v2"));
            b.set_stream = reinterpret_cast<Blas::SetStream>(dlsym(lib, "cublasSetStream_v2"));
            b.set_workspace = reinterpret_cast<Blas::SetWorkspace>(dlsym(lib, "cublasSetWorkspace_v2"));
            b.gemm = reinterpret_cast<Blas::GemmEx>(dlsym(lib, "cublasGemmEx"));
        }
    }
    if (!b.create || !b.set_stream || !b.set_workspace || !b.gemm) return nullptr;
    if (!b.handle[dev] && b.create(&b.handle[dev]) != CUBLAS_STATUS_SUCCESS) b.handle[dev] = nullptr;
    return b.handle[dev];
}

// Workspace of lemo_segment_loss.
struct SegLayout {
    size_t n_valid, token_loss, blas, z, g, total;
    int64_t ld;    // row stride of the segment's logits and gradient
    int64_t rows;  // rows of one segment buffer
};

SegLayout seg_layout(int64_t T, int V, int seg_rows) {
    SegLayout l;
    l.ld = ((int64_t)V + 7) / 8 * 8;
    l.rows = T < seg_rows ? (T > 0 ? T : 1) : seg_rows;
    size_t off = 0;
    l.n_valid = off; off = lemo::align_up(off + 4, 256);
    l.token_loss = off; off = lemo::align_up(off + 4 * (size_t)(T > 0 ? T : 1), 256);
    l.blas = off; off = lemo::align_up(off + kBlasWorkspace, 256);
    l.z = off; off = lemo::align_up(off + 4 * (size_t)l.rows * l.ld, 256);
    l.g = off; off = lemo::align_up(off + 2 * (size_t)l.rows * l.ld, 256);
    l.total = off;
    return l;
}

bool seg_args_ok(int64_t T, int V, int seg_rows) {
    return T >= 0 && T <= INT_MAX && V >= 1 && seg_rows >= 1 && (int64_t)V + 7 <= INT_MAX;
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

lemo_status lemo_score_blocks(const lemo_shape* shape, const uint16_t* q, const uint16_t* k,
                              float scale, float* block_max, float* block_scores, void* ws,
                              size_t ws_bytes, lemo_stream stream) {
    lemo_status e = check_shape(shape, true);
    if (e != LEMO_OK) return e;
    if (!q || !k || !block_scores) return LEMO_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(block_scores, 4) ||
        (block_max && !aligned(block_max, 4)))
        return LEMO_ERR_INVALID_ARG;
    if (!(scale > 0.f) || scale == __builtin_inff()) return LEMO_ERR_INVALID_ARG;
    if ((e = check_ws(shape, ws, ws_bytes)) != LEMO_OK) return e;
    int dev = 0;
    const int sms = device_sms(&dev);
    if (sms <= 0) return LEMO_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const lemo::WsLayout lay = layout_of(shape);
    char* w = static_cast<char*>(ws);
    float* mblk = block_max ? block_max : reinterpret_cast<float*>(w + lay.mblk);

    launch_plan(shape, w, lay, nullptr, st);
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
        launch(sc::score_tiles_kernel, 2 * pairs, sc::THREADS, sc::SMEM_BYTES, st, tm_q, tm_k, a);
        if ((e = launch_status()) != LEMO_OK) return e;
        // one warp per token block; the host knows an upper bound of their number
        const int64_t nb_bound =
            ((int64_t)shape->total_L + (int64_t)shape->batch * (shape->block - 1)) / shape->block;
        const int64_t cs_ctas = (nb_bound + 7) / 8;
        const int cs_grid = (int)(cs_ctas < (int64_t)sms * 8 ? (cs_ctas > 0 ? cs_ctas : 1) : sms * 8);
        launch(sc::column_sum_kernel, cs_grid, 256, 0, st, mblk, w, lay, shape->batch,
               block_scores);
        if ((e = launch_status()) != LEMO_OK) return e;
    }
    return LEMO_OK;
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
    if (ws_bytes < p.total) return LEMO_ERR_INVALID_ARG;
    int dev = 0;
    const int sms = device_sms(&dev);
    if (sms <= 0) return LEMO_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* w = static_cast<char*>(ws);
    const lemo::WsLayout& lay = p.base;
    const lemo::PlanHeader* hdr = reinterpret_cast<const lemo::PlanHeader*>(w + lay.hdr);
    float* part = reinterpret_cast<float*>(w + p.part);
    float* P = reinterpret_cast<float*>(w + lay.mblk);
    auto plane = [&](size_t off) { return reinterpret_cast<uint16_t*>(w + off); };
    const int hdp = shape->H * p.ldh;  // columns of the Qhat / Khat planes (heads padded)

    launch_plan(shape, w, lay, nullptr, st);
    if ((e = launch_status()) != LEMO_OK) return e;
    if (shape->total_L == 0) return LEMO_OK;
    // weights whose rows are not 16-byte aligned: padded copies
    const bool w1_vec16 = rank % 8 == 0 && aligned(w1q, 16) && aligned(w1k, 16);
    const bool w1_vec4 = !w1_vec16 && rank % 2 == 0 && aligned(w1q, 4) && aligned(w1k, 4);
    const bool pad_w1 = !w1_vec16 && !w1_vec4;
    const bool pad_w2 = shape->dh % 8 != 0 || !aligned(w2q, 16) || !aligned(w2k, 16);
    if (pad_w1) {
        pr::PadArgs pa1 = {};
        pa1.src[0] = w1q;
        pa1.src[1] = w1k;
        pa1.dst[0] = plane(p.w1p[0]);
        pa1.dst[1] = plane(p.w1p[1]);
        pa1.rows = pa1.rows_out = d;
        pa1.cols = pa1.run = rank;
        pa1.run_ld = p.ldr;
        pa1.ld_out = p.ldr;
        launch(pr::pad_kernel, dim3((unsigned)((d + 7) / 8), 2u), 256, 0, st, pa1);
    }
    if (pad_w2) {
        pr::PadArgs pa2 = {};
        pa2.src[0] = w2q;
        pa2.src[1] = w2k;
        pa2.dst[0] = plane(p.w2p[0]);
        pa2.dst[1] = plane(p.w2p[1]);
        pa2.rows = pa2.rows_out = rank;
        pa2.cols = shape->H * shape->dh;
        pa2.run = shape->dh;
        pa2.run_ld = p.ldh;
        pa2.ld_out = hdp;
        launch(pr::pad_kernel, dim3((unsigned)((rank + 7) / 8), 2u), 256, 0, st, pa2);
    }
    const uint16_t* w1s[2] = {pad_w1 ? plane(p.w1p[0]) : w1q, pad_w1 ? plane(p.w1p[1]) : w1k};
    const uint16_t* w2s[2] = {pad_w2 ? plane(p.w2p[0]) : w2q, pad_w2 ? plane(p.w2p[1]) : w2k};
    // block means, as hi / lo planes
    launch(pr::pool_kernel,
           dim3((unsigned)p.tb, (unsigned)((d + pr::kPoolCols - 1) / pr::kPoolCols)),
           pr::kPoolThreads, 0, st, x, ld_x, d, shape->cu_seqlens, shape->batch, shape->block, w,
           lay, plane(p.xb_hi), plane(p.xb_lo));
    if ((e = launch_status()) != LEMO_OK) return e;
    const unsigned mtiles = (unsigned)((p.tb + pr::TM - 1) / pr::TM);
    // hidden layers of both predictors: split-K partials, then relu of their sum
    pr::GemmArgs g1 = {};
    g1.a_hi[0] = g1.a_hi[1] = plane(p.xb_hi);
    g1.a_lo[0] = g1.a_lo[1] = plane(p.xb_lo);
    g1.lda = d;
    g1.w[0] = w1s[0];
    g1.w[1] = w1s[1];
    g1.ldw = pad_w1 ? p.ldr : rank;
    g1.c[0] = part;
    g1.c[1] = part + (int64_t)p.splits * p.tb * p.ldr;
    g1.ldc = p.ldr;
    g1.c_split = p.tb * p.ldr;
    g1.hdr = hdr;
    g1.N = p.ldr;
    g1.K = d;
    g1.w_rows = d;
    g1.w_cols = pad_w1 ? p.ldr : rank;
    g1.w_vec4 = w1_vec4;
    g1.k_chunk = p.k_chunk;
    g1.splits = p.splits;
    launch(pr::gemm_kernel<false>,
           dim3((unsigned)((p.ldr + pr::TN - 1) / pr::TN), mtiles, 2u * p.splits), pr::kMmaThreads,
           0, st, g1);
    launch(pr::reduce_kernel, dim3((unsigned)sms, 2u), 256, 0, st, part,
           (int64_t)p.splits * p.tb * p.ldr, p.tb * p.ldr, p.splits, hdr, p.ldr, plane(p.hid_hi),
           plane(p.hid_lo), p.tb * p.ldr);
    // block embeddings of both predictors, as hi / lo planes
    pr::GemmArgs g2 = {};
    g2.a_hi[0] = plane(p.hid_hi);
    g2.a_hi[1] = plane(p.hid_hi) + p.tb * p.ldr;
    g2.a_lo[0] = plane(p.hid_lo);
    g2.a_lo[1] = plane(p.hid_lo) + p.tb * p.ldr;
    g2.lda = p.ldr;
    g2.w[0] = w2s[0];
    g2.w[1] = w2s[1];
    g2.ldw = hdp;
    g2.c_hi[0] = plane(p.q_hi);
    g2.c_lo[0] = plane(p.q_lo);
    g2.c_hi[1] = plane(p.k_hi);
    g2.c_lo[1] = plane(p.k_lo);
    g2.ldc = hdp;
    g2.c_split = 0;
    g2.hdr = hdr;
    g2.N = hdp;
    g2.K = p.ldr;
    g2.w_rows = rank;
    g2.w_cols = hdp;
    g2.w_vec4 = false;
    g2.k_chunk = (p.ldr + pr::TK - 1) / pr::TK * pr::TK;
    g2.splits = 1;
    launch(pr::gemm_kernel<true>, dim3((unsigned)((hdp + pr::TN - 1) / pr::TN), mtiles, 2u),
           pr::kMmaThreads, 0, st, g2);
    if ((e = launch_status()) != LEMO_OK) return e;
    // block products, mean over heads of the positive parts
    pr::ProductsArgs pa;
    pa.q_hi = plane(p.q_hi);
    pa.q_lo = plane(p.q_lo);
    pa.k_hi = plane(p.k_hi);
    pa.k_lo = plane(p.k_lo);
    pa.H = shape->H;
    pa.ldh = p.ldh;
    pa.hpg = p.hpg;
    pa.groups = p.groups;
    pa.batch = shape->batch;
    pa.tb_cap = p.tb;
    pa.inv_h = 1.f / (float)shape->H;
    pa.part = reinterpret_cast<float*>(w + p.ppart);
    pa.P = P;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_prod_smem_set[dev]) {
            if (cudaFuncSetAttribute(pr::products_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     pr::PROD_SMEM) != cudaSuccess)
                return LEMO_ERR_CUDA;
            g_prod_smem_set[dev] = true;
        }
    }
    launch(pr::products_kernel, dim3((unsigned)p.ptiles, (unsigned)p.groups), pr::kMmaThreads,
           pr::PROD_SMEM, st, pa, w, lay);
    if ((e = launch_status()) != LEMO_OK) return e;
    if (p.groups > 1) launch(pr::products_reduce_kernel, sms * 2, 256, 0, st, pa, w, lay);
    const int64_t cs_ctas = (p.tb + 7) / 8;
    const int cs_grid = (int)(cs_ctas < (int64_t)sms * 8 ? cs_ctas : sms * 8);
    launch(lemo::score::column_sum_kernel, cs_grid, 256, 0, st, P, w, lay, shape->batch,
           block_scores);
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
    launch(at::attn_kernel, (unsigned)(items * shape->H), at::THREADS, at::SMEM_BYTES, st, tq, tk,
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
    if (device_sms(&dev) <= 0) return LEMO_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    char* wsp = static_cast<char*>(ws);
    int32_t* n_valid = reinterpret_cast<int32_t*>(wsp + l.n_valid);
    float* tl = token_loss ? token_loss : reinterpret_cast<float*>(wsp + l.token_loss);
    float* z = reinterpret_cast<float*>(wsp + l.z);
    uint16_t* g = reinterpret_cast<uint16_t*>(wsp + l.g);

    // The handle's stream and workspace are per call: hold the lock until
    // every GEMM of this call is enqueued.
    std::lock_guard<std::mutex> lk(g_mu);
    cublasHandle_t hb = nullptr;
    if (T > 0) {
        hb = blas_handle(dev);
        if (!hb) return LEMO_ERR_UNSUPPORTED;
        if (g_blas.set_stream(hb, st) != CUBLAS_STATUS_SUCCESS ||
            g_blas.set_workspace(hb, wsp + l.blas, kBlasWorkspace) != CUBLAS_STATUS_SUCCESS)
            return LEMO_ERR_CUDA;
    }
    launch(sl::count_kernel, 1, sl::kCountThreads, 0, st, targets, T, V, ignore_index, n_valid);
    lemo_status e = launch_status();
    if (e != LEMO_OK) return e;
    const float one = 1.f, zero = 0.f;
    for (int64_t s0 = 0; s0 < T; s0 += seg_rows) {
        const int S = (int)(T - s0 < seg_rows ? T - s0 : seg_rows);
        const uint16_t* hs = h + s0 * ld_h;
        // z^T [V, S] = W [V, d] . h_seg^T   (column-major view of row-major z [S, ld])
        if (g_blas.gemm(hb, CUBLAS_OP_T, CUBLAS_OP_N, V, S, d, &one, w, CUDA_R_16BF, (int)ld_w, hs,
                        CUDA_R_16BF, (int)ld_h, &zero, z, CUDA_R_32F, (int)l.ld, CUBLAS_COMPUTE_32F,
                        CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
            return LEMO_ERR_CUDA;
        sl::RowArgs a;
        a.z = z;
        a.ldz = l.ld;
        a.g = g;
        a.ldg = l.ld;
        a.y = targets + s0;
        a.token_loss = tl + s0;
        a.n_valid = n_valid;
        a.V = V;
        a.ignore = ignore_index;
        launch(sl::row_kernel, S, sl::kRowThreads, 0, st, a);
        if ((e = launch_status()) != LEMO_OK) return e;
        // dh_seg^T [d, S] = W^T [d, V] . dz^T [V, S]
        if (dh && g_blas.gemm(hb, CUBLAS_OP_N, CUBLAS_OP_N, d, S, V, &one, w, CUDA_R_16BF, (int)ld_w,
                              g, CUDA_R_16BF, (int)l.ld, &zero, dh + s0 * ld_dh, CUDA_R_16BF,
                              (int)ld_dh, CUBLAS_COMPUTE_32F,
                              CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
            return LEMO_ERR_CUDA;
        // dW^T [d, V] += h_seg^T [d, S] . dz [S, V]
        if (dw && g_blas.gemm(hb, CUBLAS_OP_N, CUBLAS_OP_T, d, V, S, &one, hs, CUDA_R_16BF, (int)ld_h,
                              g, CUDA_R_16BF, (int)l.ld, &one, dw, CUDA_R_32F, (int)ld_dw,
                              CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
            return LEMO_ERR_CUDA;
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

void lemo_set_test_hooks(int32_t select_skip_publish_tile, int64_t spin_limit_ns) {
    std::lock_guard<std::mutex> lk(g_mu);
    g_skip_publish_tile = select_skip_publish_tile < 0 ? -1 : select_skip_publish_tile;
    g_spin_ns = spin_limit_ns > 0 ? spin_limit_ns : kDefaultSpinNs;
}

}  // extern "C"
