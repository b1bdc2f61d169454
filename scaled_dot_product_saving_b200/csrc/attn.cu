// attn.cu -- the C ABI declared in include/attn.h: argument checks, workspace
// carving, TMA descriptors, kernel-path choice and launches. All kernels are
// compiled into this one translation unit.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>

#include "attn.h"
#include "sm100.cuh"
#include "simt.cuh"
#include "prep.cuh"
#include "fwd_tc.cuh"
#include "bwd_tc.cuh"
#include "kv_tc.cuh"
#include "dq_tc.cuh"
#include "gemm_tc.cuh"
#include "proj.cuh"
#include "f32x_tc.cuh"

namespace {

constexpr unsigned long long kWaitBudgetNs = 2000000000ull;   // 2 s per bounded wait
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kTile = 128;
constexpr int kSimtMaxHeads = 65535;   // the CUDA-core kernels put B*H in gridDim.y

// Per host thread: the kernel path a thread selected, and the launch count of
// its last call (the trace state below is per thread too), so calls from
// different threads never share mutable library state.
thread_local int g_path = ATTN_PATH_AUTO;
thread_local int g_dq_path = ATTN_DQ_AUTO;
thread_local int g_last_launches = 0;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

attn_status_t check_sizes(int B, int H, int n, int m, int d, int dv, attn_dtype_t dtype,
                          int causal) {
    if (dtype != ATTN_F32 && dtype != ATTN_BF16) return ATTN_ERR_DTYPE;
    if (B < 1 || H < 1 || n < 1 || m < 1 || d < 1 || dv < 1) return ATTN_ERR_SHAPE;
    if (static_cast<long long>(B) * H >= (1ll << 31)) return ATTN_ERR_SHAPE;
    if (n >= (1 << 24) || m >= (1 << 24)) return ATTN_ERR_SHAPE;
    if (causal && n != m) return ATTN_ERR_SHAPE;
    if (d > attn::simt::kMaxWidth || dv > attn::simt::kMaxWidth) return ATTN_ERR_UNSUPPORTED;
    return ATTN_OK;
}

enum class Path { kSimt, kTensorBf16, kTensorF32x };

bool tensor_path_fits(attn_dtype_t dtype, int d, int dv) {
    return dtype == ATTN_BF16 && d == dv && (d == 64 || d == 128);
}

// fp32 on the tensor cores by bf16 pieces: widths padded to 64 columns,
// 16-byte row loads.
bool f32x_path_fits(attn_dtype_t dtype, int d, int dv) {
    return dtype == ATTN_F32 && d <= attn::f32x::kWidth && dv <= attn::f32x::kWidth &&
           d % 4 == 0 && dv % 4 == 0;
}

// Decide the path; ATTN_OK and *path set, or an error.
attn_status_t choose_path(attn_dtype_t dtype, int d, int dv, Path* path) {
    const int p = g_path;
    const bool bf16 = tensor_path_fits(dtype, d, dv);
    const bool f32x = f32x_path_fits(dtype, d, dv);
    if (p == ATTN_PATH_TENSOR && !bf16 && !f32x) return ATTN_ERR_UNSUPPORTED;
    if (p == ATTN_PATH_SIMT || (!bf16 && !f32x)) *path = Path::kSimt;
    else *path = bf16 ? Path::kTensorBf16 : Path::kTensorF32x;
    return ATTN_OK;
}

// The key padding mask as the kernels take it: valid keys per batch element
// (device int32 [B], or null for none) and the head count that maps a
// (batch, head) index to its batch element.
struct Mask {
    const int* key_len;
    int H;
};

// Backward workspace: base-2 LSE and D ([BH, n_pad] fp32 each), the fp32 dQ
// accumulator [BH, n, d], then the tensor-core backwards' counters (int32):
// work-item and converter-claim counters in the first 256 bytes, then one
// count of landed work items per head. Every region starts on a 256-byte
// boundary.
struct Workspace {
    size_t lse2_off, dd_off, dq_off, cnt_off, n_counters, total;
    int n_pad;
};


Workspace carve(int B, int H, int n, int d) {
    Workspace w;
    const size_t bh = static_cast<size_t>(B) * H;
    w.n_pad = static_cast<int>(round_up(static_cast<size_t>(n), kTile));
    const size_t row_bytes = round_up(bh * w.n_pad * sizeof(float), 256);
    w.lse2_off = 0;
    w.dd_off = row_bytes;
    w.dq_off = 2 * row_bytes;
    w.cnt_off = w.dq_off + round_up(bh * static_cast<size_t>(n) * d * sizeof(float), 256);
    w.n_counters = attn::bwdtc::kCntHeadBase + bh;
    w.total = w.cnt_off + round_up(w.n_counters * sizeof(int), 256);
    return w;
}

// ---------------------------------------------------------------- TMA maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [BH, rows, width] viewed as 3-D (width innermost) with the 128-byte swizzle.
// bf16 operand tiles use boxes of 64 x 128 x 1 (the layout the UMMA
// descriptors expect); the fp32 dQ accumulator uses 32 x 32 x 1 boxes for the
// dQ warpgroup's reduce-adds.
bool make_map_typed(CUtensorMap* map, const void* base, int width, int rows, int bh,
                    CUtensorMapDataType type, int elem_bytes, int box_x, int box_y) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(width), static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(bh)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(width) * elem_bytes,
                             static_cast<cuuint64_t>(width) * elem_bytes * rows};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(box_x), static_cast<cuuint32_t>(box_y), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, type, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A bf16 matrix of `rows` x `width` whose rows are `row_stride` elements apart,
// viewed as [1, rows, width] with the 128-byte swizzle and box_x x box_y boxes.
bool make_map_rows(CUtensorMap* map, const void* base, int width, int rows, size_t row_stride,
                   int box_x, int box_y) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(width), static_cast<cuuint64_t>(rows), 1};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_stride) * 2,
                             static_cast<cuuint64_t>(row_stride) * 2 * rows};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(box_x), static_cast<cuuint32_t>(box_y), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map(CUtensorMap* map, const void* base, int width, int rows, int bh) {
    return make_map_typed(map, base, width, rows, bh, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 64,
                          kTile);
}

// ---------------------------------------------------------------- tracing
struct TraceEntry {
    int kernel;
    cudaEvent_t start, stop;
};
struct TraceState {
    bool on = false;
    int capacity = 0;
    std::vector<TraceEntry> entries;
    std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pool;   // reused across sessions
};
thread_local TraceState g_trace;

// Launch through `launch()`, bracketed by events when tracing is on.
template <typename F>
attn_status_t traced(int kernel, cudaStream_t st, F&& launch) {
    TraceState& t = g_trace;
    if (!t.on || static_cast<int>(t.entries.size()) >= t.capacity) return launch();
    const size_t k = t.entries.size();
    if (k == t.pool.size()) {
        cudaEvent_t a, b;
        if (cudaEventCreate(&a) != cudaSuccess) return launch();
        if (cudaEventCreate(&b) != cudaSuccess) {
            cudaEventDestroy(a);
            return launch();
        }
        t.pool.emplace_back(a, b);
    }
    TraceEntry e{kernel, t.pool[k].first, t.pool[k].second};
    cudaEventRecord(e.start, st);
    const attn_status_t s = launch();
    cudaEventRecord(e.stop, st);
    t.entries.push_back(e);
    return s;
}

inline attn_status_t launched() {
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Number of SMs of the current device (cached per device).
int sm_count() {
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cache[dev]) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v < 1)
            v = 148;
        cache[dev] = v;
    }
    return cache[dev];
}

int grid_for(size_t work_items, int per_block, int cap) {
    size_t g = (work_items + per_block - 1) / per_block;
    if (g < 1) g = 1;
    if (g > static_cast<size_t>(cap)) g = cap;
    return static_cast<int>(g);
}

template <typename T>
attn_status_t fwd_simt(const void* Q, const void* K, const void* V, void* O, float* LSE, int BH,
                       int n, int m, int d, int dv, int causal, float scale, Mask mask,
                       cudaStream_t st) {
    const size_t smem = attn::simt::fwd_smem_bytes<T>(d, dv);
    auto kern = attn::simt::fwd_kernel<T>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return ATTN_ERR_CUDA;
    dim3 grid((n + attn::simt::kTile - 1) / attn::simt::kTile, BH);
    return traced(ATTN_KERNEL_FWD_SIMT, st, [&] {
        kern<<<grid, attn::simt::kThreads, smem, st>>>(
            static_cast<const T*>(Q), static_cast<const T*>(K), static_cast<const T*>(V),
            static_cast<T*>(O), LSE, n, m, d, dv, causal, scale, mask.key_len, mask.H);
        return launched();
    });
}

template <int D>
attn_status_t fwd_tensor(const void* Q, const void* K, const void* V, void* O, float* LSE,
                         int BH, int n, int m, int causal, float scale, Mask mask,
                         cudaStream_t st) {
    using C = attn::fwdtc::Cfg<D>;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, Q, D, n, BH) || !make_map(&mk, K, D, m, BH) || !make_map(&mv, V, D, m, BH) ||
        !make_map_typed(&mo, O, D, n, BH, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 64, 32))
        return ATTN_ERR_CUDA;
    auto kern = attn::fwdtc::fwd_kernel<D>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess)
        return ATTN_ERR_CUDA;
    // One CTA per pair of adjacent query tiles (2p, 2p + 1) of one head; heads
    // in groups of about 256 CTAs.
    const int num_qt = (n + attn::fwdtc::kBM - 1) / attn::fwdtc::kBM;
    const int num_pairs = (num_qt + 1) / 2;
    const long long grid = static_cast<long long>(num_pairs) * BH;
    if (grid > 0x7fffffffll) return ATTN_ERR_SHAPE;
    const int head_group = std::max(1, std::min(BH, 256 / num_pairs));
    return traced(ATTN_KERNEL_FWD_TENSOR, st, [&] {
        kern<<<static_cast<unsigned>(grid), attn::fwdtc::kThreads, C::kSmemBytes, st>>>(
            mq, mk, mv, mo, LSE, n, m, BH, head_group, causal, scale * kLog2e, mask.key_len,
            mask.H, kWaitBudgetNs);
        return launched();
    });
}

template <typename T>
attn_status_t preprocess(const void* O, const void* dO, const float* LSE, float* lse2, float* Dd,
                         float* dQacc, int* counters, size_t n_counters, int BH, int n, int n_pad,
                         int d, int dv, float d_scale, bool zero_dq, cudaStream_t st) {
    const size_t rows = static_cast<size_t>(BH) * n_pad;
    const size_t dq_elems = zero_dq ? static_cast<size_t>(BH) * n * d : 0;
    const bool vec = sizeof(T) == 2 && dv % 8 == 0 && (dv / 8) <= 32 && 32 % (dv / 8) == 0 &&
                     dq_elems % 4 == 0;
    if (vec) {
        const int rows_per_block =
            (attn::prep::kThreads / 32) * (32 / (dv / 8)) * attn::prep::kRowsInFlight;
        const int grid = grid_for(rows, rows_per_block, sm_count() * attn::prep::kBlocksPerSm);
        return traced(ATTN_KERNEL_PREPROCESS, st, [&] {
            attn::prep::preprocess_bf16_vec<<<grid, attn::prep::kThreads, 0, st>>>(
                static_cast<const __nv_bfloat16*>(O), static_cast<const __nv_bfloat16*>(dO), LSE,
                lse2, Dd, dQacc, counters, n_counters, dq_elems, BH, n, n_pad, dv, d_scale);
            return launched();
        });
    }
    const int grid = grid_for(rows, attn::prep::kThreads / 32, 148 * 16);
    return traced(ATTN_KERNEL_PREPROCESS, st, [&] {
        attn::prep::preprocess_generic<T><<<grid, attn::prep::kThreads, 0, st>>>(
            static_cast<const T*>(O), static_cast<const T*>(dO), LSE, lse2, Dd, dQacc, counters,
            n_counters, dq_elems, BH, n, n_pad, dv, d_scale);
        return launched();
    });
}

template <typename T>
attn_status_t finalize(const float* dQacc, void* dQ, size_t elems, float post_scale,
                       cudaStream_t st) {
    const int grid = grid_for(elems / 4 + 1, attn::prep::kThreads, 148 * 16);
    return traced(ATTN_KERNEL_FINALIZE, st, [&] {
        attn::prep::finalize_dq<T><<<grid, attn::prep::kThreads, 0, st>>>(
            dQacc, static_cast<T*>(dQ), elems, post_scale);
        return launched();
    });
}

template <typename T>
attn_status_t bwd_simt(const void* Q, const void* K, const void* V, const void* dO,
                       const float* LSE, const float* Dd, int n_pad, float* dQacc, void* dK,
                       void* dV, int BH, int n, int m, int d, int dv, int causal, float scale,
                       Mask mask, cudaStream_t st) {
    const size_t smem = attn::simt::bwd_smem_bytes<T>(d, dv);
    auto kern = attn::simt::bwd_kernel<T>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return ATTN_ERR_CUDA;
    dim3 grid((m + attn::simt::kTile - 1) / attn::simt::kTile, BH);
    return traced(ATTN_KERNEL_BWD_SIMT, st, [&] {
        kern<<<grid, attn::simt::kThreads, smem, st>>>(
            static_cast<const T*>(Q), static_cast<const T*>(K), static_cast<const T*>(V),
            static_cast<const T*>(dO), LSE, Dd, n_pad, dQacc, static_cast<T*>(dK),
            static_cast<T*>(dV), n, m, d, dv, causal, scale, mask.key_len, mask.H);
        return launched();
    });
}

template <int D>
attn_status_t bwd_tensor(const void* Q, const void* K, const void* V, const void* dO,
                         const float* lse2, const float* Dd, int* counters, int n_pad, float* dQacc,
                         void* dQ, void* dK, void* dV, int BH, int n, int m, int causal, float scale,
                         Mask mask, cudaStream_t st) {
    using C = attn::bwdtc::Cfg<D>;
    CUtensorMap mq, mk, mv, mdo, mdq, mdk, mdv;
    if (!make_map(&mq, Q, D, n, BH) || !make_map(&mk, K, D, m, BH) ||
        !make_map(&mv, V, D, m, BH) || !make_map(&mdo, dO, D, n, BH) ||
        !make_map_typed(&mdq, dQacc, D, n, BH, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 32, 32) ||
        !make_map_typed(&mdk, dK, D, m, BH, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 64, 32) ||
        !make_map_typed(&mdv, dV, D, m, BH, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 64, 32))
        return ATTN_ERR_CUDA;
    auto kern = attn::bwdtc::bwd_kernel<D>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess)
        return ATTN_ERR_CUDA;
    // Persistent: one CTA per SM (at most one per work item), each walking
    // the work items (key tile, head) with a stride of the grid size; heads
    // per scheduling group: about 256 items a group.
    const int num_kt = (m + kTile - 1) / kTile;
    const long long items = static_cast<long long>(num_kt) * BH;
    if (items > 0x7fffffffll) return ATTN_ERR_SHAPE;          // the kernel counts items in int
    const int grid = static_cast<int>(std::min<long long>(items, sm_count()));
    const int head_group = std::max(1, std::min(BH, 256 / num_kt));
    // A programmatic dependent of the preprocess kernel launched just before
    // it on the stream: launched early, it waits for that kernel's results in
    // the kernel (griddepcontrol); its CTAs need an SM's whole register file,
    // so they start as the preprocess CTAs leave. Not while tracing: the early
    // start would then be counted in this kernel's time.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(attn::bwdtc::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = g_trace.on ? 0 : 1;
    __nv_bfloat16* dq16 = static_cast<__nv_bfloat16*>(dQ);
    const float scale_log2 = scale * kLog2e;
    const int* key_len = mask.key_len;
    return traced(ATTN_KERNEL_BWD_TENSOR, st, [&] {
        if (cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mdo, mdq, mdk, mdv, lse2, Dd, counters, dQacc,
                               dq16, n_pad, n, m, BH, head_group, causal, scale, scale_log2,
                               key_len, mask.H, kWaitBudgetNs) != cudaSuccess) {
            (void)cudaGetLastError();
            return ATTN_ERR_CUDA;
        }
        return launched();
    });
}

// The bf16 backward as two passes (ATTN_DQ_SEPARATE): dK/dV key-tile major,
// then dQ query-tile major, each persistent with one CTA per SM and its own
// work counter.
template <int D>
attn_status_t bwd_separate(const void* Q, const void* K, const void* V, const void* dO,
                           const float* lse2, const float* Dd, int* counters, int n_pad, void* dQ,
                           void* dK, void* dV, int BH, int n, int m, int causal, float scale,
                           Mask mask, cudaStream_t st) {
    CUtensorMap mq, mk, mv, mdo, mdk, mdv;
    if (!make_map(&mq, Q, D, n, BH) || !make_map(&mk, K, D, m, BH) ||
        !make_map(&mv, V, D, m, BH) || !make_map(&mdo, dO, D, n, BH) ||
        !make_map_typed(&mdk, dK, D, m, BH, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 64, 32) ||
        !make_map_typed(&mdv, dV, D, m, BH, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 64, 32))
        return ATTN_ERR_CUDA;
    using CK = attn::kvtc::Cfg<D>;
    using CQ = attn::dqtc::Cfg<D>;
    auto kv = attn::kvtc::kv_kernel<D>;
    auto dq = attn::dqtc::dq_kernel<D>;
    if (cudaFuncSetAttribute(kv, cudaFuncAttributeMaxDynamicSharedMemorySize, CK::kSmemBytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(dq, cudaFuncAttributeMaxDynamicSharedMemorySize, CQ::kSmemBytes) !=
            cudaSuccess)
        return ATTN_ERR_CUDA;
    const int num_kt = (m + kTile - 1) / kTile, num_qt = (n + kTile - 1) / kTile;
    const long long kv_items = static_cast<long long>(num_kt) * BH;
    const long long dq_items = static_cast<long long>(num_qt) * BH;
    if (kv_items > 0x7fffffffll || dq_items > 0x7fffffffll) return ATTN_ERR_SHAPE;
    const int kv_grid = static_cast<int>(std::min<long long>(kv_items, sm_count()));
    const int dq_grid = static_cast<int>(std::min<long long>(dq_items, sm_count()));
    const int kv_hg = std::max(1, std::min(BH, 256 / num_kt));
    const int dq_hg = std::max(1, std::min(BH, 256 / num_qt));
    attn_status_t s = traced(ATTN_KERNEL_BWD_KV, st, [&] {
        kv<<<static_cast<unsigned>(kv_grid), attn::kvtc::kThreads, CK::kSmemBytes, st>>>(
            mq, mk, mv, mdo, mdk, mdv, lse2, Dd, counters + attn::bwdtc::kCntSched, n_pad, n, m, BH,
            kv_hg, causal, scale, scale * kLog2e, mask.key_len, mask.H, kWaitBudgetNs);
        return launched();
    });
    if (s != ATTN_OK) return s;
    return traced(ATTN_KERNEL_BWD_DQ, st, [&] {
        dq<<<static_cast<unsigned>(dq_grid), attn::dqtc::kThreads, CQ::kSmemBytes, st>>>(
            mq, mk, mv, mdo, lse2, Dd, counters + attn::bwdtc::kCntSchedDq,
            static_cast<__nv_bfloat16*>(dQ), n_pad, n, m, BH, dq_hg, causal, scale,
            scale * kLog2e, mask.key_len, mask.H, kWaitBudgetNs);
        return launched();
    });
}

// Which dQ design the bf16 tensor-core backward uses (ATTN_DQ_AUTO: the one
// measured faster).
bool dq_separate() {
    return g_dq_path == ATTN_DQ_SEPARATE;
}

// fp32 by bf16 pieces: one CTA per (128-row tile, head), heads fastest.
attn_status_t f32x_grid(int rows, int BH, unsigned* grid) {
    const long long g = static_cast<long long>((rows + attn::f32x::kBig - 1) / attn::f32x::kBig) * BH;
    if (g > 0x7fffffffll) return ATTN_ERR_SHAPE;
    *grid = static_cast<unsigned>(g);
    return ATTN_OK;
}

attn_status_t fwd_f32x(const void* Q, const void* K, const void* V, void* O, float* LSE, int BH,
                       int n, int m, int d, int dv, int causal, float scale, Mask mask,
                       cudaStream_t st) {
    namespace fx = attn::f32x;
    unsigned grid = 0;
    attn_status_t s = f32x_grid(n, BH, &grid);
    if (s != ATTN_OK) return s;
    if (cudaFuncSetAttribute(fx::fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fx::kFwdSmemBytes) != cudaSuccess)
        return ATTN_ERR_CUDA;
    return traced(ATTN_KERNEL_FWD_F32X, st, [&] {
        fx::fwd_kernel<<<grid, fx::kFwdThreads, fx::kFwdSmemBytes, st>>>(
            static_cast<const float*>(Q), static_cast<const float*>(K),
            static_cast<const float*>(V), static_cast<float*>(O), LSE, n, m, d, dv, BH, causal,
            scale * kLog2e, mask.key_len, mask.H, kWaitBudgetNs);
        return launched();
    });
}

attn_status_t bwd_f32x(const void* Q, const void* K, const void* V, const void* dO,
                       const float* lse2, const float* Dd, int n_pad, void* dQ, void* dK, void* dV,
                       int BH, int n, int m, int d, int dv, int causal, float scale, Mask mask,
                       cudaStream_t st) {
    namespace fx = attn::f32x;
    unsigned grid_kv = 0, grid_dq = 0;
    attn_status_t s = f32x_grid(m, BH, &grid_kv);
    if (s == ATTN_OK) s = f32x_grid(n, BH, &grid_dq);
    if (s != ATTN_OK) return s;
    if (static_cast<unsigned long long>(grid_kv) + grid_dq > 0x7fffffffull) return ATTN_ERR_SHAPE;
    if (cudaFuncSetAttribute(fx::bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fx::kBwdSmemBytes) != cudaSuccess)
        return ATTN_ERR_CUDA;
    // One launch: the dK/dV pass's CTAs first, then the dQ pass's.
    return traced(ATTN_KERNEL_BWD_F32X, st, [&] {
        fx::bwd_kernel<<<grid_kv + grid_dq, fx::kBwdThreads, fx::kBwdSmemBytes, st>>>(
            static_cast<const float*>(Q), static_cast<const float*>(K),
            static_cast<const float*>(V), static_cast<const float*>(dO), lse2, Dd, n_pad,
            static_cast<float*>(dQ), static_cast<float*>(dK), static_cast<float*>(dV), n, m, d, dv,
            BH, causal, scale, scale * kLog2e, mask.key_len, mask.H, static_cast<int>(grid_kv),
            kWaitBudgetNs);
        return launched();
    });
}

__global__ void probe_timeout_kernel(unsigned long long budget_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x == 0) {
        abort = 0;
        attn::mbar_init(&bar, 1);
        attn::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // Nothing ever arrives on `bar`: the wait must give up after budget_ns.
        if (!attn::mbar_wait(&bar, 0, &abort, budget_ns))
            attn::record_device_error(attn::kErrTimeout);
    }
}

}  // namespace

// ------------------------------------------------------ projection grads
struct ProjWorkspace {
    size_t acat_off, wcat_off, total;
    int wtot;
};

ProjWorkspace carve_proj(int B, int n, int d_model, int H, int d, int dv) {
    ProjWorkspace w;
    w.wtot = 2 * H * d + H * dv;
    w.acat_off = 0;
    w.wcat_off = round_up(static_cast<size_t>(B) * n * w.wtot * 2, 256);
    w.total = w.wcat_off + round_up(static_cast<size_t>(d_model) * w.wtot * 2, 256);
    return w;
}

attn_status_t check_proj(int B, int n, int d_model, int H, int d, int dv, attn_dtype_t dtype) {
    if (dtype != ATTN_F32 && dtype != ATTN_BF16) return ATTN_ERR_DTYPE;
    if (B < 1 || n < 1 || d_model < 1 || H < 1 || d < 1 || dv < 1) return ATTN_ERR_SHAPE;
    if (static_cast<long long>(B) * n >= (1ll << 31) || d_model >= (1 << 24) ||
        static_cast<long long>(H) * (2 * d + dv) >= (1 << 24))
        return ATTN_ERR_SHAPE;
    if (dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
    if (d % 8 || dv % 8 || d_model % 8) return ATTN_ERR_SHAPE;
    return ATTN_OK;
}

template <bool AK, bool BK>
attn_status_t gemm(const CUtensorMap& ma, const CUtensorMap& mb, void* D, int M, int N, int K,
                   int ldd, cudaStream_t st) {
    auto kern = attn::gemmtc::gemm_kernel<AK, BK>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             attn::gemmtc::kSmemBytes) != cudaSuccess)
        return ATTN_ERR_CUDA;
    const long long tiles = static_cast<long long>((M + attn::gemmtc::kBM - 1) / attn::gemmtc::kBM) *
                            ((N + attn::gemmtc::kBN - 1) / attn::gemmtc::kBN);
    if (tiles > 0x7fffffffll) return ATTN_ERR_SHAPE;
    const dim3 grid(static_cast<unsigned>(tiles));
    return traced(ATTN_KERNEL_GEMM, st, [&] {
        kern<<<grid, attn::gemmtc::kThreads, attn::gemmtc::kSmemBytes, st>>>(
            ma, mb, static_cast<__nv_bfloat16*>(D), M, N, K, ldd, kWaitBudgetNs);
        return launched();
    });
}

extern "C" {

attn_status_t attn_set_path(attn_path_t path) {
    if (path != ATTN_PATH_AUTO && path != ATTN_PATH_SIMT && path != ATTN_PATH_TENSOR)
        return ATTN_ERR_UNSUPPORTED;
    g_path = path;
    return ATTN_OK;
}

attn_status_t attn_set_dq_path(attn_dq_path_t path) {
    if (path != ATTN_DQ_AUTO && path != ATTN_DQ_REDUCE && path != ATTN_DQ_SEPARATE)
        return ATTN_ERR_UNSUPPORTED;
    g_dq_path = path;
    return ATTN_OK;
}

int attn_last_launch_count(void) { return g_last_launches; }

size_t attn_bwd_workspace_size(int B, int H, int n, int m, int d, int dv, attn_dtype_t dtype) {
    if (check_sizes(B, H, n, m, d, dv, dtype, 0) != ATTN_OK) return 0;
    return carve(B, H, n, d).total;
}

attn_status_t attn_fwd_masked(const void* Q, const void* K, const void* V, void* O, float* LSE,
                              const int* key_len, int B, int H, int n, int m, int d, int dv,
                              attn_dtype_t dtype, int causal, float scale, void* stream) {
    attn_status_t s = check_sizes(B, H, n, m, d, dv, dtype, causal);
    if (s != ATTN_OK) return s;
    if (!std::isfinite(scale)) return ATTN_ERR_SHAPE;
    if (!Q || !K || !V || !O || !LSE) return ATTN_ERR_NULL;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE) ||
        (reinterpret_cast<uintptr_t>(key_len) & 3u) != 0)
        return ATTN_ERR_ALIGN;
    Path path = Path::kSimt;
    if ((s = choose_path(dtype, d, dv, &path)) != ATTN_OK) return s;
    const int BH = B * H;
    if (path == Path::kSimt && BH > kSimtMaxHeads) return ATTN_ERR_UNSUPPORTED;
    const Mask mask{key_len, H};
    cudaStream_t st = as_stream(stream);
    if (path == Path::kTensorF32x)
        s = fwd_f32x(Q, K, V, O, LSE, BH, n, m, d, dv, causal, scale, mask, st);
    else if (path == Path::kTensorBf16)
        s = (d == 64) ? fwd_tensor<64>(Q, K, V, O, LSE, BH, n, m, causal, scale, mask, st)
                      : fwd_tensor<128>(Q, K, V, O, LSE, BH, n, m, causal, scale, mask, st);
    else if (dtype == ATTN_F32)
        s = fwd_simt<float>(Q, K, V, O, LSE, BH, n, m, d, dv, causal, scale, mask, st);
    else
        s = fwd_simt<__nv_bfloat16>(Q, K, V, O, LSE, BH, n, m, d, dv, causal, scale, mask, st);
    if (s == ATTN_OK) g_last_launches = 1;
    return s;
}

attn_status_t attn_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                       int H, int n, int m, int d, int dv, attn_dtype_t dtype, int causal,
                       float scale, void* stream) {
    return attn_fwd_masked(Q, K, V, O, LSE, nullptr, B, H, n, m, d, dv, dtype, causal, scale,
                           stream);
}

attn_status_t attn_bwd_masked(const void* Q, const void* K, const void* V, const void* O,
                              const void* dO, const float* LSE, const int* key_len, void* dQ,
                              void* dK, void* dV, void* workspace, size_t workspace_bytes, int B,
                              int H, int n, int m, int d, int dv, attn_dtype_t dtype, int causal,
                              float scale, void* stream) {
    attn_status_t s = check_sizes(B, H, n, m, d, dv, dtype, causal);
    if (s != ATTN_OK) return s;
    if (!std::isfinite(scale)) return ATTN_ERR_SHAPE;
    if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV) return ATTN_ERR_NULL;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) ||
        !aligned16(LSE) || !aligned16(dQ) || !aligned16(dK) || !aligned16(dV) ||
        (reinterpret_cast<uintptr_t>(key_len) & 3u) != 0)
        return ATTN_ERR_ALIGN;
    const Workspace w = carve(B, H, n, d);
    if (!workspace || workspace_bytes < w.total) return ATTN_ERR_WORKSPACE;
    if (!aligned16(workspace)) return ATTN_ERR_ALIGN;
    Path path = Path::kSimt;
    if ((s = choose_path(dtype, d, dv, &path)) != ATTN_OK) return s;
    const bool tensor = path != Path::kSimt;
    if (!tensor && static_cast<long long>(B) * H > kSimtMaxHeads) return ATTN_ERR_UNSUPPORTED;

    const int BH = B * H;
    const Mask mask{key_len, H};
    cudaStream_t st = as_stream(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* lse2 = reinterpret_cast<float*>(ws + w.lse2_off);
    float* Dd = reinterpret_cast<float*>(ws + w.dd_off);
    float* dQacc = reinterpret_cast<float*>(ws + w.dq_off);
    int* counters = reinterpret_cast<int*>(ws + w.cnt_off);
    const size_t dq_elems = static_cast<size_t>(BH) * n * d;

    // The tensor-core backwards take D already multiplied by the scale. The
    // paths that add dQ partials into the accumulator need it zeroed; the
    // fp32 tensor-core backward and the separate dQ pass write dQ once.
    const float d_scale = tensor ? scale : 1.0f;
    const bool separate = path == Path::kTensorBf16 && dq_separate();
    const bool zero_dq = path == Path::kSimt || (path == Path::kTensorBf16 && !separate);
    s = (dtype == ATTN_F32)
            ? preprocess<float>(O, dO, LSE, lse2, Dd, dQacc, counters, w.n_counters, BH, n,
                                w.n_pad, d, dv, d_scale, zero_dq, st)
            : preprocess<__nv_bfloat16>(O, dO, LSE, lse2, Dd, dQacc, counters, w.n_counters, BH,
                                        n, w.n_pad, d, dv, d_scale, zero_dq, st);
    if (s != ATTN_OK) return s;
    if (path == Path::kTensorF32x) {
        s = bwd_f32x(Q, K, V, dO, lse2, Dd, w.n_pad, dQ, dK, dV, BH, n, m, d, dv, causal, scale,
                     mask, st);
    } else if (path == Path::kTensorBf16 && separate) {
        s = (d == 64) ? bwd_separate<64>(Q, K, V, dO, lse2, Dd, counters, w.n_pad, dQ, dK, dV, BH,
                                         n, m, causal, scale, mask, st)
                      : bwd_separate<128>(Q, K, V, dO, lse2, Dd, counters, w.n_pad, dQ, dK, dV,
                                          BH, n, m, causal, scale, mask, st);
    } else if (path == Path::kTensorBf16) {
        s = (d == 64) ? bwd_tensor<64>(Q, K, V, dO, lse2, Dd, counters, w.n_pad, dQacc, dQ, dK,
                                       dV, BH, n, m, causal, scale, mask, st)
                      : bwd_tensor<128>(Q, K, V, dO, lse2, Dd, counters, w.n_pad, dQacc, dQ, dK,
                                        dV, BH, n, m, causal, scale, mask, st);
    } else if (dtype == ATTN_F32) {
        s = bwd_simt<float>(Q, K, V, dO, LSE, Dd, w.n_pad, dQacc, dK, dV, BH, n, m, d, dv, causal,
                            scale, mask, st);
        if (s == ATTN_OK) s = finalize<float>(dQacc, dQ, dq_elems, scale, st);
    } else {
        s = bwd_simt<__nv_bfloat16>(Q, K, V, dO, LSE, Dd, w.n_pad, dQacc, dK, dV, BH, n, m, d, dv,
                                    causal, scale, mask, st);
        if (s == ATTN_OK) s = finalize<__nv_bfloat16>(dQacc, dQ, dq_elems, scale, st);
    }
    if (s == ATTN_OK) g_last_launches = (path == Path::kTensorF32x || (tensor && !separate)) ? 2 : 3;
    return s;
}

attn_status_t attn_bwd(const void* Q, const void* K, const void* V, const void* O,
                       const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                       void* workspace, size_t workspace_bytes, int B, int H, int n, int m, int d,
                       int dv, attn_dtype_t dtype, int causal, float scale, void* stream) {
    return attn_bwd_masked(Q, K, V, O, dO, LSE, nullptr, dQ, dK, dV, workspace, workspace_bytes, B,
                           H, n, m, d, dv, dtype, causal, scale, stream);
}

attn_status_t attn_trace_begin(int capacity) {
    if (capacity < 1 || capacity > 65536) return ATTN_ERR_SHAPE;
    g_trace.on = true;
    g_trace.capacity = capacity;
    g_trace.entries.clear();
    return ATTN_OK;
}

int attn_trace_end(attn_kernel_time_t* out, int max_entries) {
    TraceState& t = g_trace;
    t.on = false;
    const int count = static_cast<int>(t.entries.size());
    int status = count;
    for (int k = 0; k < count; ++k) {
        const TraceEntry& e = t.entries[k];
        float ms = 0.f;
        if (cudaEventSynchronize(e.stop) != cudaSuccess ||
            cudaEventElapsedTime(&ms, e.start, e.stop) != cudaSuccess)
            status = -1;
        if (out && k < max_entries) {
            out[k].kernel = e.kernel;
            out[k].ms = ms;
        }
    }
    t.entries.clear();
    return status;
}

attn_status_t attn_get_device_error(void* stream) {
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, attn::g_device_error, sizeof(v)) != cudaSuccess)
        return ATTN_ERR_CUDA;
    if (v != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(attn::g_device_error, &zero, sizeof(zero)) != cudaSuccess)
            return ATTN_ERR_CUDA;
        return ATTN_ERR_DEVICE_TIMEOUT;
    }
    return ATTN_OK;
}

attn_status_t attn_probe_timeout(unsigned timeout_us, void* stream) {
    if (timeout_us < 1 || timeout_us > 1000000) return ATTN_ERR_SHAPE;
    probe_timeout_kernel<<<1, 32, 0, as_stream(stream)>>>(1000ull * timeout_us);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

size_t attn_proj_bwd_workspace_size(int B, int n, int d_model, int H, int d, int dv,
                                    attn_dtype_t dtype) {
    if (check_proj(B, n, d_model, H, d, dv, dtype) != ATTN_OK) return 0;
    return carve_proj(B, n, d_model, H, d, dv).total;
}

attn_status_t attn_proj_bwd(const void* X, const void* Wq, const void* Wk, const void* Wv,
                            const void* dQ, const void* dK, const void* dV, void* dX,
                            void* dWq, void* dWk, void* dWv, void* workspace,
                            size_t workspace_bytes, int B, int n, int d_model, int H, int d,
                            int dv, attn_dtype_t dtype, void* stream) {
    attn_status_t s = check_proj(B, n, d_model, H, d, dv, dtype);
    if (s != ATTN_OK) return s;
    const void* ins[7] = {X, Wq, Wk, Wv, dQ, dK, dV};
    void* outs[4] = {dX, dWq, dWk, dWv};
    for (const void* p : ins)
        if (!p) return ATTN_ERR_NULL;
    for (void* p : outs)
        if (!p) return ATTN_ERR_NULL;
    for (const void* p : ins)
        if (!aligned16(p)) return ATTN_ERR_ALIGN;
    for (void* p : outs)
        if (!aligned16(p)) return ATTN_ERR_ALIGN;
    const ProjWorkspace w = carve_proj(B, n, d_model, H, d, dv);
    if (!workspace || workspace_bytes < w.total) return ATTN_ERR_WORKSPACE;
    if (!aligned16(workspace)) return ATTN_ERR_ALIGN;

    cudaStream_t st = as_stream(stream);
    auto* acat = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(workspace) + w.acat_off);
    auto* wcat = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(workspace) + w.wcat_off);
    const int tokens = B * n;
    const int hd = H * d, hdv = H * dv;

    // Tensor maps first: nothing is launched unless all of them encode.
    // dX = A [Wq|Wk|Wv]^T: A K-major [tokens][wtot], B K-major [d_model][wtot].
    // dW = X^T A_block: A = X MN-major [tokens][d_model], B = the column block
    // of A MN-major [tokens][width], rows wtot apart.
    CUtensorMap m_acat, m_wcat, m_x, m_bq, m_bk, m_bv;
    if (!make_map_rows(&m_acat, acat, w.wtot, tokens, w.wtot, 64, attn::gemmtc::kBM) ||
        !make_map_rows(&m_wcat, wcat, w.wtot, d_model, w.wtot, 64, attn::gemmtc::kBN) ||
        !make_map_rows(&m_x, X, d_model, tokens, d_model, 64, 64) ||
        !make_map_rows(&m_bq, acat, hd, tokens, w.wtot, 64, 64) ||
        !make_map_rows(&m_bk, acat + hd, hd, tokens, w.wtot, 64, 64) ||
        !make_map_rows(&m_bv, acat + 2 * hd, hdv, tokens, w.wtot, 64, 64))
        return ATTN_ERR_CUDA;

    auto gather = [&](auto kernel_launch) {
        return traced(ATTN_KERNEL_PROJ_GATHER, st, [&] {
            kernel_launch();
            return launched();
        });
    };
    const int grid_g = 148 * 8;
    const struct { const void* g; int w; int col0; } heads[3] = {{dQ, d, 0}, {dK, d, hd}, {dV, dv, 2 * hd}};
    for (const auto& hh : heads) {
        s = gather([&] {
            attn::proj::heads_to_tokens<<<grid_g, attn::proj::kThreads, 0, st>>>(
                static_cast<const __nv_bfloat16*>(hh.g), acat, B, H, n, hh.w, w.wtot, hh.col0);
        });
        if (s != ATTN_OK) return s;
    }
    const struct { const void* W; int cols; int col0; } ws3[3] = {{Wq, hd, 0}, {Wk, hd, hd}, {Wv, hdv, 2 * hd}};
    for (const auto& ww : ws3) {
        s = gather([&] {
            attn::proj::concat_cols<<<grid_g, attn::proj::kThreads, 0, st>>>(
                static_cast<const __nv_bfloat16*>(ww.W), wcat, d_model, ww.cols, w.wtot, ww.col0);
        });
        if (s != ATTN_OK) return s;
    }
    s = gemm<true, true>(m_acat, m_wcat, dX, tokens, d_model, w.wtot, d_model, st);
    if (s == ATTN_OK) s = gemm<false, false>(m_x, m_bq, dWq, d_model, hd, tokens, hd, st);
    if (s == ATTN_OK) s = gemm<false, false>(m_x, m_bk, dWk, d_model, hd, tokens, hd, st);
    if (s == ATTN_OK) s = gemm<false, false>(m_x, m_bv, dWv, d_model, hdv, tokens, hdv, st);
    if (s == ATTN_OK) g_last_launches = 10;
    return s;
}

size_t attn_outproj_bwd_workspace_size(int B, int n, int d_model, int H, int dv,
                                       attn_dtype_t dtype) {
    if (check_proj(B, n, d_model, H, 8, dv, dtype) != ATTN_OK) return 0;
    return 2 * round_up(static_cast<size_t>(B) * n * H * dv * 2, 256);
}

attn_status_t attn_outproj_bwd(const void* O, const void* Wo, const void* G, void* dO, void* dWo,
                               void* workspace, size_t workspace_bytes, int B, int n,
                               int d_model, int H, int dv, attn_dtype_t dtype, void* stream) {
    attn_status_t s = check_proj(B, n, d_model, H, 8, dv, dtype);
    if (s != ATTN_OK) return s;
    if (!O || !Wo || !G || !dO || !dWo) return ATTN_ERR_NULL;
    if (!aligned16(O) || !aligned16(Wo) || !aligned16(G) || !aligned16(dO) || !aligned16(dWo))
        return ATTN_ERR_ALIGN;
    const size_t half = round_up(static_cast<size_t>(B) * n * H * dv * 2, 256);
    if (!workspace || workspace_bytes < 2 * half) return ATTN_ERR_WORKSPACE;
    if (!aligned16(workspace)) return ATTN_ERR_ALIGN;

    cudaStream_t st = as_stream(stream);
    auto* ocat = static_cast<__nv_bfloat16*>(workspace);
    auto* docat = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(workspace) + half);
    const int tokens = B * n, hdv = H * dv;
    // dWo = Ocat^T G: A = Ocat MN-major [tokens][hdv], B = G MN-major
    // [tokens][d_model]. dOcat = G Wo^T: A = G K-major, B = Wo K-major
    // [hdv][d_model].
    CUtensorMap m_ocat, m_g_mn, m_g_k, m_wo;
    if (!make_map_rows(&m_ocat, ocat, hdv, tokens, hdv, 64, 64) ||
        !make_map_rows(&m_g_mn, G, d_model, tokens, d_model, 64, 64) ||
        !make_map_rows(&m_g_k, G, d_model, tokens, d_model, 64, attn::gemmtc::kBM) ||
        !make_map_rows(&m_wo, Wo, d_model, hdv, d_model, 64, attn::gemmtc::kBN))
        return ATTN_ERR_CUDA;
    const int grid_g = 148 * 8;
    s = traced(ATTN_KERNEL_PROJ_GATHER, st, [&] {
        attn::proj::heads_to_tokens<<<grid_g, attn::proj::kThreads, 0, st>>>(
            static_cast<const __nv_bfloat16*>(O), ocat, B, H, n, dv, hdv, 0);
        return launched();
    });
    if (s == ATTN_OK) s = gemm<false, false>(m_ocat, m_g_mn, dWo, hdv, d_model, tokens, d_model, st);
    if (s == ATTN_OK) s = gemm<true, true>(m_g_k, m_wo, docat, tokens, hdv, d_model, hdv, st);
    if (s == ATTN_OK)
        s = traced(ATTN_KERNEL_PROJ_GATHER, st, [&] {
            attn::proj::tokens_to_heads<<<grid_g, attn::proj::kThreads, 0, st>>>(
                docat, static_cast<__nv_bfloat16*>(dO), B, H, n, dv, hdv, 0);
            return launched();
        });
    if (s == ATTN_OK) g_last_launches = 4;
    return s;
}

const char* attn_status_string(attn_status_t s) {
    switch (s) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_NULL: return "null pointer";
        case ATTN_ERR_SHAPE: return "invalid size or scale (or causal with n != m)";
        case ATTN_ERR_DTYPE: return "unknown dtype";
        case ATTN_ERR_UNSUPPORTED: return "unsupported by this build";
        case ATTN_ERR_ALIGN: return "pointer not 16-byte aligned";
        case ATTN_ERR_WORKSPACE: return "workspace missing or too small";
        case ATTN_ERR_CUDA: return "CUDA runtime error";
        case ATTN_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    }
    return "unknown status";
}

}  // extern "C"
