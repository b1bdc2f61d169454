// noalloc.cu -- attn_bwd_noalloc: the backward pass for callers that cannot
// allocate device memory.
//
// attn_bwd needs caller-provided scratch (the base-2 LSE, D and the fp32 dQ
// accumulator). Some callers have no way to provide it: a plugin or custom op
// inside a host framework that owns every byte of device memory and offers no
// scratch hook, so that a cudaMalloc of its own would fail against, or slip
// past, the framework's memory budget. For them this entry point takes its
// scratch from a fixed array compiled into the library instead.
//
// The array is a file-scope __device__ object of kScratchBytes. Every GPU that
// loads the library holds it until the process exits. Host code cannot use
// the array's name as a device address (on the host it names a stand-in), so
// the first call on each device looks the address up with
// cudaGetSymbolAddress while that device is current, and later calls reuse it
// for as long as the device's context lives: the address is kept with the
// context's unique id, and a call that finds another context current (after
// cudaDeviceReset, say, which unloads the module that held the array) looks
// it up again instead of passing a stale address to the kernels.
// All calls share the one array and it keeps the last call's contents; the
// kernels rewrite all of it that they read (the preprocess kernel writes the
// LSE and D slices and zeroes the counters; the backward stores each dQ slab
// before it adds into it) before use. Calls whose kernels overlap on the GPU
// -- on two streams, or from two host threads -- race on the array.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "attn.h"

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;   // 32 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct Entry {
    unsigned long long ctx_id;   // context the address belongs to (0: none yet)
    void* ptr;
};

std::mutex g_setup_mutex;
Entry g_scratch[kMaxDevices] = {};

// The unique id of the calling thread's current context (never reused within
// the process), or 0 if the driver cannot tell.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the scratch array on the current device, looked up once
// per device and context. Returns nullptr (with the runtime's error state
// cleared) if the CUDA runtime fails.
void* scratch_for_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        (void)cudaGetLastError();
        return nullptr;
    }
    // 0 if no context is current yet (the lookup below creates it).
    const unsigned long long id = current_context_id();
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    Entry& e = g_scratch[dev];
    if (!e.ptr || id == 0 || e.ctx_id != id) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            (void)cudaGetLastError();
            e = Entry{0, nullptr};
            return nullptr;
        }
        e = Entry{current_context_id(), p};   // id 0 again: looked up on every call
    }
    return e.ptr;
}

}  // namespace

extern "C" {

size_t attn_bwd_noalloc_scratch_bytes(void) { return kScratchBytes; }

attn_status_t attn_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O,
                               const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                               int B, int H, int n, int m, int d, int dv, attn_dtype_t dtype,
                               int causal, float scale, void* stream) {
    const size_t need = attn_bwd_workspace_size(B, H, n, m, d, dv, dtype);
    if (need == 0 || need > kScratchBytes) {
        // Invalid sizes, or sizes beyond the array: attn_bwd checks every
        // argument before any launch, so without a workspace it reports the
        // same status it would for these arguments (null, alignment, shape
        // ...), and ATTN_ERR_WORKSPACE only when all of them are valid.
        return attn_bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, nullptr, 0, B, H, n, m, d, dv, dtype,
                        causal, scale, stream);
    }
    void* scratch = scratch_for_current_device();
    if (!scratch) return ATTN_ERR_CUDA;
    return attn_bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, scratch, kScratchBytes, B, H, n, m, d, dv,
                    dtype, causal, scale, stream);
}

}  // extern "C"
