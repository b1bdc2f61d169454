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
// cudaGetSymbolAddress while that device is current, and later calls reuse it.
// All calls share the one array and it keeps the last call's contents; the
// kernels rewrite all of it that they read (the preprocess kernel writes the
// LSE and D slices and zeroes the dQ accumulator) before use. Calls whose
// kernels overlap on the GPU -- on two streams, or from two host threads --
// race on the array.
#include <cuda_runtime.h>

#include <mutex>

#include "attn.h"

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;   // 32 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device. Returns nullptr if the CUDA runtime fails.
void* scratch_for_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

size_t attn_bwd_noalloc_scratch_bytes(void) { return kScratchBytes; }

attn_status_t attn_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O,
                               const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                               int B, int H, int n, int m, int d, int dv, attn_dtype_t dtype,
                               int causal, float scale, void* stream) {
    const size_t need = attn_bwd_workspace_size(B, H, n, m, d, dv, dtype);
    if (need == 0) {
        // Invalid sizes: let attn_bwd report the precise status without
        // touching the device (it checks every argument before any launch).
        return attn_bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, nullptr, 0, B, H, n, m, d, dv, dtype,
                        causal, scale, stream);
    }
    if (need > kScratchBytes) return ATTN_ERR_WORKSPACE;
    void* scratch = scratch_for_current_device();
    if (!scratch) return ATTN_ERR_CUDA;
    return attn_bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, scratch, kScratchBytes, B, H, n, m, d, dv,
                    dtype, causal, scale, stream);
}

}  // extern "C"
