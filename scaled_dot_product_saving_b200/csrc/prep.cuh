// prep.cuh -- the memory-bound kernels around the backward pass.
//
// preprocess: D_i = rowsum(dO * O)_i, which equals rowsum(dP * P)_i ("Attention
//   Backpropagation: Step by step derivation", section "Gradient of S") but costs
//   O(n dv) instead of O(n m). It also writes the forward's LSE in base 2,
//   and both arrays are padded to whole 128-row tiles (D = 0 and LSE = +inf
//   in the padding, so padded query rows get P = 0 on the tensor-core path).
//   The same launch zeroes the backwards' counters (work items, claims and
//   per-head counts) and, for the backwards that add dQ partials into the
//   fp32 accumulator, the accumulator. D is stored multiplied by `d_scale`
//   (the tensor-core backward folds the attention scale into it).
// finalize: dQ = post_scale * dQacc, converted to the element type (the
//   CUDA-core backward only; the tensor-core backward writes dQ itself).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sm100.cuh"

namespace attn {
namespace prep {

constexpr int kThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Rows are handled by groups of G = dv/8 lanes with 16-byte loads (bf16,
// dv % 8 == 0, dv <= 256 so that G divides 32).
// Vectorised bf16 variant. Grid-stride over all BH * n_pad rows, kRowsInFlight
// row groups per warp per step so that enough loads are in flight to cover
// the memory latency. The grid is one wave (kBlocksPerSm per SM): no later
// wave competes for SMs with the backward's CTAs, which start under this
// kernel's tail.
constexpr int kRowsInFlight = 4;
constexpr int kBlocksPerSm = 3;

__global__ void __launch_bounds__(kThreads, kBlocksPerSm)
preprocess_bf16_vec(const __nv_bfloat16* __restrict__ O, const __nv_bfloat16* __restrict__ dO,
                    const float* __restrict__ LSE, float* __restrict__ lse2,
                    float* __restrict__ Dd, float* __restrict__ dQacc, int* __restrict__ counters,
                    size_t n_counters, size_t dq_elems, int BH, int n, int n_pad, int dv, float d_scale) {
    grid_launch_dependents();           // the backward may start its prologue
    for (size_t k = size_t(blockIdx.x) * kThreads + threadIdx.x; k < n_counters;
         k += size_t(gridDim.x) * kThreads)
        counters[k] = 0;
    const int G = dv / 8;                       // lanes per row
    const int rows_per_warp = 32 / G;
    const int lane = threadIdx.x & 31;
    const int sub = lane / G, lig = lane % G;
    const size_t warp_global = (size_t(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const size_t nwarps = (size_t(gridDim.x) * kThreads) >> 5;
    const size_t total_rows = size_t(BH) * n_pad;
    const size_t step_rows = size_t(rows_per_warp) * kRowsInFlight;
    for (size_t base = warp_global * step_rows; base < total_rows; base += nwarps * step_rows) {
        uint4 a[kRowsInFlight], b[kRowsInFlight];
        float lse[kRowsInFlight];
        bool real[kRowsInFlight];
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            const size_t row = base + size_t(u) * rows_per_warp + sub;
            real[u] = false;
            a[u] = b[u] = make_uint4(0u, 0u, 0u, 0u);
            lse[u] = 0.f;
            if (row < total_rows) {
                const size_t bh = row / n_pad;
                const int i = int(row % n_pad);
                if (i < n) {
                    const size_t src = bh * size_t(n) + i;
                    real[u] = true;
                    a[u] = reinterpret_cast<const uint4*>(O + src * dv)[lig];
                    b[u] = reinterpret_cast<const uint4*>(dO + src * dv)[lig];
                    if (lig == 0) lse[u] = LSE[src];
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kRowsInFlight; ++u) {
            const size_t row = base + size_t(u) * rows_per_warp + sub;
            float sum = 0.f;
            sum = fmaf(bf16_lo(a[u].x), bf16_lo(b[u].x), sum); sum = fmaf(bf16_hi(a[u].x), bf16_hi(b[u].x), sum);
            sum = fmaf(bf16_lo(a[u].y), bf16_lo(b[u].y), sum); sum = fmaf(bf16_hi(a[u].y), bf16_hi(b[u].y), sum);
            sum = fmaf(bf16_lo(a[u].z), bf16_lo(b[u].z), sum); sum = fmaf(bf16_hi(a[u].z), bf16_hi(b[u].z), sum);
            sum = fmaf(bf16_lo(a[u].w), bf16_lo(b[u].w), sum); sum = fmaf(bf16_hi(a[u].w), bf16_hi(b[u].w), sum);
            for (int off = G / 2; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            if (row < total_rows && lig == 0) {
                Dd[row] = real[u] ? sum * d_scale : 0.f;
                lse2[row] = real[u] ? lse[u] * kLog2e : INFINITY;
            }
        }
    }
    // zero the dQ accumulator (16-byte stores; dq_elems % 4 == 0)
    float4* z = reinterpret_cast<float4*>(dQacc);
    const size_t nz = dq_elems / 4;
    for (size_t k = size_t(blockIdx.x) * kThreads + threadIdx.x; k < nz;
         k += size_t(gridDim.x) * kThreads)
        z[k] = make_float4(0.f, 0.f, 0.f, 0.f);
}

__device__ __forceinline__ float ld_f(const float* p) { return *p; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// Generic variant (any dv, fp32 or bf16): one warp per row.
template <typename T>
__global__ void __launch_bounds__(kThreads)
preprocess_generic(const T* __restrict__ O, const T* __restrict__ dO,
                   const float* __restrict__ LSE, float* __restrict__ lse2,
                   float* __restrict__ Dd, float* __restrict__ dQacc, int* __restrict__ counters,
                   size_t n_counters, size_t dq_elems, int BH, int n, int n_pad, int dv, float d_scale) {
    for (size_t k = size_t(blockIdx.x) * kThreads + threadIdx.x; k < n_counters;
         k += size_t(gridDim.x) * kThreads)
        counters[k] = 0;
    const int lane = threadIdx.x & 31;
    const size_t warp_global = (size_t(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const size_t nwarps = (size_t(gridDim.x) * kThreads) >> 5;
    const size_t total_rows = size_t(BH) * n_pad;
    for (size_t row = warp_global; row < total_rows; row += nwarps) {
        const size_t bh = row / n_pad;
        const int i = int(row % n_pad);
        const size_t src = bh * size_t(n) + i;
        float s = 0.f;
        if (i < n)
            for (int c = lane; c < dv; c += 32) s = fmaf(ld_f(O + src * dv + c), ld_f(dO + src * dv + c), s);
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) {
            Dd[row] = (i < n) ? s * d_scale : 0.f;
            lse2[row] = (i < n) ? LSE[src] * kLog2e : INFINITY;
        }
    }
    for (size_t k = size_t(blockIdx.x) * kThreads + threadIdx.x; k < dq_elems;
         k += size_t(gridDim.x) * kThreads)
        dQacc[k] = 0.f;
}

__device__ __forceinline__ void st4(float* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void st4(__nv_bfloat16* p, float a, float b, float c, float d) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    uint2 w;
    w.x = *reinterpret_cast<uint32_t*>(&lo);
    w.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p) = w;
}

// dQ = post_scale * dQacc; elems % 4 == 0 (d is a multiple of 4 on the vector
// path), otherwise the scalar tail loop covers the rest.
template <typename T>
__global__ void __launch_bounds__(kThreads)
finalize_dq(const float* __restrict__ dQacc, T* __restrict__ dQ, size_t elems, float post_scale) {
    const size_t n4 = elems / 4;
    const float4* src = reinterpret_cast<const float4*>(dQacc);
    for (size_t k = size_t(blockIdx.x) * kThreads + threadIdx.x; k < n4;
         k += size_t(gridDim.x) * kThreads) {
        const float4 v = src[k];
        st4(dQ + 4 * k, v.x * post_scale, v.y * post_scale, v.z * post_scale, v.w * post_scale);
    }
    for (size_t k = 4 * n4 + size_t(blockIdx.x) * kThreads + threadIdx.x; k < elems;
         k += size_t(gridDim.x) * kThreads) {
        const float v = dQacc[k] * post_scale;
        if constexpr (sizeof(T) == 4) dQ[k] = v;
        else dQ[k] = __float2bfloat16_rn(v);
    }
}

}  // namespace prep
}  // namespace attn
