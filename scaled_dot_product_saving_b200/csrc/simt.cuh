// simt.cuh -- CUDA-core (FFMA, fp32 arithmetic) attention forward and backward.
//
// Used for fp32 tensors (whose 1e-5 accuracy no tensor-core kind reaches) and
// for bf16 widths the tensor-core kernels do not cover. The algorithm is the
// same as on the tensor-core path: the forward keeps a running row max and
// row sum over key tiles and saves LSE; the backward walks query tiles for a
// resident block of keys, rebuilds P = exp(S - LSE), forms
// dS = P * (dP - D) with D = rowsum(dO * O), accumulates dK and dV in
// registers and adds dQ's share into an fp32 accumulator with atomics.
#pragma once

#include "padmask.cuh"

#include <cuda_bf16.h>
#include <cstdint>

namespace attn {
namespace simt {

constexpr int kTile = 64;      // query rows per CTA (fwd) / keys per CTA (bwd)
constexpr int kThreads = 256;  // 8 warps x 8 rows
constexpr int kMaxWidth = 128;
constexpr int kCols = kMaxWidth / 32;  // per-lane output columns

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_max(float v) {
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Odd row pitch (in floats) so that lane-strided row reads hit distinct banks.
__host__ __device__ constexpr int odd_pitch(int w) { return (w % 2 == 0) ? w + 1 : w; }

// ----------------------------------------------------------------------------
// Forward. Grid: (ceil(n/64), B*H). Each warp owns 8 query rows; lanes split
// the keys of a tile (lane, lane+32) for S and the value columns for O.
// ----------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads)
fwd_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
           T* __restrict__ O, float* __restrict__ LSE, int n, int m, int d, int dv,
           int causal, float scale, const int* __restrict__ key_len, int H) {
    extern __shared__ float sm[];
    const int pk = odd_pitch(d);
    float* Qs = sm;                      // [64][d]
    float* Ks = Qs + kTile * d;          // [64][pk]
    float* Vs = Ks + kTile * pk;         // [64][dv]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q0 = blockIdx.x * kTile;
    const size_t bh = blockIdx.y;
    const T* Qh = Q + bh * size_t(n) * d;
    const T* Kh = K + bh * size_t(m) * d;
    const T* Vh = V + bh * size_t(m) * dv;

    for (int idx = threadIdx.x; idx < kTile * d; idx += kThreads) {
        int r = idx / d, c = idx % d;
        Qs[idx] = (q0 + r < n) ? to_f(Qh[size_t(q0 + r) * d + c]) : 0.f;
    }

    float mrow[8], lrow[8], acc[8][kCols];
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
        mrow[rr] = -INFINITY;
        lrow[rr] = 0.f;
#pragma unroll
        for (int k = 0; k < kCols; ++k) acc[rr][k] = 0.f;
    }

    const int mk = keys_valid(key_len, int(bh), H, m);     // keys past mk: padding
    const int kv_end = causal ? min(mk, q0 + kTile) : mk;
    for (int k0 = 0; k0 < kv_end; k0 += kTile) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < kTile * d; idx += kThreads) {
            int r = idx / d, c = idx % d;
            Ks[r * pk + c] = (k0 + r < m) ? to_f(Kh[size_t(k0 + r) * d + c]) : 0.f;
        }
        for (int idx = threadIdx.x; idx < kTile * dv; idx += kThreads) {
            int r = idx / dv, c = idx % dv;
            Vs[idx] = (k0 + r < m) ? to_f(Vh[size_t(k0 + r) * dv + c]) : 0.f;
        }
        __syncthreads();

#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
            const int r = warp * 8 + rr;
            const int i = q0 + r;
            const float* qrow = Qs + r * d;
            float s0 = 0.f, s1 = 0.f;
            for (int c = 0; c < d; ++c) {
                float q = qrow[c];
                s0 = fmaf(q, Ks[lane * pk + c], s0);
                s1 = fmaf(q, Ks[(lane + 32) * pk + c], s1);
            }
            const int j0 = k0 + lane, j1 = k0 + lane + 32;
            s0 = (j0 < mk && !(causal && j0 > i)) ? s0 * scale : -INFINITY;
            s1 = (j1 < mk && !(causal && j1 > i)) ? s1 * scale : -INFINITY;
            const float mnew = fmaxf(mrow[rr], warp_max(fmaxf(s0, s1)));
            if (mnew == -INFINITY) continue;  // whole row masked so far
            const float alpha = expf(mrow[rr] - mnew);
            const float p0 = expf(s0 - mnew), p1 = expf(s1 - mnew);
            lrow[rr] = lrow[rr] * alpha + warp_sum(p0 + p1);
            mrow[rr] = mnew;
#pragma unroll
            for (int k = 0; k < kCols; ++k) acc[rr][k] *= alpha;
            for (int j = 0; j < 32; ++j) {
                const float pa = __shfl_sync(0xffffffffu, p0, j);
                const float pb = __shfl_sync(0xffffffffu, p1, j);
#pragma unroll
                for (int k = 0; k < kCols; ++k) {
                    const int c = lane + 32 * k;
                    if (c < dv)
                        acc[rr][k] = fmaf(pa, Vs[j * dv + c],
                                          fmaf(pb, Vs[(j + 32) * dv + c], acc[rr][k]));
                }
            }
        }
    }

#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
        const int i = q0 + warp * 8 + rr;
        if (i >= n) continue;
        const float inv = 1.f / lrow[rr];
#pragma unroll
        for (int k = 0; k < kCols; ++k) {
            const int c = lane + 32 * k;
            if (c < dv) O[(bh * n + i) * size_t(dv) + c] = from_f<T>(acc[rr][k] * inv);
        }
        if (lane == 0) LSE[bh * n + i] = mrow[rr] + logf(lrow[rr]);
    }
}

template <typename T>
size_t fwd_smem_bytes(int d, int dv) {
    return sizeof(float) * size_t(kTile) * (d + odd_pitch(d) + dv);
}

// ----------------------------------------------------------------------------
// Backward, key-block major. Grid: (ceil(m/64), B*H). Each warp owns 8 keys;
// lanes split the queries of a tile (lane, lane+32) for S^T, dP^T and the
// output columns for dK/dV. Dd is rowsum(dO * O) from the preprocess kernel.
// dS carries no scale here; dK is scaled at the end and dQ at finalisation.
// ----------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kThreads)
bwd_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
           const T* __restrict__ dO, const float* __restrict__ LSE,
           const float* __restrict__ Dd, int d_pitch, float* __restrict__ dQacc,
           T* __restrict__ dK, T* __restrict__ dV, int n, int m, int d, int dv, int causal,
           float scale, const int* __restrict__ key_len, int H) {
    extern __shared__ float sm[];
    const int pq = odd_pitch(d), po = odd_pitch(dv);
    float* Ks = sm;                          // [64][d]
    float* Vs = Ks + kTile * d;              // [64][dv]
    float* Qs = Vs + kTile * dv;             // [64][pq]
    float* dOs = Qs + kTile * pq;            // [64][po]
    float* dSs = dOs + kTile * po;           // [64 keys][64 queries]
    float* lse_s = dSs + kTile * kTile;      // [64]
    float* D_s = lse_s + kTile;              // [64]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k0 = blockIdx.x * kTile;
    const size_t bh = blockIdx.y;
    const T* Qh = Q + bh * size_t(n) * d;
    const T* Kh = K + bh * size_t(m) * d;
    const T* Vh = V + bh * size_t(m) * dv;
    const T* dOh = dO + bh * size_t(n) * dv;

    for (int idx = threadIdx.x; idx < kTile * d; idx += kThreads) {
        int r = idx / d, c = idx % d;
        Ks[idx] = (k0 + r < m) ? to_f(Kh[size_t(k0 + r) * d + c]) : 0.f;
    }
    for (int idx = threadIdx.x; idx < kTile * dv; idx += kThreads) {
        int r = idx / dv, c = idx % dv;
        Vs[idx] = (k0 + r < m) ? to_f(Vh[size_t(k0 + r) * dv + c]) : 0.f;
    }

    float accK[8][kCols], accV[8][kCols];
#pragma unroll
    for (int rr = 0; rr < 8; ++rr)
#pragma unroll
        for (int k = 0; k < kCols; ++k) accK[rr][k] = accV[rr][k] = 0.f;

    const int mk = keys_valid(key_len, int(bh), H, m);     // keys past mk: padding
    const int q_begin = causal ? k0 : 0;  // queries before the block see none of its keys
    for (int q0 = q_begin; q0 < n; q0 += kTile) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < kTile * d; idx += kThreads) {
            int r = idx / d, c = idx % d;
            Qs[r * pq + c] = (q0 + r < n) ? to_f(Qh[size_t(q0 + r) * d + c]) : 0.f;
        }
        for (int idx = threadIdx.x; idx < kTile * dv; idx += kThreads) {
            int r = idx / dv, c = idx % dv;
            dOs[r * po + c] = (q0 + r < n) ? to_f(dOh[size_t(q0 + r) * dv + c]) : 0.f;
        }
        if (threadIdx.x < kTile) {
            const int i = q0 + threadIdx.x;
            lse_s[threadIdx.x] = (i < n) ? LSE[bh * n + i] : INFINITY;
            D_s[threadIdx.x] = (i < n) ? Dd[bh * size_t(d_pitch) + i] : 0.f;
        }
        __syncthreads();

#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
            const int jl = warp * 8 + rr;
            const int j = k0 + jl;
            const float* krow = Ks + jl * d;
            const float* vrow = Vs + jl * dv;
            float s0 = 0.f, s1 = 0.f, t0 = 0.f, t1 = 0.f;
            for (int c = 0; c < d; ++c) {
                const float kc = krow[c];
                s0 = fmaf(kc, Qs[lane * pq + c], s0);
                s1 = fmaf(kc, Qs[(lane + 32) * pq + c], s1);
            }
            for (int c = 0; c < dv; ++c) {
                const float vc = vrow[c];
                t0 = fmaf(vc, dOs[lane * po + c], t0);
                t1 = fmaf(vc, dOs[(lane + 32) * po + c], t1);
            }
            const int i0 = q0 + lane, i1 = q0 + lane + 32;
            const bool ok0 = j < mk && i0 < n && !(causal && j > i0);
            const bool ok1 = j < mk && i1 < n && !(causal && j > i1);
            const float p0 = ok0 ? expf(s0 * scale - lse_s[lane]) : 0.f;
            const float p1 = ok1 ? expf(s1 * scale - lse_s[lane + 32]) : 0.f;
            const float ds0 = p0 * (t0 - D_s[lane]);
            const float ds1 = p1 * (t1 - D_s[lane + 32]);
            dSs[jl * kTile + lane] = ds0;
            dSs[jl * kTile + lane + 32] = ds1;
            for (int q = 0; q < 32; ++q) {
                const float pa = __shfl_sync(0xffffffffu, p0, q);
                const float pb = __shfl_sync(0xffffffffu, p1, q);
                const float da = __shfl_sync(0xffffffffu, ds0, q);
                const float db = __shfl_sync(0xffffffffu, ds1, q);
#pragma unroll
                for (int k = 0; k < kCols; ++k) {
                    const int c = lane + 32 * k;
                    if (c < dv)
                        accV[rr][k] = fmaf(pa, dOs[q * po + c],
                                           fmaf(pb, dOs[(q + 32) * po + c], accV[rr][k]));
                    if (c < d)
                        accK[rr][k] = fmaf(da, Qs[q * pq + c],
                                           fmaf(db, Qs[(q + 32) * pq + c], accK[rr][k]));
                }
            }
        }
        __syncthreads();
        // dQ share of this key block: sum over its 64 keys of dS_ij K_j.
        for (int idx = threadIdx.x; idx < kTile * d; idx += kThreads) {
            const int il = idx / d, c = idx % d;
            const int i = q0 + il;
            if (i >= n) continue;
            float a = 0.f;
            for (int jl = 0; jl < kTile; ++jl) a = fmaf(dSs[jl * kTile + il], Ks[jl * d + c], a);
            atomicAdd(&dQacc[(bh * n + i) * size_t(d) + c], a);
        }
    }

#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
        const int j = k0 + warp * 8 + rr;
        if (j >= m) continue;
#pragma unroll
        for (int k = 0; k < kCols; ++k) {
            const int c = lane + 32 * k;
            if (c < d) dK[(bh * m + j) * size_t(d) + c] = from_f<T>(accK[rr][k] * scale);
            if (c < dv) dV[(bh * m + j) * size_t(dv) + c] = from_f<T>(accV[rr][k]);
        }
    }
}

template <typename T>
size_t bwd_smem_bytes(int d, int dv) {
    return sizeof(float) * (size_t(kTile) * (d + dv + odd_pitch(d) + odd_pitch(dv) + kTile) +
                            2 * kTile);
}

}  // namespace simt
}  // namespace attn
