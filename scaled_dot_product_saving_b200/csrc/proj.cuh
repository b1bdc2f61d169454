// proj.cuh -- layout kernels around the projection-gradient GEMMs.
//
// The attention gradients come per head, [B, H, n, w]; the projections of
// "Attention backward", Problem 7 (Q = X Wq, head h = column block h) want
// them per token. heads_to_tokens writes dQ, dK, dV side by side into one
// token-major matrix A = [dQ | dK | dV] of shape [B*n, 2*H*d + H*dv], and
// concat_cols puts [Wq | Wk | Wv] side by side the same way, so that
//   dX   = A [Wq | Wk | Wv]^T                  (one GEMM; the three paths of
//                                               Problem 7 add inside it)
//   dWq  = X^T A[:, 0:Hd], dWk, dWv likewise   (K runs over all B*n tokens:
//                                               the batch sum of "Lesson 4",
//                                               Step 4)
// For the output projection of Problem 10 the same copy merges O into
// [O_1 ... O_H] and tokens_to_heads slices G Wo^T back into per-head blocks.
// All are plain 16-byte copies, bound by HBM bandwidth.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace attn {
namespace proj {

constexpr int kThreads = 256;

// dst[(b*n + t) * ld + col0 + h*w + j] = src[((b*H + h)*n + t)*w + j], in
// 8-element (16-byte) chunks; w % 8 == 0.
__global__ void __launch_bounds__(kThreads)
heads_to_tokens(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst, int B,
                int H, int n, int w, int ld, int col0) {
    const int cw = w / 8;
    const size_t total = size_t(B) * H * n * cw;
    for (size_t i = size_t(blockIdx.x) * kThreads + threadIdx.x; i < total;
         i += size_t(gridDim.x) * kThreads) {
        const int jc = int(i % cw);
        size_t r = i / cw;
        const int t = int(r % n);
        r /= n;
        const int h = int(r % H);
        const int b = int(r / H);
        const uint4 v = reinterpret_cast<const uint4*>(src)[i];
        *reinterpret_cast<uint4*>(dst + (size_t(b) * n + t) * ld + col0 + size_t(h) * w + 8 * jc) = v;
    }
}

// dst[r * ld + col0 + c] = src[r * cols + c], in 16-byte chunks; cols % 8 == 0.
__global__ void __launch_bounds__(kThreads)
concat_cols(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst, int rows,
            int cols, int ld, int col0) {
    const int cc = cols / 8;
    const size_t total = size_t(rows) * cc;
    for (size_t i = size_t(blockIdx.x) * kThreads + threadIdx.x; i < total;
         i += size_t(gridDim.x) * kThreads) {
        const int c = int(i % cc);
        const size_t r = i / cc;
        const uint4 v = reinterpret_cast<const uint4*>(src)[i];
        *reinterpret_cast<uint4*>(dst + r * ld + col0 + 8 * c) = v;
    }
}

// The inverse of heads_to_tokens: dst[((b*H + h)*n + t)*w + j] =
// src[(b*n + t) * ld + col0 + h*w + j] (the column blocks of G Wo^T back into
// per-head gradients, "Attention backward", Problem 10).
__global__ void __launch_bounds__(kThreads)
tokens_to_heads(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst, int B,
                int H, int n, int w, int ld, int col0) {
    const int cw = w / 8;
    const size_t total = size_t(B) * H * n * cw;
    for (size_t i = size_t(blockIdx.x) * kThreads + threadIdx.x; i < total;
         i += size_t(gridDim.x) * kThreads) {
        const int jc = int(i % cw);
        size_t r = i / cw;
        const int t = int(r % n);
        r /= n;
        const int h = int(r % H);
        const int b = int(r / H);
        reinterpret_cast<uint4*>(dst)[i] = *reinterpret_cast<const uint4*>(
            src + (size_t(b) * n + t) * ld + col0 + size_t(h) * w + 8 * jc);
    }
}

}  // namespace proj
}  // namespace attn
