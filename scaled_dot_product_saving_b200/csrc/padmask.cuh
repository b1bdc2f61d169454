// padmask.cuh -- the key padding mask shared by every attention kernel.
//
// "Is there any Reference About Backpropagation of the Transformer's
// Multi-Head Layer?", section 4 ("Practical Tips for Implementers"): causal
// or padding masks are applied before the softmax, and the backward pass then
// zeroes the masked gradients. The pages give padding masks no layout; here a
// mask is the number of valid keys of each batch element, key_len[B] (int32,
// device memory), and the keys at or past it are masked exactly like keys past
// the end of the tensor: S = -inf before the softmax, so P = 0 and dS = 0, and
// their dK and dV rows are zero.
#pragma once

namespace attn {

// Valid keys of head bh (batch element bh / H): key_len[bh / H] clamped to
// [1, m], or m without a mask.
__device__ __forceinline__ int keys_valid(const int* __restrict__ key_len, int bh, int H, int m) {
    if (key_len == nullptr) return m;
    const int L = __ldg(key_len + bh / H);
    return min(max(L, 1), m);
}

}  // namespace attn
