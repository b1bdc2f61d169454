/*
 * attn.h -- C ABI of the B200 (sm_100a) scaled dot-product attention library.
 *
 * The library computes the forward pass of scaled dot-product attention, which
 * saves one log-sum-exp per query row, and the backward pass, which turns the
 * upstream gradient dO into dQ, dK and dV:
 *
 *   forward   S = scale * Q K^T,  S_ij = -inf for j > i if causal,
 *             P = softmax(S) row by row,  O = P V,  LSE_i = log sum_j exp(S_ij)
 *   backward  dV = P^T dO,  dP = dO V^T,  dS = P * (dP - rowsum(dO * O)),
 *             dQ = scale * dS K,  dK = scale * dS^T Q
 *
 * Sources: "Attention Backward Pass (dQ, dK, dV) - Transformer Architecture",
 * sections "Forward", "Backward" and "Expected Return Format" (the two calls,
 * the shapes, the causal rule n == m); "Attention backward" (eulerpad practice
 * set), Problems 2-6 and 8 (each gradient, the exact zeros under the mask);
 * "Attention Backpropagation: Step by step derivation", section "Gradient of S"
 * (rowsum(dP * P) = rowsum(dO * O), which lets the backward pass use O instead
 * of a row of P). The LSE output is not on the pages: it is the natural log of
 * the row's softmax denominator over the unmasked, already scaled scores, so
 * that the backward pass can rebuild P = exp(S - LSE) without storing P.
 *
 * Conventions shared by every call
 *  - Tensors are dense, row-major [B, H, N, width] arrays in device memory,
 *    owned by the caller. The library never allocates device memory and never
 *    frees a caller's pointer.
 *  - Every pointer must be 16-byte aligned. LSE is [B, H, n] fp32.
 *  - Q, K, V, O, dO, dQ, dK, dV share one element type, attn_dtype_t. LSE and
 *    the backward workspace are fp32 whatever the element type.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream) and never synchronise the host.
 *  - Every argument is checked before anything is launched. A status other
 *    than ATTN_OK means that nothing was launched and no output was written.
 *    ATTN_ERR_CUDA reports a launch error from the CUDA runtime.
 *  - Kernel paths: bf16 with d == dv in {64, 128} runs on the tcgen05 tensor
 *    cores (TMA-fed, TMEM accumulators). f32 with d, dv <= 64 (multiples of
 *    4) also runs on the tensor cores, each fp32 operand split into three
 *    bf16 pieces and each product taken as the six piece products that
 *    reach fp32 precision (about 2^-25 relative per product). Other f32
 *    shapes, and bf16 of any other width up to 128, run on a CUDA-core
 *    (FFMA) path in fp32 arithmetic.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_NULL = 1,           /* a required pointer is NULL                     */
    ATTN_ERR_SHAPE = 2,          /* a size is < 1, causal with n != m, or too big  */
    ATTN_ERR_DTYPE = 3,          /* unknown attn_dtype_t                           */
    ATTN_ERR_UNSUPPORTED = 4,    /* valid request this build does not implement    */
    ATTN_ERR_ALIGN = 5,          /* a pointer is not 16-byte aligned               */
    ATTN_ERR_WORKSPACE = 6,      /* workspace NULL or smaller than required        */
    ATTN_ERR_CUDA = 7,           /* the CUDA runtime reported an error             */
    ATTN_ERR_DEVICE_TIMEOUT = 8  /* a kernel gave up a bounded wait (see below)    */
} attn_status_t;

typedef enum { ATTN_F32 = 0, ATTN_BF16 = 1 } attn_dtype_t;

/* Which kernels a call may use. ATTN_PATH_AUTO picks the tensor-core path
 * where it applies (bf16 with d == dv in {64, 128}; f32 with d, dv <= 64 and
 * multiples of 4) and the CUDA-core path otherwise. ATTN_PATH_SIMT forces
 * the CUDA-core path. ATTN_PATH_TENSOR requires the tensor-core path and
 * makes other shapes ATTN_ERR_UNSUPPORTED. The CUDA-core path takes at most
 * 65535 (batch, head) problems per call (ATTN_ERR_UNSUPPORTED beyond).
 * The setting belongs to the calling host thread (each thread starts with
 * ATTN_PATH_AUTO) and applies to that thread's later calls, so threads that
 * use different paths do not race on it. */
typedef enum { ATTN_PATH_AUTO = 0, ATTN_PATH_SIMT = 1, ATTN_PATH_TENSOR = 2 } attn_path_t;

/* How the bf16 tensor-core backward computes dQ ("Attention backward",
 * Problem 5: dQ = scale * dS K, a sum over key tiles). ATTN_DQ_REDUCE: one
 * key-tile-major kernel computes dK, dV and every partial dQ, and adds the
 * partials into an fp32 accumulator in the workspace with TMA reduce-adds
 * (converted to bf16 inside the same launch). ATTN_DQ_SEPARATE: a
 * key-tile-major kernel computes dK and dV, then a query-tile-major kernel
 * recomputes S and dP per query tile and sums dQ inside one CTA (seven
 * contractions instead of five, no accumulator traffic). ATTN_DQ_AUTO picks
 * the one measured faster. Results agree within rounding; the choice, like
 * attn_path_t, belongs to the calling host thread. */
typedef enum { ATTN_DQ_AUTO = 0, ATTN_DQ_REDUCE = 1, ATTN_DQ_SEPARATE = 2 } attn_dq_path_t;

/*
 * attn_fwd -- O and LSE from Q, K, V.
 *   Q   [B,H,n,d]   K [B,H,m,d]   V [B,H,m,dv]          (read only)
 *   O   [B,H,n,dv]  element type; LSE [B,H,n] fp32     (written)
 *   causal != 0 masks key j > query i before the softmax and needs n == m.
 *   scale multiplies Q K^T; the pages use 1/sqrt(d). It must be finite.
 *   Limits: 1 <= B*H < 2^31, 1 <= n, m < 2^24, 1 <= d, dv <= 128.
 */
attn_status_t attn_fwd(const void* Q, const void* K, const void* V,
                       void* O, float* LSE,
                       int B, int H, int n, int m, int d, int dv,
                       attn_dtype_t dtype, int causal, float scale, void* stream);

/*
 * attn_bwd_workspace_size -- bytes of device scratch that attn_bwd needs for
 * these sizes: D = rowsum(dO * O) and the LSE in base 2, both [B,H,n] fp32
 * padded to whole 128-row tiles, plus an fp32 [B,H,n,d] accumulator for dQ,
 * then 256 bytes of counters of the persistent tensor-core backward (work
 * items, and the dQ slabs its converter warps have claimed) and 4 bytes per
 * (batch, head) for the head's count of finished work items (each region
 * rounded up to 256 bytes).
 * Returns 0 if the sizes are invalid.
 */
size_t attn_bwd_workspace_size(int B, int H, int n, int m, int d, int dv,
                               attn_dtype_t dtype);

/*
 * attn_bwd -- dQ, dK, dV from Q, K, V, O, dO and the forward's LSE.
 *   Q, K, V, O, dO, LSE as in attn_fwd (read only); O and LSE must come
 *   from attn_fwd on the same Q, K, V, causal and scale.
 *   dQ [B,H,n,d], dK [B,H,m,d], dV [B,H,m,dv]  element type (written)
 *   workspace: caller-owned device memory of at least
 *   attn_bwd_workspace_size(...) bytes; its contents on entry do not matter
 *   and are overwritten. It must not be in use by another call in flight.
 *   P is rebuilt from Q, K and LSE; neither P nor the softmax Jacobian is
 *   ever stored.
 */
attn_status_t attn_bwd(const void* Q, const void* K, const void* V,
                       const void* O, const void* dO, const float* LSE,
                       void* dQ, void* dK, void* dV,
                       void* workspace, size_t workspace_bytes,
                       int B, int H, int n, int m, int d, int dv,
                       attn_dtype_t dtype, int causal, float scale, void* stream);

/*
 * attn_fwd_masked, attn_bwd_masked -- attn_fwd and attn_bwd with a key
 * padding mask ("Is there any Reference About Backpropagation of the
 * Transformer's Multi-Head Layer?", section 4, "Practical Tips for
 * Implementers": causal or padding masks go before the softmax, and the
 * backward pass then zeroes the masked gradients). The pages give padding
 * masks no layout; here the mask is
 *   key_len  [B] int32 in device memory (4-byte aligned; NULL: no mask):
 *            the number of valid keys of batch element b. Keys j >= key_len[b]
 *            of every head of b get S = -inf before the softmax, so P = 0 and
 *            dS = 0 there, and their dK and dV rows are zero. Values are
 *            clamped to [1, m] on the device (a row with no valid key has no
 *            softmax). Query rows are never masked: rows of padded queries
 *            attend to the valid keys as usual.
 * Both calls must see the same key_len; with causal != 0 the two masks
 * combine. All other arguments, limits and errors are those of attn_fwd and
 * attn_bwd, which are these calls with key_len = NULL. Key tiles made only of
 * padding are skipped by the forward and do one masked query tile's work in
 * the backward.
 */
attn_status_t attn_fwd_masked(const void* Q, const void* K, const void* V,
                              void* O, float* LSE, const int* key_len,
                              int B, int H, int n, int m, int d, int dv,
                              attn_dtype_t dtype, int causal, float scale, void* stream);

attn_status_t attn_bwd_masked(const void* Q, const void* K, const void* V,
                              const void* O, const void* dO, const float* LSE,
                              const int* key_len, void* dQ, void* dK, void* dV,
                              void* workspace, size_t workspace_bytes,
                              int B, int H, int n, int m, int d, int dv,
                              attn_dtype_t dtype, int causal, float scale, void* stream);

/*
 * attn_bwd_noalloc -- attn_bwd for callers that cannot allocate device memory.
 * The pages have no counterpart: this is a deployment convenience, not part
 * of the method. Some callers cannot hand attn_bwd a workspace: a plugin or
 * custom op inside a host framework that owns all device memory and gives
 * the op no scratch buffer, where a cudaMalloc of its own would fail against,
 * or bypass, the framework's budget. This call takes the same arguments as
 * attn_bwd minus the workspace, and uses instead a scratch array compiled
 * into the library: attn_bwd_noalloc_scratch_bytes() bytes (32 MiB) of
 * device memory that every GPU loading the library holds until the process
 * exits. It allocates nothing and calls no allocating routine.
 *  - Sizes whose attn_bwd_workspace_size() exceeds the array are rejected
 *    with ATTN_ERR_WORKSPACE before anything is launched (the d = 64,
 *    B*H*n = 65536 problem fits; the long-context ones do not). Argument
 *    errors take precedence: the status is the one attn_bwd would give for
 *    the same arguments without a workspace.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and keeps it for as
 *    long as that device's context lives; the first call after the context
 *    has been replaced (cudaDeviceReset) looks it up again. Make those first
 *    calls before any stream capture on the device. If the lookup fails the
 *    call returns ATTN_ERR_CUDA, with the runtime's error state cleared.
 *  - Every call shares the one array, which keeps the last call's contents;
 *    the kernels rewrite what they read. Calls whose kernels overlap on the
 *    GPU (two streams, or two host threads) race on the array: serialise them.
 * Other statuses are those of attn_bwd.
 */
attn_status_t attn_bwd_noalloc(const void* Q, const void* K, const void* V,
                               const void* O, const void* dO, const float* LSE,
                               void* dQ, void* dK, void* dV,
                               int B, int H, int n, int m, int d, int dv,
                               attn_dtype_t dtype, int causal, float scale, void* stream);

/* Size in bytes of the scratch array attn_bwd_noalloc uses. */
size_t attn_bwd_noalloc_scratch_bytes(void);

/*
 * attn_get_device_error -- synchronise `stream`, then report and clear the
 * device-side error word of the current device. Every wait inside the
 * tensor-core kernels is bounded; a wait that runs out writes
 * ATTN_ERR_DEVICE_TIMEOUT there, and the kernel releases its tensor memory
 * and exits instead of hanging. The word is sticky: while it is set, the
 * tensor-core kernels skip their work, so outputs of calls made after a
 * timeout are undefined until this function has read and cleared it.
 * Returns ATTN_OK, ATTN_ERR_DEVICE_TIMEOUT, or ATTN_ERR_CUDA if synchronising
 * or reading failed.
 */
attn_status_t attn_get_device_error(void* stream);

/*
 * attn_probe_timeout -- launch one CTA that waits on a barrier nothing will
 * ever complete, with a wait bound of `timeout_us` microseconds (1..10^6), so
 * that a test can check the timeout path end to end: afterwards
 * attn_get_device_error() must return ATTN_ERR_DEVICE_TIMEOUT.
 */
attn_status_t attn_probe_timeout(unsigned timeout_us, void* stream);

/*
 * Kernel tracing. Between attn_trace_begin and attn_trace_end, every kernel
 * that attn_fwd/attn_bwd launch from the calling host thread is bracketed by
 * a pair of CUDA events on the call's stream (at most `capacity` launches,
 * 1..65536, are recorded; later ones run untraced). attn_trace_end stops
 * recording, waits for the recorded events, and writes up to `max_entries`
 * (kernel id, milliseconds) pairs in launch order to `out` (which may be NULL
 * when max_entries is 0). It returns the number of launches recorded, or -1
 * if the CUDA runtime failed. The events are created on first use and reused;
 * no device memory is allocated.
 */
typedef enum {
    ATTN_KERNEL_FWD_TENSOR = 1,   /* tcgen05 forward                          */
    ATTN_KERNEL_FWD_SIMT = 2,     /* CUDA-core forward                        */
    ATTN_KERNEL_PREPROCESS = 3,   /* D = rowsum(dO*O), base-2 LSE, zero dQacc */
    ATTN_KERNEL_BWD_TENSOR = 4,   /* tcgen05 backward                         */
    ATTN_KERNEL_BWD_SIMT = 5,     /* CUDA-core backward                       */
    ATTN_KERNEL_FINALIZE = 6,     /* dQ accumulator -> dQ (CUDA-core path)     */
    ATTN_KERNEL_PROJ_GATHER = 7,  /* per-head gradients / weights side by side */
    ATTN_KERNEL_GEMM = 8,         /* tcgen05 GEMM of the projection gradients  */
    ATTN_KERNEL_FWD_F32X = 9,     /* tcgen05 forward, fp32 by bf16 pieces      */
    ATTN_KERNEL_BWD_F32X = 10,    /* ... backward: dK/dV and dQ passes, one launch */
    ATTN_KERNEL_BWD_KV = 11,      /* tcgen05 dK/dV pass (ATTN_DQ_SEPARATE)      */
    ATTN_KERNEL_BWD_DQ = 12       /* tcgen05 dQ pass (ATTN_DQ_SEPARATE)         */
} attn_kernel_id_t;

typedef struct {
    int kernel;    /* attn_kernel_id_t */
    float ms;      /* device time between the bracketing events */
} attn_kernel_time_t;

attn_status_t attn_trace_begin(int capacity);
int attn_trace_end(attn_kernel_time_t* out, int max_entries);

/*
 * Projection and input gradients of multi-head self-attention ("Lesson 4 -
 * The Backward Pass for Attention", section "Step 4: Back to the Parameters
 * and Input"; "Attention backward", Problem 7). With Q = X Wq, K = X Wk,
 * V = X Wv and head h the column block h of each projection (Q [B,n,H*d]
 * split into [B,H,n,d], as attn_fwd/attn_bwd take it), and dQ, dK, dV from
 * attn_bwd:
 *   dWq = sum over the batch of X_b^T dQ_b   [d_model, H*d]   (same for dWk;
 *   dWv [d_model, H*dv])
 *   dX  = dQ Wq^T + dK Wk^T + dV Wv^T        [B, n, d_model]
 * with dQ, dK, dV merged back to [B, n, H*w]. Arguments:
 *   X [B,n,d_model], Wq, Wk [d_model, H*d], Wv [d_model, H*dv]  (read only)
 *   dQ, dK [B,H,n,d], dV [B,H,n,dv]                              (read only)
 *   dX, dWq, dWk, dWv: outputs with the shapes of X, Wq, Wk, Wv  (written)
 *   bf16 only (ATTN_ERR_UNSUPPORTED otherwise); fp32 accumulation; d, dv and
 *   d_model multiples of 8 (ATTN_ERR_SHAPE otherwise); all pointers 16-byte
 *   aligned; contiguous row-major tensors.
 *   workspace: caller-owned device memory of attn_proj_bwd_workspace_size()
 *   bytes (token-major copies of the gradients and the weights side by side);
 *   contents on entry do not matter. Stream-ordered and asynchronous; a
 *   non-OK status means nothing was launched.
 */
size_t attn_proj_bwd_workspace_size(int B, int n, int d_model, int H, int d, int dv,
                                    attn_dtype_t dtype);
attn_status_t attn_proj_bwd(const void* X, const void* Wq, const void* Wk, const void* Wv,
                            const void* dQ, const void* dK, const void* dV, void* dX,
                            void* dWq, void* dWk, void* dWv, void* workspace,
                            size_t workspace_bytes, int B, int n, int d_model, int H, int d,
                            int dv, attn_dtype_t dtype, void* stream);

/*
 * Gradients of the multi-head output projection ("Attention backward",
 * Problem 10): with Y = [O_1 ... O_H] Wo (O_h the heads of attn_fwd's output,
 * concatenated along columns) and G = dL/dY,
 *   dWo  = [O_1 ... O_H]^T G          summed over the batch   [H*dv, d_model]
 *   dO_h = columns h*dv .. (h+1)*dv of G Wo^T                  [B,H,n,dv]
 * dO is what attn_bwd takes as its dO. Arguments:
 *   O [B,H,n,dv], Wo [H*dv, d_model], G [B,n,d_model]  (read only)
 *   dO [B,H,n,dv], dWo [H*dv, d_model]                  (written)
 *   bf16 only (ATTN_ERR_UNSUPPORTED otherwise); dv and d_model multiples of 8
 *   (ATTN_ERR_SHAPE otherwise); pointers 16-byte aligned; workspace of
 *   attn_outproj_bwd_workspace_size() bytes (the merged O and G Wo^T), its
 *   contents on entry irrelevant. Stream-ordered; a non-OK status means
 *   nothing was launched.
 */
size_t attn_outproj_bwd_workspace_size(int B, int n, int d_model, int H, int dv,
                                       attn_dtype_t dtype);
attn_status_t attn_outproj_bwd(const void* O, const void* Wo, const void* G, void* dO, void* dWo,
                               void* workspace, size_t workspace_bytes, int B, int n,
                               int d_model, int H, int dv, attn_dtype_t dtype, void* stream);

/* Select the kernel path for the calling thread's later calls (see
 * attn_path_t). */
attn_status_t attn_set_path(attn_path_t path);

/* Select how the calling thread's later bf16 tensor-core backward calls
 * compute dQ (see attn_dq_path_t). */
attn_status_t attn_set_dq_path(attn_dq_path_t path);

/* Number of kernels the calling thread's last successful attn_fwd/attn_bwd/
 * attn_proj_bwd/attn_outproj_bwd call launched. */
int attn_last_launch_count(void);

/* A static, human-readable name for a status code. */
const char* attn_status_string(attn_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
