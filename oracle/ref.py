"""Plain float64 CPU oracle for scaled dot-product attention, forward and backward.

TEST INFRASTRUCTURE ONLY. The tests, the smoke check and the benchmark's CPU
baseline are the only code that may import this module. The library's
product path never calls it, and this module shares no code with the CUDA
kernels.

What it computes is the plain definition from the pages. Each step is a
small function named after the quantity it produces, so a reader can check it
against the formula by eye, and the mutation tests can swap one step for a
known mistake:

  Forward ("Attention Backward Pass (dQ, dK, dV)", section "Forward"):
      S = Q K^T * scale                 scale = 1/sqrt(d), d = Q.shape[-1]
      S_ij = -inf for j > i             only if causal (then n == m)
      P = softmax(S) row by row         stable: subtract the row max
      O = P V
  Optional padding mask ("Is there any Reference About Backpropagation of
  the Transformer's Multi-Head Layer?", section 4, "Practical Tips for
  Implementers": causal or padding masks go before the softmax, and the
  backward then zeroes the masked gradients):
      S_ij = -inf for j >= key_len[b]   keys past batch element b's length
  plus the per-row log-sum-exp LSE_i = log sum_j exp(S_ij). The pages do not
  define it. This oracle reads it as the natural log over the unmasked,
  already scaled scores, so that P = exp(S - LSE).

  Backward (same page, section "Backward"; "Attention backward" practice set,
  Problems 2-6):
      dV = P^T dO
      dP = dO V^T
      dS = P * (dP - rowsum(dP * P))    the softmax Jacobian-vector product,
                                        row by row, no m x m Jacobian
      dQ = scale * dS K
      dK = scale * dS^T Q
  P is recomputed from Q and K inside the backward pass, as that page's
  "Edge cases and conventions" asks. The row sum is taken over dP * P exactly
  as printed, not through the rowsum(dO * O) identity, so the identity stays
  an independent check.

Evaluation order. Each query row is independent in the forward pass and in
dS, and dK and dV are sums over query rows. The head-level functions
therefore apply the definition to ``row_block`` query rows at a time, so that
the n x m score matrix of a long sequence never has to exist at once.
Within a block nothing is fused or reordered.

Projection and input gradients of self-attention ("Lesson 4 - The Backward
Pass for Attention", section "Step 4: Back to the Parameters and Input";
"Attention backward", Problem 7), with Q = X Wq, K = X Wk, V = X Wv and the
H heads taken as consecutive column blocks of each projection:
      dWq = sum over the batch of X^T dQ   (likewise dWk, dWv)
      dX  = dQ Wq^T + dK Wk^T + dV Wv^T    (X feeds all three projections)
with dQ, dK, dV merged back from heads to columns. The multi-head output
projection ("Attention backward", Problem 10), Y = [O_1 ... O_H] Wo:
      dWo  = [O_1 ... O_H]^T G
      dO_h = columns h*dv .. (h+1)*dv of G Wo^T

Pins (tests/test_oracle.py): the worked examples of "Attention Backward Pass
(dQ, dK, dV)" (section "Examples"); the loss value printed in "Lesson 4 - The
Backward Pass for Attention" (section "A Scalar Loss So dout Is Known"),
reproduced from the same seed; central finite differences of
L = sum(O * dO); float64 torch autograd of the library's
scaled_dot_product_attention; the explicit softmax Jacobian diag(a) - a a^T
("Lesson 4", Exercise 2); the rowsum(dP * P) = rowsum(dO * O) identity
("Attention Backpropagation: Step by step derivation", "Gradient of S");
exact zeros at masked positions ("Attention backward", Problem 8); the
padding mask against the unmasked definition on keys cut to the valid
length, and against finite differences; and
mutation tests that plant each of the pages' wrong variants and check that
the pins catch it. No function here is left unpinned.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "default_scale", "scores", "apply_causal_mask", "apply_padding_mask", "row_softmax",
    "grad_v", "grad_p", "softmax_jvp", "grad_q", "grad_k",
    "head_forward", "head_backward",
    "attention_forward", "attention_backward",
    "split_heads", "merge_heads", "project_qkv", "grad_weight", "grad_input",
    "projection_backward", "output_projection", "output_projection_backward",
]

ROW_BLOCK = 256


def default_scale(d: int) -> float:
    """1/sqrt(d) with d the width of Q and K ("Forward": d = Q.shape[-1])."""
    return 1.0 / math.sqrt(d)


# --------------------------------------------------------------------------
# Forward steps
# --------------------------------------------------------------------------
def scores(Qb: np.ndarray, K: np.ndarray, scale: float) -> np.ndarray:
    """S = Q K^T * scale for a block of query rows ("Forward"; Problem 1)."""
    return (Qb @ K.T) * scale


def apply_causal_mask(S: np.ndarray, row0: int) -> np.ndarray:
    """Set S_ij = -inf where key j lies after query i, before the softmax.

    ``row0`` is the global index of the block's first query row. The
    diagonal is kept ("Attention backward", Problem 8: the mask keeps the
    diagonal and everything below it).
    """
    rows = np.arange(row0, row0 + S.shape[0])[:, None]
    cols = np.arange(S.shape[1])[None, :]
    return np.where(cols > rows, -np.inf, S)


def apply_padding_mask(S: np.ndarray, key_len: int) -> np.ndarray:
    """Set S_ij = -inf for every key j at or past ``key_len``, before the
    softmax ("Is there any Reference ...", section 4: padding masks are
    applied before the softmax). The pages name padding masks without a
    layout; here they are given as the number of valid keys of each batch
    element, the keys after it being padding."""
    cols = np.arange(S.shape[1])[None, :]
    return np.where(cols >= key_len, -np.inf, S)


def row_softmax(S: np.ndarray):
    """Row-wise softmax with the row max subtracted, and the row LSE.

    Returns (P, lse) with P = exp(S - lse) and lse = max + log(sum exp(S - max)).
    Masked entries (-inf) give exactly 0 in P.
    """
    mx = S.max(axis=-1, keepdims=True)
    e = np.exp(S - mx)
    total = e.sum(axis=-1, keepdims=True)
    P = e / total
    lse = (mx + np.log(total))[:, 0]
    return P, lse


# --------------------------------------------------------------------------
# Backward steps
# --------------------------------------------------------------------------
def grad_v(P: np.ndarray, dO: np.ndarray) -> np.ndarray:
    """dV = P^T dO ("Backward"; Problem 2)."""
    return P.T @ dO


def grad_p(dO: np.ndarray, V: np.ndarray) -> np.ndarray:
    """dP = dO V^T ("Backward"; Problem 3)."""
    return dO @ V.T


def softmax_jvp(P: np.ndarray, dP: np.ndarray) -> np.ndarray:
    """dS = P * (dP - rowsum(dP * P)), row by row ("Backward"; Problem 4)."""
    return P * (dP - (dP * P).sum(axis=-1, keepdims=True))


def grad_q(dS: np.ndarray, K: np.ndarray, scale: float) -> np.ndarray:
    """dQ = scale * dS K ("Backward"; Problem 5)."""
    return scale * (dS @ K)


def grad_k(dS: np.ndarray, Q: np.ndarray, scale: float) -> np.ndarray:
    """dK = scale * dS^T Q ("Backward"; Problem 6)."""
    return scale * (dS.T @ Q)


# --------------------------------------------------------------------------
# One head: Q (n,d), K (m,d), V (m,dv), dO (n,dv)
# --------------------------------------------------------------------------
def _check_head(Q, K, V, causal):
    n, d = Q.shape
    m, dk = K.shape
    if dk != d or V.shape[0] != m:
        raise ValueError(f"shape mismatch Q{Q.shape} K{K.shape} V{V.shape}")
    if causal and n != m:
        raise ValueError("causal attention needs as many queries as keys")


def _block_probs(Q, K, r0, r1, causal, scale, key_len=None):
    S = scores(Q[r0:r1], K, scale)
    if causal:
        S = apply_causal_mask(S, r0)
    if key_len is not None:
        S = apply_padding_mask(S, key_len)
    return row_softmax(S)


def _check_key_len(key_len, m):
    if key_len is not None and not 1 <= key_len <= m:
        raise ValueError(f"key_len {key_len} outside [1, {m}]")


def head_forward(Q, K, V, causal=False, scale=None, row_block=ROW_BLOCK, key_len=None):
    """Return (O, lse) for one head, in float64. ``key_len``: number of
    unpadded keys (None: all)."""
    Q, K, V = (np.asarray(x, dtype=np.float64) for x in (Q, K, V))
    _check_head(Q, K, V, causal)
    _check_key_len(key_len, K.shape[0])
    scale = default_scale(Q.shape[1]) if scale is None else float(scale)
    n = Q.shape[0]
    O = np.empty((n, V.shape[1]))
    lse = np.empty(n)
    for r0 in range(0, n, row_block):
        r1 = min(n, r0 + row_block)
        P, lse[r0:r1] = _block_probs(Q, K, r0, r1, causal, scale, key_len)
        O[r0:r1] = P @ V
    return O, lse


def head_backward(Q, K, V, dO, causal=False, scale=None, row_block=ROW_BLOCK, key_len=None):
    """Return (dQ, dK, dV) for one head, in float64, recomputing P."""
    Q, K, V, dO = (np.asarray(x, dtype=np.float64) for x in (Q, K, V, dO))
    _check_head(Q, K, V, causal)
    _check_key_len(key_len, K.shape[0])
    scale = default_scale(Q.shape[1]) if scale is None else float(scale)
    n = Q.shape[0]
    dQ = np.empty_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for r0 in range(0, n, row_block):
        r1 = min(n, r0 + row_block)
        P, _ = _block_probs(Q, K, r0, r1, causal, scale, key_len)
        dV += grad_v(P, dO[r0:r1])
        dP = grad_p(dO[r0:r1], V)
        dS = softmax_jvp(P, dP)
        dQ[r0:r1] = grad_q(dS, K, scale)
        dK += grad_k(dS, Q[r0:r1], scale)
    return dQ, dK, dV


# --------------------------------------------------------------------------
# Batched [..., N, d] front ends, mirroring the pages' two calls
# --------------------------------------------------------------------------
def _heads(*arrays):
    lead = arrays[0].shape[:-2]
    flat = [np.asarray(a, dtype=np.float64).reshape((-1,) + a.shape[-2:])
            for a in arrays]
    return lead, flat


def _head_key_len(key_len, lead, h):
    """The key length of flattened head h: key_len is indexed by the first
    leading dimension (the batch) of [B, H, N, d] tensors."""
    if key_len is None:
        return None
    per_batch = int(np.prod(lead[1:])) if len(lead) > 1 else 1
    return int(key_len[h // per_batch])


def attention_forward(Q, K, V, causal=False, scale=None, row_block=ROW_BLOCK, key_len=None):
    """O and LSE for tensors shaped [..., n, d]; scale defaults to 1/sqrt(d).
    ``key_len`` (optional, one entry per batch element): valid keys of each
    batch element, the rest masked as padding."""
    lead, (q, k, v) = _heads(Q, K, V)
    O = np.empty(q.shape[:2] + (v.shape[2],))
    lse = np.empty(q.shape[:2])
    for h in range(q.shape[0]):
        O[h], lse[h] = head_forward(q[h], k[h], v[h], causal, scale, row_block,
                                    _head_key_len(key_len, lead, h))
    return O.reshape(lead + O.shape[1:]), lse.reshape(lead + lse.shape[1:])


def attention_backward(Q, K, V, dO, causal=False, scale=None, row_block=ROW_BLOCK,
                       key_len=None):
    """(dQ, dK, dV) with the shapes of Q, K, V, for tensors shaped [..., N, d]."""
    lead, (q, k, v, do) = _heads(Q, K, V, dO)
    dQ = np.empty_like(q)
    dK = np.empty_like(k)
    dV = np.empty_like(v)
    for h in range(q.shape[0]):
        dQ[h], dK[h], dV[h] = head_backward(q[h], k[h], v[h], do[h], causal,
                                            scale, row_block,
                                            _head_key_len(key_len, lead, h))
    return (dQ.reshape(lead + dQ.shape[1:]), dK.reshape(lead + dK.shape[1:]),
            dV.reshape(lead + dV.shape[1:]))


# --------------------------------------------------------------------------
# Projection and input gradients ("Lesson 4", Step 4; "Attention backward",
# Problem 7)
# --------------------------------------------------------------------------
def split_heads(T: np.ndarray, H: int) -> np.ndarray:
    """[B, n, H*w] -> [B, H, n, w]: head h is column block h of a projection."""
    B, n, HW = T.shape
    return T.reshape(B, n, H, HW // H).transpose(0, 2, 1, 3)


def merge_heads(T: np.ndarray) -> np.ndarray:
    """[B, H, n, w] -> [B, n, H*w], the inverse of split_heads."""
    B, H, n, w = T.shape
    return T.transpose(0, 2, 1, 3).reshape(B, n, H * w)


def project_qkv(X, Wq, Wk, Wv, H):
    """Q, K, V = X Wq, X Wk, X Wv, split into H heads (Problem 7's forward)."""
    X = np.asarray(X, dtype=np.float64)
    return (split_heads(X @ Wq, H), split_heads(X @ Wk, H), split_heads(X @ Wv, H))


def grad_weight(X: np.ndarray, dT: np.ndarray) -> np.ndarray:
    """dW = sum over the batch of X_b^T dT_b for T = X W: the weight is shared
    across the batch, so its gradient sums the per-item contributions
    ("Lesson 4", Step 4). X [B, n, C], dT [B, n, w] -> [C, w]."""
    return np.einsum("bnc,bnw->cw", X, dT)


def grad_input(dQm, dKm, dVm, Wq, Wk, Wv) -> np.ndarray:
    """dX = dQ Wq^T + dK Wk^T + dV Wv^T: X feeds all three projections and
    the three paths add (Problem 7). Gradients merged to [B, n, H*w]."""
    return dQm @ Wq.T + dKm @ Wk.T + dVm @ Wv.T


def projection_backward(X, Wq, Wk, Wv, dQ, dK, dV):
    """(dX, dWq, dWk, dWv) from dQ, dK, dV shaped [B, H, n, w] (the heads as
    split by project_qkv)."""
    X = np.asarray(X, dtype=np.float64)
    Wq, Wk, Wv = (np.asarray(W, dtype=np.float64) for W in (Wq, Wk, Wv))
    dQm, dKm, dVm = (merge_heads(np.asarray(G, dtype=np.float64)) for G in (dQ, dK, dV))
    return (grad_input(dQm, dKm, dVm, Wq, Wk, Wv),
            grad_weight(X, dQm), grad_weight(X, dKm), grad_weight(X, dVm))


def output_projection(O, Wo):
    """Y = [O_1 ... O_H] Wo for O [B, H, n, dv], Wo [H*dv, d_model] (Problem 10)."""
    return merge_heads(np.asarray(O, dtype=np.float64)) @ np.asarray(Wo, dtype=np.float64)


def output_projection_backward(O, Wo, G):
    """(dO, dWo) for Y = [O_1 ... O_H] Wo and G = dL/dY [B, n, d_model]:
    dWo = [O_1 ... O_H]^T G summed over the batch, and dO_h the column block h
    of G Wo^T, since the concatenation only copies entries (Problem 10)."""
    O = np.asarray(O, dtype=np.float64)
    Wo = np.asarray(Wo, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    H = O.shape[1]
    dWo = grad_weight(merge_heads(O), G)
    dO = split_heads(G @ Wo.T, H)
    return dO, dWo
