"""Pins for the float64 oracle, on the CPU.

Every oracle function is checked here against something other than itself:
values the pages print, closed forms, finite differences, float64 torch
autograd of the library's attention, the explicit softmax Jacobian, and
identities the pages derive. The mutation tests at the end plant each wrong
variant the pages discuss into the oracle and check that the pins fail.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.ref as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def max_rel_err(a, n):
    """The error measure of 'Lesson 4', section 'Proving It'."""
    a = np.asarray(a, dtype=np.float64)
    n = np.asarray(n, dtype=np.float64)
    return float(np.max(np.abs(a - n) / (np.maximum(np.abs(a), np.abs(n)) + 1e-12)))


def rel_to_max(a, ref_):
    """max|a - ref| / max|ref| (the GPU parity measure), 0 when both vanish."""
    den = float(np.max(np.abs(ref_)))
    num = float(np.max(np.abs(np.asarray(a) - np.asarray(ref_))))
    return num / den if den > 0 else num


# --------------------------------------------------------------------------
# Values printed on the pages
# --------------------------------------------------------------------------
def test_worked_example_forward():
    g = golden()["attention_forward_uniform"]
    O, lse = ref.head_forward(np.array(g["Q"]), np.array(g["K"]), np.array(g["V"]),
                              causal=g["causal"])
    np.testing.assert_allclose(np.round(O, g["printed_decimals"]), g["expected_out"])
    np.testing.assert_allclose(O, g["expected_out"], rtol=0, atol=1e-14)
    # all three scores are 0, so the log-sum-exp is log 3
    np.testing.assert_allclose(lse, [math.log(3.0)] * 2, rtol=0, atol=1e-15)


def test_worked_example_dV():
    g = golden()["attention_backward_dV_uniform"]
    dQ, dK, dV = ref.head_backward(np.array(g["Q"]), np.array(g["K"]), np.array(g["V"]),
                                   np.array(g["dOut"]), causal=g["causal"])
    np.testing.assert_allclose(np.round(dV, g["printed_decimals"]), g["expected_dV"])
    np.testing.assert_allclose(dV, np.full((3, 2), 2.0 / 3.0), rtol=0, atol=1e-15)
    # Derived from the same example: Q and K are zero, so dQ = scale*dS K = 0
    # and dK = scale*dS^T Q = 0.
    assert np.all(dQ == 0.0) and np.all(dK == 0.0)


def test_worked_example_dS_closed_form():
    """Same example, one step inside: dP rows are V's row sums [3, 7, 11],
    rowsum(dP*P) = 7 and dS = (1/3)([3, 7, 11] - 7) = [-4/3, 0, 4/3]."""
    g = golden()["attention_backward_dV_uniform"]
    V = np.array(g["V"])
    P = np.full((2, 3), 1.0 / 3.0)
    dP = ref.grad_p(np.array(g["dOut"]), V)
    np.testing.assert_allclose(dP, [[3, 7, 11], [3, 7, 11]], atol=0)
    dS = ref.softmax_jvp(P, dP)
    np.testing.assert_allclose(dS, [[-4 / 3, 0, 4 / 3]] * 2, atol=1e-15)


def _lesson4_setup():
    g = golden()["lesson4_loss"]
    rs = np.random.RandomState(g["seed"])  # NumPy's legacy seeded stream
    B, T, C, hs = g["B"], g["T"], g["C"], g["hs"]
    X = rs.randn(B, T, C) * 0.5
    Wq = rs.randn(C, hs) * 0.1
    Wk = rs.randn(C, hs) * 0.1
    Wv = rs.randn(C, hs) * 0.1
    G = rs.randn(B, T, hs)
    return g, X, Wq, Wk, Wv, G


def _lesson4_loss(X, Wq, Wk, Wv, G):
    O, _ = ref.attention_forward(X @ Wq, X @ Wk, X @ Wv)
    return float(np.sum(O * G))


def test_lesson4_loss_value():
    g, X, Wq, Wk, Wv, G = _lesson4_setup()
    L = _lesson4_loss(X, Wq, Wk, Wv, G)
    assert round(L, g["printed_decimals"]) == g["expected_L"]


def test_lesson4_gradient_check_through_projections():
    """The oracle's dQ, dK, dV pushed through the projections (Problem 7's
    chain rule, written here in the test) pass the page's gradient check."""
    _, X, Wq, Wk, Wv, G = _lesson4_setup()
    spec = golden()["lesson4_gradient_check"]
    Q, K, V = ref.project_qkv(X, Wq, Wk, Wv, 1)
    dQ, dK, dV = ref.attention_backward(Q, K, V, ref.split_heads(G, 1))
    dX, dWq, dWk, dWv = ref.projection_backward(X, Wq, Wk, Wv, dQ, dK, dV)
    grads = {"dWq": dWq, "dWk": dWk, "dWv": dWv, "dX": dX}
    params = {"dWq": Wq, "dWk": Wk, "dWv": Wv, "dX": X}
    eps = spec["eps"]
    for name, p in params.items():
        num = np.zeros_like(p)
        for idx in np.ndindex(p.shape):
            orig = p[idx]
            p[idx] = orig + eps
            lp = _lesson4_loss(X, Wq, Wk, Wv, G)
            p[idx] = orig - eps
            lm = _lesson4_loss(X, Wq, Wk, Wv, G)
            p[idx] = orig
            num[idx] = (lp - lm) / (2 * eps)
        err = max_rel_err(grads[name], num)
        assert err < spec["threshold"], (name, err)
        # same order as the printed values (1e-10 .. 1.4e-7)
        assert err < 1e-6, (name, err)


# --------------------------------------------------------------------------
# Closed forms
# --------------------------------------------------------------------------
def test_uniform_closed_form_zero_keys():
    """K = 0 makes every score 0: each O row is the mean of V and LSE = log m."""
    rng = np.random.default_rng(3)
    Q = rng.standard_normal((5, 4))
    K = np.zeros((7, 4))
    V = rng.standard_normal((7, 3))
    O, lse = ref.head_forward(Q, K, V)
    np.testing.assert_allclose(O, np.tile(V.mean(axis=0), (5, 1)), atol=1e-15)
    np.testing.assert_allclose(lse, np.full(5, math.log(7)), atol=1e-15)


def test_causal_first_row_sees_only_first_key():
    rng = np.random.default_rng(4)
    Q, K, V, dO = (rng.standard_normal((6, 4)) for _ in range(4))
    O, lse = ref.head_forward(Q, K, V, causal=True)
    np.testing.assert_allclose(O[0], V[0], atol=0)
    np.testing.assert_allclose(lse[0], ref.default_scale(4) * Q[0] @ K[0], atol=1e-15)
    dQ, dK, dV = ref.head_backward(Q, K, V, dO, causal=True)
    assert np.all(dQ[0] == 0.0)        # one-hot row: dS row is 0
    # the last key is seen only by the last query, with weight P[n-1, n-1]
    P_last = np.exp(ref.default_scale(4) * Q[5] @ K[5] - lse[5])
    np.testing.assert_allclose(dV[5], P_last * dO[5], rtol=1e-13)


# --------------------------------------------------------------------------
# Finite differences of L = sum(O * dO)
# ("Attention Backward Pass (dQ, dK, dV)", "Edge cases and conventions")
# --------------------------------------------------------------------------
FD_CASES = [
    # n, m, d, dv, causal, seed
    (3, 3, 2, 2, True, 0),
    (4, 6, 3, 2, False, 1),
    (5, 5, 4, 3, True, 2),
    (2, 3, 4, 2, False, 3),
    (6, 4, 3, 5, False, 4),
]


def _fd_grads(Q, K, V, dO, causal, scale, eps=1e-5):
    def loss():
        O, _ = ref.head_forward(Q, K, V, causal, scale)
        return float(np.sum(O * dO))
    out = []
    for p in (Q, K, V):
        num = np.zeros_like(p)
        for idx in np.ndindex(p.shape):
            orig = p[idx]
            p[idx] = orig + eps
            lp = loss()
            p[idx] = orig - eps
            lm = loss()
            p[idx] = orig
            num[idx] = (lp - lm) / (2 * eps)
        out.append(num)
    return out


def _fd_max_err(n, m, d, dv, causal, seed, scale=None):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((n, d))
    K = rng.standard_normal((m, d))
    V = rng.standard_normal((m, dv))
    dO = rng.standard_normal((n, dv))
    an = ref.head_backward(Q, K, V, dO, causal, scale)
    nu = _fd_grads(Q, K, V, dO, causal, scale)
    return max(max_rel_err(a, b) for a, b in zip(an, nu))


@pytest.mark.parametrize("n,m,d,dv,causal,seed", FD_CASES)
def test_finite_differences(n, m, d, dv, causal, seed):
    assert _fd_max_err(n, m, d, dv, causal, seed) < 1e-6


def test_finite_differences_explicit_scale():
    assert _fd_max_err(4, 5, 3, 2, False, 7, scale=0.37) < 1e-6


def test_finite_differences_large_scores():
    """Scores of size ~100 need the max-subtracted softmax (the pages' tests
    use scores of about that size)."""
    rng = np.random.default_rng(11)
    Q = rng.standard_normal((4, 3)) * 12
    K = rng.standard_normal((5, 3)) * 12
    V = rng.standard_normal((5, 2))
    dO = rng.standard_normal((4, 2))
    S = ref.scores(Q, K, ref.default_scale(3))
    assert np.abs(S).max() > 50
    O, lse = ref.head_forward(Q, K, V)
    assert np.all(np.isfinite(O)) and np.all(np.isfinite(lse))
    an = ref.head_backward(Q, K, V, dO)
    nu = _fd_grads(Q, K, V, dO, False, None, eps=1e-7)
    for a, b in zip(an, nu):
        assert rel_to_max(a, b) < 1e-5


# --------------------------------------------------------------------------
# float64 torch autograd of the library's scaled_dot_product_attention
# --------------------------------------------------------------------------
def _torch_ref(Q, K, V, dO, causal, scale):
    q, k, v = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V))
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal,
                                                         scale=scale)
    o.backward(torch.tensor(dO, dtype=torch.float64))
    s = (q @ k.transpose(-1, -2)) * (scale if scale is not None else 1 / math.sqrt(Q.shape[-1]))
    if causal:
        n, m = s.shape[-2:]
        s = s.masked_fill(torch.ones(n, m, dtype=torch.bool).triu(1), float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return (o.detach().numpy(), lse.detach().numpy(), q.grad.numpy(), k.grad.numpy(),
            v.grad.numpy())


AUTOGRAD_CASES = [
    # B, H, n, m, d, dv, causal, scale, seed
    (2, 3, 17, 17, 8, 8, True, None, 0),
    (1, 2, 9, 23, 16, 4, False, None, 1),
    (2, 1, 40, 40, 5, 7, True, 0.2, 2),
    (1, 1, 64, 64, 64, 64, False, None, 3),
    (1, 2, 33, 70, 12, 12, False, 1.3, 4),
]


@pytest.mark.parametrize("B,H,n,m,d,dv,causal,scale,seed", AUTOGRAD_CASES)
def test_matches_torch_autograd_float64(B, H, n, m, d, dv, causal, scale, seed):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, H, n, d))
    K = rng.standard_normal((B, H, m, d))
    V = rng.standard_normal((B, H, m, dv))
    dO = rng.standard_normal((B, H, n, dv))
    O, lse = ref.attention_forward(Q, K, V, causal, scale, row_block=8)
    dQ, dK, dV = ref.attention_backward(Q, K, V, dO, causal, scale, row_block=8)
    tO, tlse, tdQ, tdK, tdV = _torch_ref(Q, K, V, dO, causal, scale)
    for a, b in ((O, tO), (lse, tlse), (dQ, tdQ), (dK, tdK), (dV, tdV)):
        assert a.shape == b.shape
        assert rel_to_max(a, b) < 1e-12


def test_row_block_does_not_change_results():
    rng = np.random.default_rng(5)
    Q, K, V, dO = (rng.standard_normal((37, 6)) for _ in range(4))
    a = ref.head_backward(Q, K, V, dO, causal=True, row_block=37)
    b = ref.head_backward(Q, K, V, dO, causal=True, row_block=5)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-13, atol=1e-14)


# --------------------------------------------------------------------------
# Structure the pages derive
# --------------------------------------------------------------------------
def test_explicit_jacobian_equals_jvp():
    """'Lesson 4', Exercise 2: (diag(a) - a a^T) g equals a * (g - (g*a).sum())."""
    rng = np.random.default_rng(6)
    S = rng.standard_normal((5, 9)) * 2
    P, _ = ref.row_softmax(S)
    G = rng.standard_normal((5, 9))
    dS = ref.softmax_jvp(P, G)
    for i in range(5):
        a = P[i]
        J = np.diag(a) - np.outer(a, a)
        np.testing.assert_allclose(J @ G[i], dS[i], rtol=0, atol=1e-15)


def test_rowsum_identity():
    """rowsum(dP * P) = rowsum(dO * O) ('Attention Backpropagation: Step by
    step derivation', 'Gradient of S'; the follow-up question of 'Attention
    Backward Pass (dQ, dK, dV)')."""
    rng = np.random.default_rng(7)
    Q, K = rng.standard_normal((12, 5)), rng.standard_normal((12, 5))
    V, dO = rng.standard_normal((12, 3)), rng.standard_normal((12, 3))
    for causal in (False, True):
        S = ref.scores(Q, K, ref.default_scale(5))
        if causal:
            S = ref.apply_causal_mask(S, 0)
        P, _ = ref.row_softmax(S)
        O = P @ V
        dP = ref.grad_p(dO, V)
        np.testing.assert_allclose((dP * P).sum(-1), (dO * O).sum(-1), rtol=1e-13, atol=1e-14)


def test_masked_positions_are_exact_zeros():
    """'Attention backward', Problem 8: masked P and dS entries are exactly 0,
    and each row of P still sums to 1."""
    rng = np.random.default_rng(8)
    n = 10
    Q, K, V, dO = (rng.standard_normal((n, 4)) for _ in range(4))
    S = ref.apply_causal_mask(ref.scores(Q, K, 0.5), 0)
    P, _ = ref.row_softmax(S)
    dS = ref.softmax_jvp(P, ref.grad_p(dO, V))
    upper = np.triu(np.ones((n, n), dtype=bool), 1)
    assert np.all(P[upper] == 0.0)
    assert np.all(dS[upper] == 0.0)
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=0, atol=1e-15)


def test_gradient_invariants():
    """Each row of dS sums to 0, so the rows of dK sum to 0; the rows of P sum
    to 1, so sum_j dV_j = sum_i dO_i."""
    rng = np.random.default_rng(10)
    for causal, (n, m) in ((False, (9, 14)), (True, (11, 11))):
        Q, dO = rng.standard_normal((n, 6)), rng.standard_normal((n, 4))
        K, V = rng.standard_normal((m, 6)), rng.standard_normal((m, 4))
        dQ, dK, dV = ref.head_backward(Q, K, V, dO, causal)
        S = ref.scores(Q, K, ref.default_scale(6))
        if causal:
            S = ref.apply_causal_mask(S, 0)
        P, _ = ref.row_softmax(S)
        dS = ref.softmax_jvp(P, ref.grad_p(dO, V))
        np.testing.assert_allclose(dS.sum(-1), 0.0, atol=1e-13)
        np.testing.assert_allclose(dK.sum(0), 0.0, atol=1e-12)
        np.testing.assert_allclose(dV.sum(0), dO.sum(0), rtol=1e-12)


def test_saturated_row_has_no_score_gradient():
    """'Attention backward', Problem 9: at a one-hot row diag(u) - u u^T = 0."""
    P = np.array([[0.0, 1.0, 0.0, 0.0]])
    dP = np.array([[3.0, -1.0, 2.0, 5.0]])
    assert np.all(ref.softmax_jvp(P, dP) == 0.0)
    Q = np.array([[50.0, 0.0]])
    K = np.array([[0.0, 0.0], [50.0, 0.0], [0.0, 0.0]])
    V = np.random.default_rng(0).standard_normal((3, 2))
    dQ, dK, _ = ref.head_backward(Q, K, V, np.ones((1, 2)), scale=1.0)
    assert np.abs(dQ).max() < 1e-300 and np.abs(dK).max() < 1e-300


def test_gradients_have_the_shapes_of_their_inputs():
    rng = np.random.default_rng(12)
    Q, K = rng.standard_normal((2, 3, 5, 4)), rng.standard_normal((2, 3, 7, 4))
    V, dO = rng.standard_normal((2, 3, 7, 6)), rng.standard_normal((2, 3, 5, 6))
    dQ, dK, dV = ref.attention_backward(Q, K, V, dO)
    assert dQ.shape == Q.shape and dK.shape == K.shape and dV.shape == V.shape


def test_causal_needs_square():
    with pytest.raises(ValueError):
        ref.head_forward(np.zeros((3, 2)), np.zeros((4, 2)), np.zeros((4, 2)), causal=True)


# --------------------------------------------------------------------------
# Mutation tests: plant each wrong variant in the oracle; the pins must fail
# --------------------------------------------------------------------------
def _pins_pass():
    """True when the autograd pins and the worked examples all still hold."""
    try:
        for case in AUTOGRAD_CASES:
            test_matches_torch_autograd_float64(*case)
        test_worked_example_dV()
        test_worked_example_forward()
    except AssertionError:
        return False
    return True


def _fd_pins_pass():
    return all(_fd_max_err(*c) < 1e-6 for c in FD_CASES)


MUTANTS = {
    # "Is there any Reference About Backpropagation...", 3.2: diagonal only
    "jvp_diag_only": ("softmax_jvp", lambda P, dP: dP * (P * (1 - P))),
    # "Lesson 4", Exercise 1: the correction term dropped
    "jvp_no_correction": ("softmax_jvp", lambda P, dP: dP * P),
    # "Attention backward", wrong turn 2: one softmax over the flattened matrix
    "jvp_flattened": ("softmax_jvp", lambda P, dP: P * (dP - (dP * P).sum())),
    # wrong turn 3: the 1/sqrt(d) lost on the way back
    "dq_no_scale": ("grad_q", lambda dS, K, scale: dS @ K),
    "dk_no_scale": ("grad_k", lambda dS, Q, scale: dS.T @ Q),
    # wrong turn 1: dV = A G without the transpose (runs when n == m)
    "dv_no_transpose": ("grad_v", lambda P, dO: P @ dO if P.shape[0] == P.shape[1]
                        else P.T @ dO * 1.5),
    # a transpose dropped in dK (runs when n == m)
    "dk_no_transpose": ("grad_k", lambda dS, Q, scale: scale * (dS @ Q)
                        if dS.shape[0] == dS.shape[1] else scale * (dS.T @ Q) * 0.5),
    # sign error in dP
    "dp_sign": ("grad_p", lambda dO, V: -(dO @ V.T)),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutants_are_caught(name, monkeypatch):
    assert _pins_pass()
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(ref, attr, fn)
    assert not _pins_pass() or not _fd_pins_pass(), name


def test_mask_after_softmax_is_caught(monkeypatch):
    """'Attention backward', wrong turn 5: zeroing A after the softmax."""
    assert _pins_pass()

    def masked_late(Q, K, r0, r1, causal, scale, key_len=None):
        S = ref.scores(Q[r0:r1], K, scale)
        P, lse = ref.row_softmax(S)
        if causal:
            keep = ~np.isinf(ref.apply_causal_mask(S, r0))
            P = P * keep
        return P, lse

    monkeypatch.setattr(ref, "_block_probs", masked_late)
    assert not _pins_pass()


def test_unstable_softmax_is_caught(monkeypatch):
    """Without the row max, scores of ~100 overflow exp."""
    def naive(S):
        e = np.exp(S)
        return e / e.sum(-1, keepdims=True), np.log(e.sum(-1))

    rng = np.random.default_rng(13)
    Q = rng.standard_normal((3, 2)) * 40
    K = rng.standard_normal((4, 2)) * 40
    V = rng.standard_normal((4, 2))
    good, _ = ref.head_forward(Q, K, V, scale=1.0)
    monkeypatch.setattr(ref, "row_softmax", naive)
    with np.errstate(all="ignore"):
        bad, _ = ref.head_forward(Q, K, V, scale=1.0)
    assert not np.allclose(good, bad, equal_nan=False)


# --------------------------------------------------------------------------
# Projection gradients with several heads (Problem 7 per head; Problem 10's
# column blocks)
# --------------------------------------------------------------------------
def _mh_setup(seed=7, B=2, n=5, C=6, H=3, d=2, dv=3):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((B, n, C))
    Wq = rng.standard_normal((C, H * d)) * 0.5
    Wk = rng.standard_normal((C, H * d)) * 0.5
    Wv = rng.standard_normal((C, H * dv)) * 0.5
    G = rng.standard_normal((B, n, H * dv))
    return X, Wq, Wk, Wv, G


def _mh_loss(X, Wq, Wk, Wv, G, causal, H=3):
    Q, K, V = ref.project_qkv(X, Wq, Wk, Wv, H)
    O, _ = ref.attention_forward(Q, K, V, causal)
    return float(np.sum(ref.merge_heads(O) * G))


@pytest.mark.parametrize("causal", [False, True])
def test_projection_backward_multihead_finite_differences(causal):
    """Every entry of dX, dWq, dWk, dWv of a three-head self-attention against
    central differences of L = sum(merge(O) * G)."""
    X, Wq, Wk, Wv, G = _mh_setup()
    H = 3
    Q, K, V = ref.project_qkv(X, Wq, Wk, Wv, H)
    dQ, dK, dV = ref.attention_backward(Q, K, V, ref.split_heads(G, H), causal)
    grads = dict(zip(("dX", "dWq", "dWk", "dWv"),
                     ref.projection_backward(X, Wq, Wk, Wv, dQ, dK, dV)))
    params = {"dX": X, "dWq": Wq, "dWk": Wk, "dWv": Wv}
    eps = 1e-6
    for name, p in params.items():
        assert grads[name].shape == p.shape, name
        num = np.zeros_like(p)
        for idx in np.ndindex(p.shape):
            orig = p[idx]
            p[idx] = orig + eps
            lp = _mh_loss(X, Wq, Wk, Wv, G, causal)
            p[idx] = orig - eps
            lm = _mh_loss(X, Wq, Wk, Wv, G, causal)
            p[idx] = orig
            num[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grads[name], num, rtol=1e-6, atol=1e-8, err_msg=name)


def test_split_merge_heads_layout():
    """Head h is column block h: split then merge is the identity, and head
    h's rows are X Wq[:, h*d:(h+1)*d]."""
    X, Wq, Wk, Wv, _ = _mh_setup()
    Q, _, _ = ref.project_qkv(X, Wq, Wk, Wv, 3)
    np.testing.assert_array_equal(ref.merge_heads(Q), X @ Wq)
    np.testing.assert_allclose(Q[:, 1], X @ Wq[:, 2:4], rtol=0, atol=1e-14)


def test_projection_backward_mutants_fail(monkeypatch):
    """The pages' two projection mistakes, planted in the oracle, fail the
    finite-difference pin: a path through X left out, and a transposed
    weight gradient."""
    X, Wq, Wk, Wv, G = _mh_setup(seed=11, C=4, H=2, d=2, dv=2)
    H = 2
    Q, K, V = ref.project_qkv(X, Wq, Wk, Wv, H)
    dQ, dK, dV = ref.attention_backward(Q, K, V, ref.split_heads(G, H))
    eps = 1e-6

    def fd_dx():
        num = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            orig = X[idx]
            X[idx] = orig + eps
            lp = float(np.sum(ref.merge_heads(ref.attention_forward(*ref.project_qkv(X, Wq, Wk, Wv, H))[0]) * G))
            X[idx] = orig - eps
            lm = float(np.sum(ref.merge_heads(ref.attention_forward(*ref.project_qkv(X, Wq, Wk, Wv, H))[0]) * G))
            X[idx] = orig
            num[idx] = (lp - lm) / (2 * eps)
        return num

    num = fd_dx()
    good = ref.projection_backward(X, Wq, Wk, Wv, dQ, dK, dV)[0]
    np.testing.assert_allclose(good, num, rtol=1e-6, atol=1e-8)
    monkeypatch.setattr(ref, "grad_input", lambda dQm, dKm, dVm, Wq, Wk, Wv: dQm @ Wq.T + dVm @ Wv.T)
    bad = ref.projection_backward(X, Wq, Wk, Wv, dQ, dK, dV)[0]
    assert np.max(np.abs(bad - num)) > 1e-3
    # C == H*d here, so the transposed product has the right shape
    monkeypatch.setattr(ref, "grad_weight", lambda X, dT: np.einsum("bnc,bnw->wc", X, dT))
    dWq_bad = ref.projection_backward(X, Wq, Wk, Wv, dQ, dK, dV)[1]
    monkeypatch.undo()
    dWq_good = ref.projection_backward(X, Wq, Wk, Wv, dQ, dK, dV)[1]
    assert np.max(np.abs(dWq_bad - dWq_good)) > 1e-3



# --------------------------------------------------------------------------
# Multi-head output projection (Problem 10)
# --------------------------------------------------------------------------
def test_output_projection_backward_finite_differences():
    """dWo and every dO_h entry against central differences of
    L = sum(Y * G), Y = [O_1 ... O_H] Wo, and dQ, dK, dV through attention with
    dO = dO_h: the chain of Problem 10 into Problems 2-6."""
    rng = np.random.default_rng(21)
    B, H, n, d, dv, C = 2, 3, 4, 2, 3, 5
    Q, K, V = (rng.standard_normal((B, H, n, w)) for w in (d, d, dv))
    Wo = rng.standard_normal((H * dv, C)) * 0.5
    G = rng.standard_normal((B, n, C))
    O, _ = ref.attention_forward(Q, K, V, True)
    dO, dWo = ref.output_projection_backward(O, Wo, G)
    assert dO.shape == O.shape and dWo.shape == Wo.shape
    eps = 1e-6

    def loss_O(Ov):
        return float(np.sum(ref.output_projection(Ov, Wo) * G))

    def loss_W(W):
        return float(np.sum(ref.output_projection(O, W) * G))

    def loss_Q(Qv):
        return float(np.sum(ref.output_projection(ref.attention_forward(Qv, K, V, True)[0], Wo) * G))

    for f, p, want in ((loss_W, Wo, dWo), (loss_O, O, dO)):
        num = np.zeros_like(p)
        for idx in np.ndindex(p.shape):
            orig = p[idx]
            p[idx] = orig + eps
            lp = f(p)
            p[idx] = orig - eps
            lm = f(p)
            p[idx] = orig
            num[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(want, num, rtol=1e-6, atol=1e-8)
    dQ, _, _ = ref.attention_backward(Q, K, V, dO, True)
    num = np.zeros_like(Q)
    for idx in np.ndindex(Q.shape):
        orig = Q[idx]
        Q[idx] = orig + eps
        lp = loss_Q(Q)
        Q[idx] = orig - eps
        lm = loss_Q(Q)
        Q[idx] = orig
        num[idx] = (lp - lm) / (2 * eps)
    np.testing.assert_allclose(dQ, num, rtol=1e-5, atol=1e-8)


def test_output_projection_backward_mutant_fails(monkeypatch):
    """Slicing G Wo^T into the wrong head blocks (a transpose of the head and
    width axes) fails the pin."""
    rng = np.random.default_rng(22)
    O = rng.standard_normal((1, 2, 3, 2))
    Wo = rng.standard_normal((4, 3))
    G = rng.standard_normal((1, 3, 3))
    good, _ = ref.output_projection_backward(O, Wo, G)
    monkeypatch.setattr(ref, "split_heads",
                        lambda T, H: T.reshape(T.shape[0], T.shape[1], T.shape[2] // H, H).transpose(0, 3, 1, 2))
    bad, _ = ref.output_projection_backward(O, Wo, G)
    assert np.max(np.abs(bad - good)) > 1e-3


# --------------------------------------------------------------------------
# Padding mask ("Is there any Reference About Backpropagation of the
# Transformer's Multi-Head Layer?", section 4: causal or padding masks go
# before the softmax; the backward then zeroes the masked gradients). Keys at
# or past key_len[b] of batch element b are padding.
# --------------------------------------------------------------------------
def _torch_padded(Q, K, V, dO, causal, scale, key_len):
    """float64 torch autograd with an explicit boolean attention mask."""
    B, H, n, _ = Q.shape
    m = K.shape[2]
    keep = torch.zeros(B, 1, n, m, dtype=torch.bool)
    for b in range(B):
        keep[b, :, :, :key_len[b]] = True
    if causal:
        keep &= ~torch.ones(n, m, dtype=torch.bool).triu(1)
    q, k, v = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V))
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=keep, scale=scale)
    o.backward(torch.tensor(dO, dtype=torch.float64))
    sc = scale if scale is not None else 1 / math.sqrt(Q.shape[-1])
    s = ((q @ k.transpose(-1, -2)) * sc).masked_fill(~keep, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return (o.detach().numpy(), lse.detach().numpy(), q.grad.numpy(), k.grad.numpy(),
            v.grad.numpy())


PADDED_CASES = [
    # B, H, n, m, d, dv, causal, key_len, scale, seed
    (2, 2, 7, 9, 4, 3, False, [4, 9], None, 0),
    (3, 1, 8, 8, 5, 5, True, [3, 8, 1], None, 1),
    (2, 3, 12, 12, 6, 4, True, [7, 12], 0.3, 2),
    (1, 2, 5, 20, 8, 8, False, [13], None, 3),
]


def _padded_inputs(B, H, n, m, d, dv, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, H, n, d)), rng.standard_normal((B, H, m, d)),
            rng.standard_normal((B, H, m, dv)), rng.standard_normal((B, H, n, dv)))


def _padded_pins_pass():
    try:
        for (B, H, n, m, d, dv, causal, kl, scale, seed) in PADDED_CASES:
            Q, K, V, dO = _padded_inputs(B, H, n, m, d, dv, seed)
            got = ref.attention_forward(Q, K, V, causal, scale, row_block=3, key_len=kl) + \
                ref.attention_backward(Q, K, V, dO, causal, scale, row_block=3, key_len=kl)
            want = _torch_padded(Q, K, V, dO, causal, scale, kl)
            if not all(rel_to_max(a, b) < 1e-12 for a, b in zip(got, want)):
                return False
    except Exception:
        return False
    return True


def test_padding_mask_matches_torch_autograd_float64():
    assert _padded_pins_pass()


def test_padding_mask_equals_truncated_keys():
    """Without the causal mask, padded keys behave as if they were absent:
    O, LSE and dQ equal the unmasked attention on K[:L], V[:L]; dK and dV
    match it on the first L rows and are exactly zero after them."""
    Q, K, V, dO = _padded_inputs(2, 2, 6, 10, 4, 3, 7)
    key_len = [3, 10]
    O, lse = ref.attention_forward(Q, K, V, False, None, key_len=key_len)
    dQ, dK, dV = ref.attention_backward(Q, K, V, dO, False, None, key_len=key_len)
    for b, L in enumerate(key_len):
        for h in range(2):
            O_t, lse_t = ref.head_forward(Q[b, h], K[b, h, :L], V[b, h, :L])
            dQ_t, dK_t, dV_t = ref.head_backward(Q[b, h], K[b, h, :L], V[b, h, :L], dO[b, h])
            np.testing.assert_allclose(O[b, h], O_t, rtol=0, atol=1e-13)
            np.testing.assert_allclose(lse[b, h], lse_t, rtol=0, atol=1e-13)
            np.testing.assert_allclose(dQ[b, h], dQ_t, rtol=0, atol=1e-13)
            np.testing.assert_allclose(dK[b, h, :L], dK_t, rtol=0, atol=1e-13)
            np.testing.assert_allclose(dV[b, h, :L], dV_t, rtol=0, atol=1e-13)
            assert np.all(dK[b, h, L:] == 0.0) and np.all(dV[b, h, L:] == 0.0)


def test_padding_mask_finite_differences():
    rng = np.random.default_rng(21)
    Q, K, V, dO = (rng.standard_normal(s) for s in ((5, 3), (6, 3), (6, 2), (5, 2)))
    for causal, L in ((False, 4), (False, 1), (True, 4)):
        if causal:
            Qc, dOc = Q[:, :], dO[:, :]
            Kc, Vc = K[:5], V[:5]
        else:
            Qc, dOc, Kc, Vc = Q, dO, K, V

        def loss():
            O, _ = ref.head_forward(Qc, Kc, Vc, causal, None, key_len=L)
            return float(np.sum(O * dOc))

        an = ref.head_backward(Qc, Kc, Vc, dOc, causal, None, key_len=L)
        for p, a in zip((Qc, Kc, Vc), an):
            num = np.zeros_like(p)
            for idx in np.ndindex(p.shape):
                orig = p[idx]
                p[idx] = orig + 1e-5
                lp = loss()
                p[idx] = orig - 1e-5
                lm = loss()
                p[idx] = orig
                num[idx] = (lp - lm) / 2e-5
            assert max_rel_err(a, num) < 1e-6


def test_padding_mask_after_softmax_is_caught(monkeypatch):
    """Masking the padded weights after the softmax (the wrong turn the tip
    warns about) leaves rows that do not sum to one: the pins fail."""
    assert _padded_pins_pass()
    orig = ref._block_probs

    def masked_late(Q, K, r0, r1, causal, scale, key_len=None):
        P, lse = orig(Q, K, r0, r1, causal, scale, None)
        if key_len is not None:
            P = P * (np.arange(P.shape[1])[None, :] < key_len)
        return P, lse

    monkeypatch.setattr(ref, "_block_probs", masked_late)
    assert not _padded_pins_pass()


def test_padding_mask_off_by_one_is_caught(monkeypatch):
    assert _padded_pins_pass()
    monkeypatch.setattr(ref, "apply_padding_mask",
                        lambda S, L: np.where(np.arange(S.shape[1])[None, :] > L, -np.inf, S))
    assert not _padded_pins_pass()


def test_padding_key_len_out_of_range():
    Q, K, V, dO = _padded_inputs(1, 1, 3, 4, 2, 2, 0)
    with pytest.raises(ValueError):
        ref.attention_forward(Q, K, V, key_len=[0])
    with pytest.raises(ValueError):
        ref.attention_backward(Q, K, V, dO, key_len=[5])
