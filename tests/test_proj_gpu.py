"""GPU parity of the projection and input gradients (attn_proj_bwd) against
the float64 oracle ("Lesson 4", Step 4; "Attention backward", Problem 7), on
the same bf16-rounded inputs. Tolerance: max|gpu - ref| / max|ref| per output,
2e-2 (bf16 operands and result, fp32 accumulation)."""
import numpy as np
import pytest
import torch

import oracle.ref as ref
from parity_util import TOL, rel_err, to64

pytestmark = pytest.mark.gpu

lib = pytest.importorskip("scaled_dot_product_saving_b200")


def _inputs(B, n, d_model, H, d, dv, seed):
    g = torch.Generator().manual_seed(seed)
    def r(*shape, std=1.0):
        return (torch.randn(*shape, generator=g) * std).to(torch.bfloat16)
    X = r(B, n, d_model)
    Wq = r(d_model, H * d, std=d_model ** -0.5)
    Wk = r(d_model, H * d, std=d_model ** -0.5)
    Wv = r(d_model, H * dv, std=d_model ** -0.5)
    dQ, dK, dV = r(B, H, n, d), r(B, H, n, d), r(B, H, n, dv)
    return X, Wq, Wk, Wv, dQ, dK, dV


@pytest.mark.parametrize("B,n,d_model,H,d,dv", [
    (2, 200, 200, 3, 64, 40),       # ragged in every GEMM dimension, dv != d
    (1, 300, 256, 2, 128, 128),
    (2, 64, 8, 1, 8, 8),            # the smallest widths
    (4, 512, 1024, 8, 128, 128),    # several tiles in M, N and K
])
def test_projection_backward(B, n, d_model, H, d, dv):
    cpu = _inputs(B, n, d_model, H, d, dv, seed=B * 100 + n + d_model)
    dev = torch.device("cuda:0")
    got = lib.attn_proj_bwd(*(t.to(dev) for t in cpu))
    torch.cuda.synchronize()
    assert lib.attn_get_device_error() == 0
    assert lib.attn_last_launch_count() == 10
    X, Wq, Wk, Wv, dQ, dK, dV = (t.to(torch.float64).numpy() for t in cpu)
    want = ref.projection_backward(X, Wq, Wk, Wv, dQ, dK, dV)
    errs = {name: rel_err(to64(g), w) for name, g, w in zip(("dX", "dWq", "dWk", "dWv"), got, want)}
    bad = {k: v for k, v in errs.items() if not v <= TOL["bf16"]}
    assert not bad, errs


def test_projection_backward_after_attention():
    """The chain of Problem 7 end to end: X -> Q, K, V (torch, plumbing) ->
    attn_fwd -> attn_bwd -> attn_proj_bwd, against the oracle's chain."""
    B, n, d_model, H, d = 1, 256, 256, 2, 128
    X, Wq, Wk, Wv, _, _, _ = _inputs(B, n, d_model, H, d, d, seed=5)
    g = torch.Generator().manual_seed(6)
    G = torch.randn(B, H, n, d, generator=g).to(torch.bfloat16)
    dev = torch.device("cuda:0")
    Xd, Wqd, Wkd, Wvd, Gd = (t.to(dev) for t in (X, Wq, Wk, Wv, G))
    split = lambda T: T.reshape(B, n, H, -1).transpose(1, 2).contiguous()
    Q, K, V = (split((Xd.float() @ W.float()).to(torch.bfloat16)) for W in (Wqd, Wkd, Wvd))
    o, lse = lib.attn_fwd(Q, K, V, causal=True)
    dq, dk, dv = lib.attn_bwd(Q, K, V, o, Gd, lse, causal=True)
    got = lib.attn_proj_bwd(Xd, Wqd, Wkd, Wvd, dq, dk, dv)
    torch.cuda.synchronize()
    assert lib.attn_get_device_error() == 0
    # oracle chain on the same bf16 Q, K, V (their rounding is an input here)
    Qn, Kn, Vn = (t.cpu().to(torch.float64).numpy() for t in (Q, K, V))
    dQr, dKr, dVr = ref.attention_backward(Qn, Kn, Vn, G.to(torch.float64).numpy(), True)
    want = ref.projection_backward(*(t.to(torch.float64).numpy() for t in (X, Wq, Wk, Wv)),
                                   dQr, dKr, dVr)
    errs = {name: rel_err(to64(g_), w) for name, g_, w in zip(("dX", "dWq", "dWk", "dWv"), got, want)}
    # The same 2e-2 bar: the chain rounds to bf16 twice (the attention
    # gradients, then the projection outputs), which a CPU emulation of this
    # arithmetic on these inputs puts at about 4e-3 of max|ref|.
    assert all(v <= TOL["bf16"] for v in errs.values()), errs


@pytest.mark.parametrize("B,n,d_model,H,dv", [
    (2, 200, 200, 3, 40),      # ragged everywhere
    (1, 384, 512, 4, 128),
    (2, 64, 8, 1, 8),
])
def test_output_projection_backward(B, n, d_model, H, dv):
    g = torch.Generator().manual_seed(B + n + d_model)
    O = torch.randn(B, H, n, dv, generator=g).to(torch.bfloat16)
    Wo = (torch.randn(H * dv, d_model, generator=g) * (H * dv) ** -0.5).to(torch.bfloat16)
    G = torch.randn(B, n, d_model, generator=g).to(torch.bfloat16)
    dev = torch.device("cuda:0")
    dO, dWo = lib.attn_outproj_bwd(O.to(dev), Wo.to(dev), G.to(dev))
    torch.cuda.synchronize()
    assert lib.attn_get_device_error() == 0
    assert lib.attn_last_launch_count() == 4
    want_dO, want_dWo = ref.output_projection_backward(*(t.to(torch.float64).numpy() for t in (O, Wo, G)))
    errs = {"dO": rel_err(to64(dO), want_dO), "dWo": rel_err(to64(dWo), want_dWo)}
    assert all(v <= TOL["bf16"] for v in errs.values()), errs
