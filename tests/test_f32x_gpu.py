"""GPU parity of the fp32 tensor-core path (every fp32 operand split into
three bf16 pieces, six piece products per product) against the float64
oracle, through the C ABI. Tolerance: the fp32 bar, max|gpu - ref| / max|ref|
per output tensor <= 1e-5, the same as the CUDA-core fp32 path."""
import pytest
import torch

import synth
from parity_util import TOL, all_heads, full_compare, heads_compare

pytestmark = pytest.mark.gpu

lib = pytest.importorskip("scaled_dot_product_saving_b200")


@pytest.fixture(autouse=True)
def _auto_path():
    lib.attn_set_path(lib.ATTN_PATH_AUTO)
    yield
    lib.attn_set_path(lib.ATTN_PATH_AUTO)


def _assert_within(errs, tol, label):
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"{label}: {errs}"


SHAPES = [
    # B, H, n, m, d, dv, causal, std_qk
    (1, 1, 64, 64, 64, 64, False, 1.0),       # one partial tile each way
    (2, 2, 300, 300, 64, 64, True, 1.0),      # causal, ragged tail, several tiles
    (1, 2, 200, 333, 40, 24, False, 1.0),     # n != m, widths below 64, d != dv
    (1, 1, 1, 1, 64, 64, True, 1.0),          # n = m = 1
    (1, 1, 1, 700, 64, 64, False, 1.0),       # a single query
    (1, 1, 130, 1, 32, 32, False, 1.0),       # a single key
    (1, 1, 257, 257, 64, 64, True, 1.0),      # one row past two tiles
    (1, 2, 256, 1024, 64, 64, False, 3.0),    # scaled scores up to about 50
    (1, 1, 129, 65, 4, 64, False, 2.0),       # the narrowest width
    (3, 1, 384, 384, 16, 48, True, 1.0),
]


@pytest.mark.parametrize("B,H,n,m,d,dv,causal,std", SHAPES)
def test_f32_tensor_path(B, H, n, m, d, dv, causal, std):
    lib.attn_set_path(lib.ATTN_PATH_TENSOR)
    w = synth.make_small(B, H, n, m, d, dv, "f32", causal, seed=B * 100 + n + m + d + dv,
                         std_qk=std)
    _assert_within(full_compare(w), TOL["f32"], w.name)


def test_f32_tensor_kernels_run():
    """AUTO takes the split-bf16 kernels for fp32 with widths <= 64."""
    w = synth.make_small(1, 2, 200, 200, 64, 64, "f32", True, seed=9)
    lib.attn_trace_begin(16)
    errs = full_compare(w)
    names = [k for k, _ in lib.attn_trace_end()]
    assert names == ["fwd_f32x", "preprocess", "bwd_f32x"], names
    assert lib.attn_last_launch_count() == 2
    _assert_within(errs, TOL["f32"], w.name)


@pytest.mark.parametrize("scale", [-0.2, 0.0, 0.4])
def test_f32_tensor_scales(scale):
    import oracle.ref as ref
    from parity_util import rel_err, to64
    w = synth.make_small(1, 1, 200, 200, 64, 64, "f32", True, seed=31)
    q, k, v, do = synth.make_inputs(w)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = lib.attn_fwd(qd, kd, vd, causal=True, scale=scale)
    dq, dk, dv = lib.attn_bwd(qd, kd, vd, o, dod, lse, causal=True, scale=scale)
    torch.cuda.synchronize()
    assert lib.attn_get_device_error() == 0
    Q, K, V, dO = (t.to(torch.float64).numpy() for t in (q, k, v, do))
    O_r, lse_r = ref.attention_forward(Q, K, V, True, scale)
    dQ_r, dK_r, dV_r = ref.attention_backward(Q, K, V, dO, True, scale)
    errs = {name: rel_err(to64(g), r) for name, g, r in
            zip(("O", "LSE", "dQ", "dK", "dV"), (o, lse, dq, dk, dv), (O_r, lse_r, dQ_r, dK_r, dV_r))}
    _assert_within(errs, TOL["f32"], f"scale={scale}")


def test_f32_full_size():
    """The fp32 workload at full size in the benchmark's launch configuration:
    every (batch, head) problem element by element, and invariants."""
    w = synth.workload("causal_b4h16_n1024_d64_f32")
    errs, inv = heads_compare(w, all_heads(w))
    _assert_within(errs, TOL["f32"], w.name)
    _assert_within(inv, TOL["f32"], w.name + " invariants")


def test_f32_tensor_matches_cuda_core_path():
    """The two fp32 paths agree with each other as well as with the oracle."""
    w = synth.make_small(1, 2, 300, 300, 48, 48, "f32", True, seed=13)
    from parity_util import gpu_run, rel_err, to64
    inputs = synth.make_inputs(w)
    _, tc = gpu_run(w, inputs)
    lib.attn_set_path(lib.ATTN_PATH_SIMT)
    _, cc = gpu_run(w, inputs)
    for name, a, b in zip(("O", "LSE", "dQ", "dK", "dV"), tc, cc):
        assert rel_err(to64(a), to64(b)) <= TOL["f32"], name
