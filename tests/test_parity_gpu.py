"""GPU parity: the CUDA path against the float64 oracle on the same seeded
inputs, through the C ABI. Tolerance: max|gpu - ref| / max|ref| per output
tensor, 1e-5 for fp32 inputs and 2e-2 for bf16 inputs (fp32 accumulation)."""
import pytest
import torch

import synth
from parity_util import TOL, all_heads, full_compare, heads_compare, scheduler_heads

pytestmark = pytest.mark.gpu

lib = pytest.importorskip("scaled_dot_product_saving_b200")


@pytest.fixture(autouse=True)
def _auto_path():
    lib.attn_set_path(lib.ATTN_PATH_AUTO)
    lib.attn_set_dq_path(lib.ATTN_DQ_AUTO)
    yield
    lib.attn_set_path(lib.ATTN_PATH_AUTO)
    lib.attn_set_dq_path(lib.ATTN_DQ_AUTO)


# The bf16 tensor-core backward's two dQ designs: partial sums reduce-added
# into an accumulator, or a separate query-tile-major pass.
DQ_PATHS = [lib.ATTN_DQ_REDUCE, lib.ATTN_DQ_SEPARATE]
DQ_IDS = ["dq_reduce", "dq_separate"]


def _tensor_bf16(dt, d, dv):
    return dt == "bf16" and d == dv and d in (64, 128)


def _assert_within(errs, tol, label):
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"{label}: {errs}"


# ----------------------------------------------------------------------------
# The single-head fp32 workload, compared in full
# ----------------------------------------------------------------------------
def test_single_head_f32_64():
    w = synth.workload("single_head_f32_64")
    _assert_within(full_compare(w), TOL["f32"], w.name)


# ----------------------------------------------------------------------------
# Small and edge shapes, compared in full. bf16 with d == dv in {64, 128}
# runs on the tensor cores; the others on the CUDA-core path.
# ----------------------------------------------------------------------------
SMALL = [
    # B, H, n, m, d, dv, dtype, causal, std_qk
    (1, 2, 384, 384, 64, 64, "bf16", True, 1.0),      # several tiles, causal
    (1, 2, 384, 384, 128, 128, "bf16", True, 1.0),
    (2, 1, 128, 128, 128, 128, "bf16", False, 1.0),   # exactly one tile
    (1, 2, 300, 300, 128, 128, "bf16", True, 1.0),    # ragged tail, causal
    (1, 2, 200, 520, 64, 64, "bf16", False, 1.0),     # n != m, both ragged
    (1, 1, 130, 1, 128, 128, "bf16", False, 1.0),     # a single key
    (1, 1, 1, 700, 64, 64, "bf16", False, 1.0),       # a single query
    (1, 1, 1, 1, 64, 64, "bf16", True, 1.0),          # n = m = 1
    (1, 2, 256, 1024, 64, 64, "bf16", False, 3.0),    # large scores, stable LSE
    (1, 1, 513, 513, 128, 128, "bf16", True, 1.0),    # one row past a tile
    (1, 2, 100, 100, 40, 40, "bf16", True, 1.0),      # CUDA-core path widths
    (1, 1, 70, 90, 32, 48, "bf16", False, 1.0),
    (2, 2, 77, 77, 24, 24, "f32", True, 1.0),
    (1, 1, 129, 65, 128, 96, "f32", False, 2.0),
]


@pytest.mark.parametrize("dq_path", DQ_PATHS, ids=DQ_IDS)
@pytest.mark.parametrize("B,H,n,m,d,dv,dt,causal,std", SMALL)
def test_small_shapes(B, H, n, m, d, dv, dt, causal, std, dq_path):
    if dq_path == lib.ATTN_DQ_SEPARATE and not _tensor_bf16(dt, d, dv):
        pytest.skip("the dQ design applies to the bf16 tensor-core path only")
    w = synth.make_small(B, H, n, m, d, dv, dt, causal, seed=B * 1000 + n + m + d, std_qk=std)
    _assert_within(full_compare(w, dq_path=dq_path), TOL[dt], w.name)


@pytest.mark.parametrize("d,causal", [(64, True), (128, False)])
def test_cuda_core_path_bf16(d, causal):
    """The CUDA-core path forced on shapes the tensor cores would take."""
    lib.attn_set_path(lib.ATTN_PATH_SIMT)
    w = synth.make_small(1, 2, 200, 200, d, d, "bf16", causal, seed=11)
    _assert_within(full_compare(w), TOL["bf16"], w.name)


@pytest.mark.parametrize("B,H,n,m,d,causal", [
    (2, 40, 700, 700, 128, True),      # 240 forward / 480 backward items: several per CTA, ragged
    (4, 50, 300, 1000, 64, False),     # 400 / 1600 items, n != m, both ragged
    (1, 160, 130, 130, 128, True),     # one-key-tile items and one-tile pairs (has no tile B)
    (1, 160, 130, 130, 64, True),      # the same at d = 64 (items of one and two query tiles)
    (3, 37, 1000, 1000, 64, True),     # d = 64, 296 key-tile items in several causal head groups
])
@pytest.mark.parametrize("dq_path", DQ_PATHS, ids=DQ_IDS)
def test_persistent_many_items(B, H, n, m, d, causal, dq_path):
    """Problems with more work items than SMs, so that every persistent CTA
    walks several items of different lengths (every head compared in full)."""
    w = synth.make_small(B, H, n, m, d, d, "bf16", causal, seed=B * H + n + d)
    _assert_within(full_compare(w, dq_path=dq_path), TOL["bf16"], w.name)


@pytest.mark.parametrize("d,causal,scale", [
    (128, True, -0.09),    # negative scale: the softmax keeps the smallest raw score
    (64, False, -0.3),
    (128, False, 0.0),     # zero scale: uniform weights, dQ = dK = 0
    (64, True, 0.35),      # scale above 1/sqrt(d)
])
@pytest.mark.parametrize("dq_path", DQ_PATHS, ids=DQ_IDS)
def test_scale_values(d, causal, scale, dq_path):
    """Scales other than 1/sqrt(d) through the tensor-core path."""
    lib.attn_set_dq_path(dq_path)
    import numpy as np
    import oracle.ref as ref
    from parity_util import rel_err, to64
    w = synth.make_small(1, 2, 300, 300, d, d, "bf16", causal, seed=77 + d)
    q, k, v, do = synth.make_inputs(w)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = lib.attn_fwd(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = lib.attn_bwd(qd, kd, vd, o, dod, lse, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert lib.attn_get_device_error() == 0
    Q, K, V, dO = (t.to(torch.float64).numpy() for t in (q, k, v, do))
    O_r, lse_r = ref.attention_forward(Q, K, V, causal, scale)
    dQ_r, dK_r, dV_r = ref.attention_backward(Q, K, V, dO, causal, scale)
    errs = {name: rel_err(to64(g), r) for name, g, r in
            zip(("O", "LSE", "dQ", "dK", "dV"), (o, lse, dq, dk, dv), (O_r, lse_r, dQ_r, dK_r, dV_r))}
    if scale == 0.0:
        assert np.max(np.abs(dQ_r)) == 0.0 and np.max(np.abs(dK_r)) == 0.0
    _assert_within(errs, TOL["bf16"], f"d={d} causal={causal} scale={scale}")


@pytest.mark.parametrize("dq_path,launches", [(lib.ATTN_DQ_REDUCE, 2), (lib.ATTN_DQ_SEPARATE, 3)],
                         ids=DQ_IDS)
def test_tensor_path_is_taken(dq_path, launches):
    """preprocess + the fused backward (dQ written in it), or preprocess +
    the dK/dV pass + the dQ pass."""
    lib.attn_set_path(lib.ATTN_PATH_TENSOR)
    w = synth.make_small(1, 1, 256, 256, 64, 64, "bf16", True, seed=3)
    _assert_within(full_compare(w, dq_path=dq_path), TOL["bf16"], w.name)
    assert lib.attn_last_launch_count() == launches      # of the backward call


# ----------------------------------------------------------------------------
# The four bf16 workloads at full size, in the launch configuration the
# benchmark times, compared element by element with the oracle head by head
# (the worst head's error is kept), plus invariants over all heads:
#  - the two small workloads: every head;
#  - B2 H32 N4096: the first, middle and last head of every head group of the
#    persistent schedules (groups of about 256 work items);
#  - B1 H32 N16384: the groups there are two heads each; the first head of
#    every group and the last head (a complete head of this size costs the
#    float64 oracle several seconds).
# ----------------------------------------------------------------------------
def _full_size_heads(w):
    if w.name in ("causal_b4h16_n1024_d64", "cross_b8h16_n512_m2048_d64"):
        return all_heads(w)
    if w.name == "causal_b1h32_n16384_d128":
        return [(0, h) for h in range(0, w.H, 2)] + [(0, w.H - 1)]
    return scheduler_heads(w)


FULL = ["causal_b4h16_n1024_d64", "causal_b2h32_n4096_d128",
        "cross_b8h16_n512_m2048_d64", "causal_b1h32_n16384_d128"]


@pytest.mark.parametrize("name", FULL)
def test_full_size(name):
    """Both dQ designs, against one oracle evaluation per head."""
    w = synth.workload(name)
    res = heads_compare(w, _full_size_heads(w), dq_paths=tuple(DQ_PATHS))
    for p, label in zip(DQ_PATHS, DQ_IDS):
        errs, inv = res[p]
        _assert_within(errs, TOL["bf16"], f"{name} {label}")
        _assert_within(inv, TOL["bf16"], f"{name} {label} invariants")


def test_timeout_path_reports_error():
    """A bounded wait that nothing completes must come back as an error
    status, with the context still usable afterwards."""
    assert lib.attn_get_device_error() == 0
    lib.attn_probe_timeout(2000)
    assert lib.attn_get_device_error() == lib.ATTN_ERR_DEVICE_TIMEOUT
    assert lib.attn_get_device_error() == 0
    w = synth.make_small(1, 1, 128, 128, 64, 64, "bf16", False, seed=5)
    _assert_within(full_compare(w), TOL["bf16"], "after timeout")
