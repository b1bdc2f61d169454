"""GPU parity of the key padding mask (attn_fwd_masked / attn_bwd_masked,
"Is there any Reference About Backpropagation of the Transformer's Multi-Head
Layer?", section 4: padding masks go before the softmax) against the float64
oracle, on every kernel path. Tolerance as for the unmasked calls:
max|gpu - ref| / max|ref| per output tensor, 2e-2 bf16, 1e-5 fp32."""
import pytest
import torch

import synth
from parity_util import TOL, all_heads, full_compare, gpu_run, heads_compare

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


CASES = [
    # B, H, n, m, d, dv, dtype, causal, lengths
    (3, 2, 300, 300, 64, 64, "bf16", False, (300, 129, 1)),     # full, ragged, a single key
    (2, 2, 384, 384, 128, 128, "bf16", True, (200, 384)),       # causal and padding combined
    (2, 1, 200, 520, 64, 64, "bf16", False, (257, 128)),        # n != m, tile-aligned length
    (2, 2, 256, 700, 128, 128, "bf16", False, (640, 5)),        # whole key tiles of padding
    (2, 2, 300, 300, 64, 64, "f32", True, (150, 300)),          # fp32 tensor-core path
    (2, 1, 200, 333, 40, 24, "f32", False, (64, 333)),
    (2, 1, 100, 100, 40, 40, "bf16", True, (37, 100)),          # CUDA-core path widths
    (2, 1, 129, 65, 128, 96, "f32", False, (1, 64)),            # fp32 on the CUDA-core path
]


@pytest.mark.parametrize("dq_path", [lib.ATTN_DQ_REDUCE, lib.ATTN_DQ_SEPARATE],
                         ids=["dq_reduce", "dq_separate"])
@pytest.mark.parametrize("B,H,n,m,d,dv,dt,causal,lengths", CASES)
def test_padding_mask(B, H, n, m, d, dv, dt, causal, lengths, dq_path):
    if dq_path == lib.ATTN_DQ_SEPARATE and not (dt == "bf16" and d == dv and d in (64, 128)):
        pytest.skip("the dQ design applies to the bf16 tensor-core path only")
    w = synth.make_small(B, H, n, m, d, dv, dt, causal, seed=B * 7 + n + m + d, lengths=lengths)
    _assert_within(full_compare(w, dq_path=dq_path), TOL[dt], w.name)


def test_padded_rows_of_dk_dv_are_zero():
    w = synth.make_small(2, 2, 256, 512, 64, 64, "bf16", False, seed=3, lengths=(300, 77))
    _, (o, lse, dq, dk, dv) = gpu_run(w)
    for b, L in enumerate(w.key_len()):
        assert torch.count_nonzero(dk[b, :, L:]) == 0
        assert torch.count_nonzero(dv[b, :, L:]) == 0


def test_lengths_out_of_range_are_clamped():
    """key_len <= 0 means one valid key and key_len > m means m, on the device."""
    w_clamped = synth.make_small(2, 1, 128, 256, 64, 64, "bf16", False, seed=4, lengths=(1, 256))
    inputs = synth.make_inputs(w_clamped)
    _, want = gpu_run(w_clamped, inputs)
    dev = torch.device("cuda:0")
    q, k, v, do = (t.to(dev) for t in inputs)
    kl = torch.tensor([-5, 1000], dtype=torch.int32, device=dev)
    o, lse = lib.attn_fwd(q, k, v, key_len=kl)
    dq, dk, dv = lib.attn_bwd(q, k, v, o, do, lse, key_len=kl)
    torch.cuda.synchronize()
    for name, a, b in zip(("O", "LSE", "dK", "dV"), (o, lse, dk, dv), want[:2] + want[3:]):
        assert torch.equal(a, b), name
    # dQ is summed with reduce-adds in no fixed order
    assert (dq.float() - want[2].float()).abs().max() <= 1e-2 * want[2].float().abs().max()


def test_padded_full_size():
    """The padded workload at full size in the benchmark's launch
    configuration: every head element by element, and invariants."""
    w = synth.workload("padded_b8h16_n1024_d64")
    res = heads_compare(w, all_heads(w), dq_paths=(lib.ATTN_DQ_REDUCE, lib.ATTN_DQ_SEPARATE))
    for p, (errs, inv) in res.items():
        _assert_within(errs, TOL["bf16"], f"{w.name} dq path {p}")
        _assert_within(inv, TOL["bf16"], f"{w.name} dq path {p} invariants")


def test_no_mask_equals_full_length_mask():
    """key_len = m everywhere gives the unmasked call's results bit for bit."""
    w = synth.make_small(2, 2, 256, 256, 128, 128, "bf16", True, seed=8)
    inputs = synth.make_inputs(w)
    _, plain = gpu_run(w, inputs)
    wm = synth.make_small(2, 2, 256, 256, 128, 128, "bf16", True, seed=8, lengths=(256, 256))
    _, masked = gpu_run(wm, inputs)
    for name, a, b in zip(("O", "LSE"), plain[:2], masked[:2]):
        assert torch.equal(a, b), name
    for name, a, b in zip(("dK", "dV"), plain[3:], masked[3:]):
        assert torch.equal(a, b), name
    # dQ is summed with reduce-adds in no fixed order
    assert (plain[2].float() - masked[2].float()).abs().max() <= 1e-2 * masked[2].float().abs().max()
