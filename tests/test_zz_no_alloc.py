"""attn_bwd_noalloc through the C ABI: against the float64 oracle and against
attn_bwd.

attn_bwd_noalloc exists for callers that may not allocate device memory (an
op inside a framework that owns all device memory and gives it no scratch
buffer): it takes its scratch from a fixed array compiled into the library.
On two calls in a row (the array keeps the previous call's contents, so the
second call shows that nothing stale leaks in) its results must
 - match the oracle within the parity tolerance (max|err| / max|ref| per
   output: 2e-2 bf16, 1e-5 fp32), and
 - match attn_bwd on the same inputs far more tightly: dK and dV bit for bit
   (each is summed in a fixed order), dQ up to the order in which partial
   sums from different key tiles were added (one rounding step of the output
   type per element, plus fp32 summation noise).
Sizes beyond the array must be refused before anything runs, with the status
attn_bwd gives for the same arguments.

This file is named so that pytest collects it last.
"""
import ctypes
import math

import pytest
import torch

import oracle.ref as ref
import synth
from parity_util import TOL, rel_err, to64

pytestmark = pytest.mark.gpu

lib = pytest.importorskip("scaled_dot_product_saving_b200")

ATTN_ERR_NULL = 1
ATTN_ERR_ALIGN = 5
ATTN_ERR_WORKSPACE = 6


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _outputs(q, k, v):
    return (torch.full_like(q, float("nan")), torch.full_like(k, float("nan")),
            torch.full_like(v, float("nan")))


def _noalloc_raw(w, q, k, v, o, do, lse, stream_handle):
    """The C entry point itself, through ctypes."""
    dq, dk, dv = _outputs(q, k, v)
    code = lib.lib.attn_bwd_noalloc(
        _p(q), _p(k), _p(v), _p(o), _p(do), _p(lse), _p(dq), _p(dk), _p(dv),
        w.B, w.H, w.n, w.m, w.d, w.dv, lib.dtype_code(q.dtype), int(w.causal),
        w.scale, stream_handle)
    assert code == 0, lib.attn_status_string(code)
    return dq, dk, dv


def _noalloc_wrapper(w, q, k, v, o, do, lse):
    """The package's binding of the same entry point."""
    dq, dk, dv = _outputs(q, k, v)
    got = lib.attn_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, causal=w.causal, scale=w.scale)
    assert all(a is b for a, b in zip(got, (dq, dk, dv)))
    return got


def _assert_same_up_to_sum_order(got, want, dtype, name):
    g, r = got.double(), want.double()
    big = r.abs().max().item()
    if dtype == "bf16":
        bound = 2.0 ** -7 * torch.maximum(g.abs(), r.abs()) + 1e-5 * big
    else:
        bound = 2.0 ** -20 * torch.maximum(g.abs(), r.abs()) + 1e-6 * big
    worst = ((g - r).abs() - bound).max().item()
    assert worst <= 0.0, (name, worst)


CASES = [
    # (workload, how the entry point is called)
    (synth.make_small(2, 4, 300, 300, 64, 64, "bf16", True, seed=71), "current stream"),
    (synth.make_small(1, 3, 257, 400, 128, 128, "bf16", False, seed=72), "wrapper"),
    (synth.make_small(1, 2, 200, 200, 64, 64, "f32", True, seed=74), "legacy default stream"),
    (synth.make_small(1, 2, 100, 90, 40, 40, "f32", False, seed=73), "current stream"),
]


def _check_case(w, how, dev):
    assert lib.attn_bwd_workspace_size(w.B, w.H, w.n, w.m, w.d, w.dv,
                                       0 if w.dtype == "f32" else 1) \
        <= lib.attn_bwd_noalloc_scratch_bytes()
    cpu = synth.make_inputs(w)
    q, k, v, do = (t.to(dev) for t in cpu)
    o, lse = lib.attn_fwd(q, k, v, causal=w.causal, scale=w.scale)
    want = lib.attn_bwd(q, k, v, o, do, lse, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize(dev)
    Q, K, V, dO = (t.to(torch.float64).numpy() for t in cpu)
    oracle = ref.attention_backward(Q, K, V, dO, w.causal, w.scale)
    for call in range(2):
        if how == "wrapper":
            got = _noalloc_wrapper(w, q, k, v, o, do, lse)
        elif how == "legacy default stream":
            got = _noalloc_raw(w, q, k, v, o, do, lse, None)
        else:
            got = _noalloc_raw(w, q, k, v, o, do, lse,
                               ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
        torch.cuda.synchronize(dev)
        assert lib.attn_get_device_error() == 0
        for name, g, r, orc in zip(("dQ", "dK", "dV"), got, want, oracle):
            assert not torch.isnan(g).any(), (call, name)
            err = rel_err(to64(g), orc)
            assert err <= TOL[w.dtype], (w.name, call, name, err)
            if name == "dQ":
                _assert_same_up_to_sum_order(g, r, w.dtype, (w.name, call, name))
            else:
                assert torch.equal(g, r), (w.name, call, name)


@pytest.mark.parametrize("w,how", CASES, ids=lambda x: getattr(x, "name", x))
def test_noalloc_matches_oracle_and_attn_bwd_on_two_calls(w, how):
    _check_case(w, how, torch.device("cuda:0"))


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2,
                    reason="needs a second device")
def test_noalloc_on_a_second_device():
    """The array's address is looked up per device: a call with device 1
    current must use device 1's copy."""
    dev = torch.device("cuda:1")
    with torch.cuda.device(dev):
        _check_case(CASES[0][0], "current stream", dev)


def test_noalloc_refuses_sizes_beyond_its_array():
    B, H, n, d = 2, 32, 4096, 128          # needs ~130 MiB of scratch
    assert lib.attn_bwd_workspace_size(B, H, n, n, d, d, 1) > lib.attn_bwd_noalloc_scratch_bytes()
    fake = ctypes.c_void_p(1 << 20)        # never dereferenced: refused first
    args = (B, H, n, n, d, d, 1, 1, 1.0 / math.sqrt(d), None)
    code = lib.lib.attn_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake, *args)
    assert code == ATTN_ERR_WORKSPACE
    # Argument errors take precedence, as they would in attn_bwd.
    code = lib.lib.attn_bwd_noalloc(None, fake, fake, fake, fake, fake, fake, fake, fake, *args)
    assert code == ATTN_ERR_NULL
    odd = ctypes.c_void_p((1 << 20) + 4)
    code = lib.lib.attn_bwd_noalloc(fake, fake, fake, fake, fake, fake, odd, fake, fake, *args)
    assert code == ATTN_ERR_ALIGN
