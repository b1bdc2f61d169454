"""attn_bwd_noalloc against attn_bwd, through the C ABI.

attn_bwd_noalloc exists for callers that may not allocate device memory
(an op inside a framework that owns all device memory and gives it no
scratch buffer): it takes its scratch from a fixed array compiled into the
library. Its results must match the workspace-taking attn_bwd within the
parity tolerance, on two calls in a row (the array keeps the previous call's
contents, so the second call shows that nothing stale leaks in), and sizes
beyond the array must be refused before anything runs.

This file is named so that pytest collects it last.
"""
import ctypes
import math

import pytest
import torch

import synth
from parity_util import TOL, rel_err, to64

pytestmark = pytest.mark.gpu

lib = pytest.importorskip("scaled_dot_product_saving_b200")

ATTN_ERR_WORKSPACE = 6


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc_call(w, q, k, v, o, do, lse):
    dq = torch.full_like(q, float("nan"))
    dk = torch.full_like(k, float("nan"))
    dv = torch.full_like(v, float("nan"))
    code = lib.lib.attn_bwd_noalloc(
        _p(q), _p(k), _p(v), _p(o), _p(do), _p(lse), _p(dq), _p(dk), _p(dv),
        w.B, w.H, w.n, w.m, w.d, w.dv, lib.dtype_code(q.dtype), int(w.causal),
        w.scale, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == 0, lib.attn_status_string(code)
    torch.cuda.synchronize()
    assert lib.attn_get_device_error() == 0
    return dq, dk, dv


CASES = [
    synth.make_small(2, 4, 300, 300, 64, 64, "bf16", True, seed=71),     # tensor cores, d=64
    synth.make_small(1, 3, 257, 400, 128, 128, "bf16", False, seed=72),  # tensor cores, d=128
    synth.make_small(1, 2, 100, 90, 40, 40, "f32", False, seed=73),      # CUDA-core path
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_matches_attn_bwd_on_two_calls(w):
    assert lib.attn_bwd_workspace_size(w.B, w.H, w.n, w.m, w.d, w.dv,
                                       0 if w.dtype == "f32" else 1) \
        <= lib.attn_bwd_noalloc_scratch_bytes()
    dev = torch.device("cuda:0")
    q, k, v, do = (t.to(dev) for t in synth.make_inputs(w))
    o, lse = lib.attn_fwd(q, k, v, causal=w.causal, scale=w.scale)
    want = lib.attn_bwd(q, k, v, o, do, lse, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    tol = TOL[w.dtype]
    for _ in range(2):
        got = _noalloc_call(w, q, k, v, o, do, lse)
        for name, g, r in zip(("dQ", "dK", "dV"), got, want):
            assert not torch.isnan(g).any(), name
            err = rel_err(to64(g), to64(r))
            assert err <= tol, (w.name, name, err)


def test_noalloc_refuses_sizes_beyond_its_array():
    B, H, n, d = 2, 32, 4096, 128          # needs ~130 MiB of scratch
    assert lib.attn_bwd_workspace_size(B, H, n, n, d, d, 1) > lib.attn_bwd_noalloc_scratch_bytes()
    fake = ctypes.c_void_p(1 << 20)        # never dereferenced: refused first
    code = lib.lib.attn_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake,
                                    B, H, n, n, d, d, 1, 1, 1.0 / math.sqrt(d), None)
    assert code == ATTN_ERR_WORKSPACE
