"""The C ABI on the CPU: the library builds, loads, exports every function the
header declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def L():
    import __graft_entry__
    __graft_entry__.build()
    import scaled_dot_product_saving_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_calls():
    names = declared_functions()
    for required in ("attn_fwd", "attn_bwd", "attn_bwd_workspace_size",
                     "attn_get_device_error", "attn_status_string"):
        assert required in names


def test_library_exports_every_declared_function(L):
    lib = ctypes.CDLL(L.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


# Fake, aligned, non-null device addresses: validation must reject the calls
# below before any of them is used.
P = ctypes.c_void_p(0x10000)
MIS = ctypes.c_void_p(0x10008)
NUL = ctypes.c_void_p(0)


def fwd(L, q=P, k=P, v=P, o=P, lse=P, B=1, H=1, n=64, m=64, d=64, dv=64, dt=1, causal=0,
        scale=0.125):
    return L.lib.attn_fwd(q, k, v, o, lse, B, H, n, m, d, dv, dt, causal, scale, NUL)


def bwd(L, ws=P, wsb=1 << 40, q=P, B=1, H=1, n=64, m=64, d=64, dv=64, dt=1, causal=0,
        scale=0.125, dq=P):
    return L.lib.attn_bwd(q, P, P, P, P, P, dq, P, P, ws, wsb, B, H, n, m, d, dv, dt, causal,
                          scale, NUL)


def test_argument_checks_forward(L):
    assert fwd(L, q=NUL) == 1
    assert fwd(L, lse=NUL) == 1
    assert fwd(L, B=0) == 2
    assert fwd(L, n=0) == 2
    assert fwd(L, n=64, m=65, causal=1) == 2          # causal needs n == m
    assert fwd(L, n=1 << 24, m=1 << 24) == 2
    assert fwd(L, n=64, m=1 << 24) == 2
    assert fwd(L, B=1 << 16, H=1 << 15) == 2          # B*H must stay below 2^31
    assert fwd(L, dt=7) == 3
    assert fwd(L, d=129) == 4
    assert fwd(L, q=MIS) == 5
    assert fwd(L, scale=float("nan")) == 2
    assert fwd(L, scale=float("inf")) == 2


def test_argument_checks_backward(L):
    assert bwd(L, q=NUL) == 1
    assert bwd(L, dq=NUL) == 1
    assert bwd(L, n=63, causal=1) == 2
    assert bwd(L, dt=2) == 3
    assert bwd(L, dv=200) == 4
    assert bwd(L, q=MIS) == 5
    assert bwd(L, ws=NUL) == 6
    need = L.attn_bwd_workspace_size(1, 1, 64, 64, 64, 64, 1)
    assert bwd(L, wsb=need - 1) == 6
    assert bwd(L, ws=MIS, wsb=need) == 5


def test_tensor_path_request_rejects_other_shapes(L):
    try:
        L.attn_set_path(L.ATTN_PATH_TENSOR)
        assert fwd(L, dt=0, d=72, dv=72) == 4     # fp32 on the tensor cores: widths <= 64
        assert fwd(L, dt=0, d=62, dv=62) == 4     # ... and multiples of 4
        assert fwd(L, dt=0, d=64, dv=96) == 4
        assert fwd(L, d=32, dv=32) == 4           # bf16: d == dv in {64, 128}
        assert fwd(L, d=64, dv=128) == 4
        if not torch.cuda.is_available():
            assert fwd(L, dt=0, d=40, dv=24) == 7  # accepted; fails only at the launch
            assert bwd(L, dt=0, d=64, dv=64) == 7
    finally:
        L.attn_set_path(L.ATTN_PATH_AUTO)
    assert L.lib.attn_set_path(9) == 4


def test_path_setting_is_per_thread(L):
    """attn_set_path in one host thread leaves the others' calls alone."""
    import threading
    seen = {}

    def worker():
        L.attn_set_path(L.ATTN_PATH_TENSOR)
        seen["worker"] = fwd(L, d=32, dv=32)        # bf16 width 32: tensor path refuses
    t = threading.Thread(target=worker)
    t.start()
    t.join()
    assert seen["worker"] == 4
    # This thread still has ATTN_PATH_AUTO: width 32 is accepted for the
    # CUDA-core path and gets as far as the launch, which fails with no device.
    if not torch.cuda.is_available():
        assert fwd(L, d=32, dv=32) == 7
    L.attn_set_path(L.ATTN_PATH_TENSOR)
    try:
        assert fwd(L, d=32, dv=32) == 4
    finally:
        L.attn_set_path(L.ATTN_PATH_AUTO)


def test_dq_path_setting(L):
    """attn_set_dq_path takes the three designs and refuses other values."""
    for p in (L.ATTN_DQ_REDUCE, L.ATTN_DQ_SEPARATE, L.ATTN_DQ_AUTO):
        assert L.lib.attn_set_dq_path(p) == 0
    assert L.lib.attn_set_dq_path(7) == 4
    assert L.lib.attn_set_dq_path(-1) == 4
    L.attn_set_dq_path(L.ATTN_DQ_AUTO)


def test_workspace_size_formula(L):
    def expect(B, H, n, d):
        bh = B * H
        n_pad = -(-n // 128) * 128
        rows = -(-(bh * n_pad * 4) // 256) * 256
        counters = 64 + bh                      # counters padded to 256 bytes, then one per head
        return 2 * rows + -(-(bh * n * d * 4) // 256) * 256 + -(-(counters * 4) // 256) * 256
    for (B, H, n, m, d) in [(1, 1, 1, 1, 1), (4, 16, 1024, 1024, 64), (2, 32, 4096, 4096, 128),
                            (8, 16, 512, 2048, 64), (1, 3, 77, 90, 40)]:
        assert L.attn_bwd_workspace_size(B, H, n, m, d, d, 1) == expect(B, H, n, d)
    assert L.attn_bwd_workspace_size(0, 1, 1, 1, 1, 1, 1) == 0
    assert L.attn_bwd_workspace_size(1, 1, 1, 1, 300, 1, 1) == 0


def test_status_strings(L):
    for code in range(9):
        s = L.attn_status_string(code)
        assert s and s != "unknown status"
    assert L.attn_status_string(99) == "unknown status"


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_valid_call_without_a_device_reports_cuda_error(L):
    assert fwd(L) == 7
    assert fwd(L, dt=0) == 7


def proj(L, x=P, dq=P, ws=P, wsb=1 << 40, B=2, n=64, d_model=64, H=2, d=64, dv=64, dt=1):
    return L.lib.attn_proj_bwd(x, P, P, P, dq, P, P, P, P, P, P, ws, wsb, B, n, d_model, H, d,
                               dv, dt, NUL)


def test_argument_checks_projection(L):
    assert proj(L, x=NUL) == 1                     # ATTN_ERR_NULL
    assert proj(L, B=0) == 2                       # ATTN_ERR_SHAPE
    assert proj(L, d=12) == 2                      # widths must be multiples of 8
    assert proj(L, d_model=100) == 2
    assert proj(L, dt=0) == 4                      # fp32: ATTN_ERR_UNSUPPORTED
    assert proj(L, dt=7) == 3                      # ATTN_ERR_DTYPE
    assert proj(L, dq=MIS) == 5                    # ATTN_ERR_ALIGN
    assert proj(L, wsb=16) == 6                    # ATTN_ERR_WORKSPACE
    assert proj(L, ws=NUL) == 6


def test_projection_workspace_formula(L):
    def expect(B, n, d_model, H, d, dv):
        wtot = 2 * H * d + H * dv
        r = lambda x: -(-x // 256) * 256
        return r(B * n * wtot * 2) + r(d_model * wtot * 2)
    for args in [(2, 64, 64, 2, 64, 64), (2, 4096, 4096, 32, 128, 128), (3, 77, 200, 3, 64, 40)]:
        assert L.attn_proj_bwd_workspace_size(*args, 1) == expect(*args)
    assert L.attn_proj_bwd_workspace_size(2, 64, 64, 2, 64, 64, 0) == 0
    assert L.attn_proj_bwd_workspace_size(2, 64, 60, 2, 64, 64, 1) == 0


def outproj(L, o=P, ws=P, wsb=1 << 40, B=2, n=64, d_model=64, H=2, dv=64, dt=1):
    return L.lib.attn_outproj_bwd(o, P, P, P, P, ws, wsb, B, n, d_model, H, dv, dt, NUL)


def test_argument_checks_output_projection(L):
    assert outproj(L, o=NUL) == 1
    assert outproj(L, H=0) == 2
    assert outproj(L, dv=20) == 2
    assert outproj(L, dt=0) == 4
    assert outproj(L, o=MIS) == 5
    assert outproj(L, wsb=16) == 6
    r = lambda x: -(-x // 256) * 256
    assert L.attn_outproj_bwd_workspace_size(2, 64, 64, 2, 64, 1) == 2 * r(2 * 64 * 2 * 64 * 2)
    assert L.attn_outproj_bwd_workspace_size(2, 64, 64, 2, 64, 0) == 0


def test_argument_checks_masked(L):
    """The padding-mask calls check like attn_fwd / attn_bwd, plus key_len's
    4-byte alignment; a NULL key_len is the unmasked call."""
    kl_mis = ctypes.c_void_p(0x10002)
    assert L.lib.attn_fwd_masked(P, P, P, P, P, kl_mis, 1, 1, 64, 64, 64, 64, 1, 0, 0.125, NUL) == 5
    assert L.lib.attn_fwd_masked(NUL, P, P, P, P, P, 1, 1, 64, 64, 64, 64, 1, 0, 0.125, NUL) == 1
    assert L.lib.attn_fwd_masked(P, P, P, P, P, P, 1, 1, 64, 65, 64, 64, 1, 1, 0.125, NUL) == 2
    need = L.attn_bwd_workspace_size(1, 1, 64, 64, 64, 64, 1)
    assert L.lib.attn_bwd_masked(P, P, P, P, P, P, kl_mis, P, P, P, P, need, 1, 1, 64, 64, 64, 64,
                                 1, 0, 0.125, NUL) == 5
    assert L.lib.attn_bwd_masked(P, P, P, P, P, P, P, P, P, P, P, need - 1, 1, 1, 64, 64, 64, 64,
                                 1, 0, 0.125, NUL) == 6
    if not torch.cuda.is_available():
        assert L.lib.attn_fwd_masked(P, P, P, P, P, NUL, 1, 1, 64, 64, 64, 64, 1, 0, 0.125, NUL) == 7


def test_cuda_core_path_head_limit(L):
    """The CUDA-core kernels put B*H in gridDim.y: more than 65535 problems
    on that path are refused before any launch; the tensor-core paths take
    them."""
    assert fwd(L, dt=0, d=128, dv=128, B=65536, H=1) == 4      # fp32, width > 64: CUDA-core
    assert fwd(L, d=40, dv=40, B=256, H=256) == 4             # bf16 odd width: CUDA-core
    need = L.attn_bwd_workspace_size(65536, 1, 64, 64, 128, 128, 0)
    assert bwd(L, dt=0, d=128, dv=128, B=65536, H=1, wsb=need) == 4
    if not torch.cuda.is_available():
        assert fwd(L, B=65536, H=1) == 7                       # bf16 d = 64: tensor cores


def test_kernel_names_match_the_header(L):
    """Every kernel id attn.h declares has a name in the binding's table used
    by the tracer, and no name is left over."""
    text = open(HEADER).read()
    body = text[text.index("typedef enum {", text.index("ATTN_KERNEL_FWD_TENSOR") - 200):]
    body = body[:body.index("attn_kernel_id_t")]
    ids = {int(v) for v in re.findall(r"ATTN_KERNEL_[A-Z0-9_]+\s*=\s*(\d+)", body)}
    assert ids == set(L.KERNEL_NAMES), (ids, sorted(L.KERNEL_NAMES))


def test_import_fails_loudly_without_the_library(tmp_path):
    """No CPU fallback: the binding refuses to import when libattn.so is
    absent, rather than running anything in Python."""
    import shutil
    import subprocess
    import sys
    pkg = tmp_path / "scaled_dot_product_saving_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "scaled_dot_product_saving_b200", "__init__.py"), pkg)
    r = subprocess.run([sys.executable, "-c", "import scaled_dot_product_saving_b200"],
                       cwd=tmp_path, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "libattn.so is missing" in r.stderr
