"""Python binding of the B200 attention library (``libattn.so``).

Argument marshalling only: each function checks that it was given contiguous
CUDA tensors of one element type, allocates outputs with torch when the caller
did not pass them, and calls the C entry point of the same name on torch's
current stream. Every arithmetic step runs in the library's CUDA kernels;
there is no fallback, and importing this package fails loudly when the
library has not been built, or is older than the header it must export
(``python scaled_dot_product_saving_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "AttnError", "LIB_PATH", "lib", "ATTN_F32", "ATTN_BF16",
    "ATTN_PATH_AUTO", "ATTN_PATH_SIMT", "ATTN_PATH_TENSOR",
    "ATTN_DQ_AUTO", "ATTN_DQ_REDUCE", "ATTN_DQ_SEPARATE", "attn_set_dq_path",
    "attn_fwd", "attn_bwd", "attn_bwd_workspace_size", "attn_get_device_error",
    "attn_probe_timeout", "attn_set_path", "attn_last_launch_count", "attn_status_string",
    "dtype_code", "attn_trace_begin", "attn_trace_end", "KERNEL_NAMES",
    "attn_bwd_noalloc", "attn_bwd_noalloc_scratch_bytes",
    "attn_proj_bwd", "attn_proj_bwd_workspace_size",
    "attn_outproj_bwd", "attn_outproj_bwd_workspace_size",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libattn.so")

ATTN_F32, ATTN_BF16 = 0, 1
ATTN_PATH_AUTO, ATTN_PATH_SIMT, ATTN_PATH_TENSOR = 0, 1, 2
ATTN_DQ_AUTO, ATTN_DQ_REDUCE, ATTN_DQ_SEPARATE = 0, 1, 2
ATTN_OK = 0
ATTN_ERR_DEVICE_TIMEOUT = 8

KERNEL_NAMES = {1: "fwd_tensor", 2: "fwd_simt", 3: "preprocess", 4: "bwd_tensor",
                5: "bwd_simt", 6: "finalize", 7: "proj_gather", 8: "gemm",
                9: "fwd_f32x", 10: "bwd_f32x", 11: "bwd_kv", 12: "bwd_dq"}


class _KernelTime(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int), ("ms", ctypes.c_float)]


class AttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {attn_status_string(code)} (status {code})")


_BUILD_HINT = "build it with `python scaled_dot_product_saving_b200/build.py` (nvcc, sm_100a)"


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: {_BUILD_HINT}")
    L = ctypes.CDLL(LIB_PATH)
    try:
        return _declare(L)
    except AttributeError as e:
        raise ImportError(f"{LIB_PATH} is stale ({e}): {_BUILD_HINT}") from None


def _declare(L: ctypes.CDLL) -> ctypes.CDLL:
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, vp]
    L.attn_fwd.restype = i
    L.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                           i, i, i, i, i, i, i, i, f, vp]
    L.attn_bwd.restype = i
    L.attn_fwd_masked.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, vp]
    L.attn_fwd_masked.restype = i
    L.attn_bwd_masked.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                  i, i, i, i, i, i, i, i, f, vp]
    L.attn_bwd_masked.restype = i
    L.attn_bwd_workspace_size.argtypes = [i, i, i, i, i, i, i]
    L.attn_bwd_workspace_size.restype = sz
    L.attn_get_device_error.argtypes = [vp]
    L.attn_get_device_error.restype = i
    L.attn_probe_timeout.argtypes = [ctypes.c_uint, vp]
    L.attn_probe_timeout.restype = i
    L.attn_set_path.argtypes = [i]
    L.attn_set_path.restype = i
    L.attn_set_dq_path.argtypes = [i]
    L.attn_set_dq_path.restype = i
    L.attn_last_launch_count.argtypes = []
    L.attn_last_launch_count.restype = i
    L.attn_status_string.argtypes = [i]
    L.attn_status_string.restype = ctypes.c_char_p
    L.attn_trace_begin.argtypes = [i]
    L.attn_trace_begin.restype = i
    L.attn_trace_end.argtypes = [ctypes.POINTER(_KernelTime), i]
    L.attn_trace_end.restype = i
    L.attn_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                   i, i, i, i, i, i, i, i, f, vp]
    L.attn_bwd_noalloc.restype = i
    L.attn_bwd_noalloc_scratch_bytes.argtypes = []
    L.attn_bwd_noalloc_scratch_bytes.restype = sz
    L.attn_proj_bwd_workspace_size.argtypes = [i, i, i, i, i, i, i]
    L.attn_proj_bwd_workspace_size.restype = sz
    L.attn_proj_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                i, i, i, i, i, i, i, vp]
    L.attn_proj_bwd.restype = i
    L.attn_outproj_bwd_workspace_size.argtypes = [i, i, i, i, i, i]
    L.attn_outproj_bwd_workspace_size.restype = sz
    L.attn_outproj_bwd.argtypes = [vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, i, vp]
    L.attn_outproj_bwd.restype = i
    return L


lib = _load()


def attn_status_string(code: int) -> str:
    return lib.attn_status_string(int(code)).decode()


def _check(code: int, where: str) -> None:
    if code != ATTN_OK:
        raise AttnError(code, where)


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return ATTN_F32
    if dt == torch.bfloat16:
        return ATTN_BF16
    raise TypeError(f"unsupported dtype {dt}; use torch.float32 or torch.bfloat16")


def _stream_handle(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _dims(q, k, v):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("Q, K, V must be [B, H, N, d] tensors")
    B, H, n, d = q.shape
    if k.shape[:2] != (B, H) or v.shape[:2] != (B, H) or k.shape[3] != d or v.shape[2] != k.shape[2]:
        raise ValueError(f"shape mismatch Q{tuple(q.shape)} K{tuple(k.shape)} V{tuple(v.shape)}")
    return B, H, n, k.shape[2], d, v.shape[3]


def _require(*ts):
    dt = ts[0].dtype
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        if t.dtype != dt:
            raise TypeError("Q, K, V, O, dO must share one dtype")


def attn_bwd_workspace_size(B, H, n, m, d, dv, dtype) -> int:
    code = dtype if isinstance(dtype, int) else dtype_code(dtype)
    return int(lib.attn_bwd_workspace_size(B, H, n, m, d, dv, code))


def _key_len(key_len, B, device):
    """The padding mask argument: None, or an int32 [B] tensor on the device."""
    if key_len is None:
        return None
    if (not isinstance(key_len, torch.Tensor) or key_len.dtype != torch.int32 or
            key_len.shape != (B,) or key_len.device != device or not key_len.is_contiguous()):
        raise ValueError("key_len must be a contiguous int32 [B] tensor on the inputs' device")
    return key_len


def attn_fwd(q, k, v, causal=False, scale=None, out=None, lse=None, stream=None, key_len=None):
    """Returns (O, LSE) for [B,H,N,d] CUDA tensors. key_len (optional int32
    [B] device tensor): valid keys per batch element; later keys are padding,
    masked before the softmax (attn_fwd_masked)."""
    _require(q, k, v)
    B, H, n, m, d, dv = _dims(q, k, v)
    key_len = _key_len(key_len, B, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, H, n, dv), dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, n), dtype=torch.float32, device=q.device)
    if key_len is None:
        _check(lib.attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, n, m, d, dv,
                            dtype_code(q.dtype), int(bool(causal)), scale,
                            _stream_handle(stream)), "attn_fwd")
    else:
        _check(lib.attn_fwd_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                   _ptr(key_len), B, H, n, m, d, dv, dtype_code(q.dtype),
                                   int(bool(causal)), scale, _stream_handle(stream)),
               "attn_fwd_masked")
    return out, lse


def attn_bwd(q, k, v, o, do, lse, causal=False, scale=None, workspace=None,
             dq=None, dk=None, dv=None, stream=None, key_len=None):
    """Returns (dQ, dK, dV) with the shapes of Q, K, V. key_len: the padding
    mask given to attn_fwd (attn_bwd_masked)."""
    _require(q, k, v, o, do)
    B, H, n, m, d, dvw = _dims(q, k, v)
    key_len = _key_len(key_len, B, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    code = dtype_code(q.dtype)
    need = attn_bwd_workspace_size(B, H, n, m, d, dvw, code)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if dq is None:
        dq = torch.empty_like(q)
    if dk is None:
        dk = torch.empty_like(k)
    if dv is None:
        dv = torch.empty_like(v)
    if key_len is None:
        _check(lib.attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                            _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                            workspace.numel() * workspace.element_size(),
                            B, H, n, m, d, dvw, code, int(bool(causal)), scale,
                            _stream_handle(stream)), "attn_bwd")
    else:
        _check(lib.attn_bwd_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                                   _ptr(key_len), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(),
                                   B, H, n, m, d, dvw, code, int(bool(causal)), scale,
                                   _stream_handle(stream)), "attn_bwd_masked")
    return dq, dk, dv


def attn_get_device_error(stream=None) -> int:
    """Synchronises the stream; returns the device status code and clears it."""
    return int(lib.attn_get_device_error(_stream_handle(stream)))


def attn_probe_timeout(timeout_us: int, stream=None) -> None:
    _check(lib.attn_probe_timeout(int(timeout_us), _stream_handle(stream)), "attn_probe_timeout")


def attn_set_path(path: int) -> None:
    _check(lib.attn_set_path(int(path)), "attn_set_path")


def attn_set_dq_path(path: int) -> None:
    _check(lib.attn_set_dq_path(int(path)), "attn_set_dq_path")


def attn_last_launch_count() -> int:
    return int(lib.attn_last_launch_count())


def attn_trace_begin(capacity: int = 4096) -> None:
    """Start bracketing every launch of this thread with CUDA events."""
    _check(lib.attn_trace_begin(int(capacity)), "attn_trace_begin")


def attn_trace_end(max_entries: int = 65536):
    """Stop tracing; returns [(kernel name, milliseconds), ...] in launch order."""
    buf = (_KernelTime * max_entries)()
    count = lib.attn_trace_end(buf, max_entries)
    if count < 0:
        raise AttnError(7, "attn_trace_end")
    return [(KERNEL_NAMES.get(buf[k].kernel, str(buf[k].kernel)), float(buf[k].ms))
            for k in range(min(count, max_entries))]


def attn_bwd_noalloc_scratch_bytes() -> int:
    return int(lib.attn_bwd_noalloc_scratch_bytes())


def attn_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, causal=False, scale=None, stream=None):
    """attn_bwd without a workspace: the library's own fixed scratch array is
    used, for callers that may not allocate device memory. The caller still
    passes every input and output tensor; nothing is allocated here."""
    _require(q, k, v, o, do, dq, dk, dv)
    B, H, n, m, d, dvw = _dims(q, k, v)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    _check(lib.attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse),
                                _ptr(dq), _ptr(dk), _ptr(dv), B, H, n, m, d, dvw,
                                dtype_code(q.dtype), int(bool(causal)), scale,
                                _stream_handle(stream)),
           "attn_bwd_noalloc")
    return dq, dk, dv


def attn_proj_bwd_workspace_size(B: int, n: int, d_model: int, H: int, d: int, dv: int,
                                 dtype_code_: int) -> int:
    return int(lib.attn_proj_bwd_workspace_size(B, n, d_model, H, d, dv, dtype_code_))


def attn_proj_bwd(x, wq, wk, wv, dq, dk, dv, workspace=None, dx=None, dwq=None, dwk=None,
                  dwv=None, stream=None):
    """Returns (dX, dWq, dWk, dWv) for X [B,n,d_model], Wq/Wk [d_model,H*d],
    Wv [d_model,H*dv] and dQ/dK [B,H,n,d], dV [B,H,n,dv] (head h = column
    block h of each projection)."""
    _require(x, wq, wk, wv, dq, dk, dv)
    B, n, d_model = x.shape
    _, H, n2, d = dq.shape
    dvw = dv.shape[-1]
    if (n2 != n or tuple(dk.shape) != (B, H, n, d) or tuple(dv.shape) != (B, H, n, dvw)
            or tuple(wq.shape) != (d_model, H * d) or tuple(wk.shape) != (d_model, H * d)
            or tuple(wv.shape) != (d_model, H * dvw)):
        raise ValueError("attn_proj_bwd: inconsistent shapes")
    code = dtype_code(x.dtype)
    need = attn_proj_bwd_workspace_size(B, n, d_model, H, d, dvw, code)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    dx = torch.empty_like(x) if dx is None else dx
    dwq = torch.empty_like(wq) if dwq is None else dwq
    dwk = torch.empty_like(wk) if dwk is None else dwk
    dwv = torch.empty_like(wv) if dwv is None else dwv
    _check(lib.attn_proj_bwd(_ptr(x), _ptr(wq), _ptr(wk), _ptr(wv), _ptr(dq), _ptr(dk), _ptr(dv),
                             _ptr(dx), _ptr(dwq), _ptr(dwk), _ptr(dwv), _ptr(workspace),
                             workspace.numel() * workspace.element_size(),
                             B, n, d_model, H, d, dvw, code, _stream_handle(stream)),
           "attn_proj_bwd")
    return dx, dwq, dwk, dwv


def attn_outproj_bwd_workspace_size(B: int, n: int, d_model: int, H: int, dv: int,
                                    dtype_code_: int) -> int:
    return int(lib.attn_outproj_bwd_workspace_size(B, n, d_model, H, dv, dtype_code_))


def attn_outproj_bwd(o, wo, g, workspace=None, do=None, dwo=None, stream=None):
    """Returns (dO, dWo) for Y = [O_1 ... O_H] Wo: O [B,H,n,dv], Wo [H*dv,d_model],
    G = dL/dY [B,n,d_model]."""
    _require(o, wo, g)
    B, H, n, dvw = o.shape
    d_model = g.shape[-1]
    if tuple(g.shape) != (B, n, d_model) or tuple(wo.shape) != (H * dvw, d_model):
        raise ValueError("attn_outproj_bwd: inconsistent shapes")
    code = dtype_code(o.dtype)
    need = attn_outproj_bwd_workspace_size(B, n, d_model, H, dvw, code)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=o.device)
    do = torch.empty_like(o) if do is None else do
    dwo = torch.empty_like(wo) if dwo is None else dwo
    _check(lib.attn_outproj_bwd(_ptr(o), _ptr(wo), _ptr(g), _ptr(do), _ptr(dwo), _ptr(workspace),
                                workspace.numel() * workspace.element_size(),
                                B, n, d_model, H, dvw, code, _stream_handle(stream)),
           "attn_outproj_bwd")
    return do, dwo
