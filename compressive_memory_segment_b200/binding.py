"""Python binding of libinfini_attn.so (the C ABI in include/infini_attn.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. torch supplies device memory and streams. There is no fallback: if the
compiled library is missing this module raises ImportError at import time.

The functions keep the C names. ``forward`` is a convenience wrapper that
allocates the outputs with torch and calls ``infini_attn_forward_ws``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libinfini_attn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libinfini_attn.so is not built (%s); run `python -m compressive_memory_segment_b200.build` "
        "or __graft_entry__.build()" % LIB_PATH)

_lib = ctypes.CDLL(LIB_PATH)

INFINI_F32, INFINI_BF16 = 0, 1
INFINI_OK = 0
INFINI_ERR_NULL, INFINI_ERR_SHAPE, INFINI_ERR_UNSUPPORTED, INFINI_ERR_ALIGN = -1, -2, -3, -4
INFINI_ERR_CUDA, INFINI_ERR_TIMEOUT, INFINI_ERR_WORKSPACE, INFINI_ERR_ALIAS, INFINI_ERR_SIZE = -5, -6, -7, -8, -9
INFINI_ERR_SCRATCH = -10
INFINI_ERR_BOUNDS = -11
INFINI_NOALLOC_SCRATCH_BYTES = 64 << 20
INFINI_PATH_AUTO, INFINI_PATH_SIMT, INFINI_PATH_TC, INFINI_PATH_TC_PAIRED = 0, 1, 2, 3

EXPORTED = ("infini_attn_forward", "infini_attn_workspace_size", "infini_attn_forward_ws",
            "infini_attn_forward_traced", "infini_attn_forward_noalloc",
            "infini_attn_select_path", "infini_attn_launch_count", "infini_attn_device_status",
            "infini_attn_selftest_timeout", "infini_attn_decode_step", "infini_attn_decode_workspace_size",
            "infini_attn_state_ws", "infini_attn_finish_ws", "infini_attn_exscan_parts",
            "infini_attn_backward", "infini_attn_backward_path", "infini_attn_backward_workspace_size",
            "infini_attn_schedule_check",
            "infini_attn_strerror", "infini_attn_version")


class infini_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("H", ctypes.c_int64), ("L", ctypes.c_int64),
                ("d", ctypes.c_int64), ("dtype", ctypes.c_int32)]


_vp, _i64, _sz, _int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
_shp = ctypes.POINTER(infini_shape)

def _declare(lib):
    """Sets the argument and result types of every entry point on `lib`."""
    lib.infini_attn_forward.argtypes = [_shp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp]
    lib.infini_attn_forward.restype = _int
    lib.infini_attn_forward_ws.argtypes = [_shp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp,
                                            _vp, _sz, _int, _vp]
    lib.infini_attn_forward_ws.restype = _int
    lib.infini_attn_forward_traced.argtypes = [_shp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp,
                                                _vp, _sz, _int, _vp, _int, _vp]
    lib.infini_attn_forward_traced.restype = _int
    lib.infini_attn_forward_noalloc.argtypes = [_shp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp]
    lib.infini_attn_forward_noalloc.restype = _int
    lib.infini_attn_workspace_size.argtypes = [_shp, _i64]
    lib.infini_attn_workspace_size.restype = _sz
    lib.infini_attn_select_path.argtypes = [_shp, _i64]
    lib.infini_attn_select_path.restype = _int
    lib.infini_attn_launch_count.argtypes = [_shp, _i64, _int]
    lib.infini_attn_launch_count.restype = _int
    lib.infini_attn_device_status.argtypes = [_vp]
    lib.infini_attn_device_status.restype = _int
    lib.infini_attn_decode_step.argtypes = [_shp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _sz, _vp]
    lib.infini_attn_decode_step.restype = _int
    lib.infini_attn_decode_workspace_size.argtypes = [_shp]
    lib.infini_attn_decode_workspace_size.restype = _sz
    lib.infini_attn_state_ws.argtypes = [_shp, _vp, _vp, _i64, _vp, _vp, _vp, _sz, _int, _vp]
    lib.infini_attn_state_ws.restype = _int
    lib.infini_attn_finish_ws.argtypes = [_shp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _sz, _int, _vp]
    lib.infini_attn_finish_ws.restype = _int
    lib.infini_attn_exscan_parts.argtypes = [_i64, _i64, _int, _int, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
    lib.infini_attn_exscan_parts.restype = _int
    lib.infini_attn_backward_workspace_size.argtypes = [_shp, _i64]
    lib.infini_attn_backward_workspace_size.restype = _sz
    lib.infini_attn_backward.argtypes = [_shp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                          _vp, _vp, _vp, _sz, _vp]
    lib.infini_attn_backward.restype = _int
    lib.infini_attn_backward_path.argtypes = [_shp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp,
                                               _vp, _vp, _vp, _vp, _sz, _int, _vp]
    lib.infini_attn_backward_path.restype = _int
    lib.infini_attn_selftest_timeout.argtypes = [ctypes.c_uint64, _vp]
    lib.infini_attn_selftest_timeout.restype = _int
    lib.infini_attn_schedule_check.argtypes = [_i64, _int, _int, ctypes.POINTER(ctypes.c_double)]
    lib.infini_attn_schedule_check.restype = _int
    lib.infini_attn_strerror.argtypes = [_int]
    lib.infini_attn_strerror.restype = ctypes.c_char_p
    lib.infini_attn_version.argtypes = []
    lib.infini_attn_version.restype = _int
    return lib


_lib = _declare(_lib)


def open_library(path: str):
    """Another build of the same C ABI (the tracing or the debug build of
    compressive_memory_segment_b200.build), with its entry points declared;
    call them with plain pointers, like the functions below."""
    return _declare(ctypes.CDLL(path))


def _ptr(x) -> Optional[int]:
    """A tensor's data pointer, an int, or None (NULL)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_shape(B: int, H: int, L: int, d: int, dtype: int) -> infini_shape:
    return infini_shape(B, H, L, d, dtype)


def infini_attn_strerror(code: int) -> str:
    return _lib.infini_attn_strerror(code).decode()


def infini_attn_version() -> int:
    return _lib.infini_attn_version()


def infini_attn_workspace_size(shape: infini_shape, seg_len: int) -> int:
    return _lib.infini_attn_workspace_size(ctypes.byref(shape), seg_len)


def infini_attn_select_path(shape: infini_shape, seg_len: int) -> int:
    return _lib.infini_attn_select_path(ctypes.byref(shape), seg_len)


def infini_attn_launch_count(shape: infini_shape, seg_len: int, path: int = INFINI_PATH_AUTO) -> int:
    return _lib.infini_attn_launch_count(ctypes.byref(shape), seg_len, path)


def infini_attn_device_status(stream=None) -> int:
    return _lib.infini_attn_device_status(_stream(stream))


def infini_attn_schedule_check(n_seg: int, n_qt: int, grid: int):
    """(return code, busiest CTA's key tiles over the mean) of the attention
    kernel's unit schedule, run on the host."""
    ratio = ctypes.c_double(0.0)
    rc = _lib.infini_attn_schedule_check(int(n_seg), int(n_qt), int(grid), ctypes.byref(ratio))
    return rc, ratio.value


def infini_attn_selftest_timeout(limit_ns: int, stream=None) -> int:
    return _lib.infini_attn_selftest_timeout(int(limit_ns), _stream(stream))


def infini_attn_forward(shape, q, k, v, beta, M_in, z_in, seg_len, out, M_out, z_out, stream=None) -> int:
    return _lib.infini_attn_forward(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                                    _ptr(M_in), _ptr(z_in), seg_len, _ptr(out), _ptr(M_out),
                                    _ptr(z_out), _stream(stream))


def infini_attn_forward_ws(shape, q, k, v, beta, M_in, z_in, seg_len, out, M_out, z_out,
                           workspace, workspace_bytes, path=INFINI_PATH_AUTO, stream=None) -> int:
    return _lib.infini_attn_forward_ws(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                                       _ptr(M_in), _ptr(z_in), seg_len, _ptr(out), _ptr(M_out),
                                       _ptr(z_out), _ptr(workspace), workspace_bytes, path,
                                       _stream(stream))


def infini_attn_forward_traced(shape, q, k, v, beta, M_in, z_in, seg_len, out, M_out, z_out,
                               workspace, workspace_bytes, path, events, stream=None) -> int:
    """events: a sequence of torch.cuda.Event (already recorded once, so the
    handle exists) or raw cudaEvent_t ints, launch_count + 1 of them."""
    n = len(events)
    arr = (ctypes.c_void_p * n)(*[e if isinstance(e, int) else e.cuda_event for e in events])
    return _lib.infini_attn_forward_traced(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                                           _ptr(M_in), _ptr(z_in), seg_len, _ptr(out), _ptr(M_out),
                                           _ptr(z_out), _ptr(workspace), workspace_bytes, path,
                                           arr, n, _stream(stream))


def infini_attn_forward_noalloc(shape, q, k, v, beta, M_in, z_in, seg_len, out, M_out, z_out,
                                stream=None) -> int:
    """The allocation-free entry point: scratch comes from the library's
    built-in buffer (see the header for the size limit and the rules on
    overlapping calls)."""
    return _lib.infini_attn_forward_noalloc(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                                            _ptr(M_in), _ptr(z_in), seg_len, _ptr(out), _ptr(M_out),
                                            _ptr(z_out), _stream(stream))


def infini_attn_decode_workspace_size(shape) -> int:
    return _lib.infini_attn_decode_workspace_size(ctypes.byref(shape))


def infini_attn_decode_step(shape, q, k, v, beta, k_cache, v_cache, pos, M, z, out, workspace, ws_bytes,
                            stream=None) -> int:
    return _lib.infini_attn_decode_step(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                                        _ptr(k_cache), _ptr(v_cache), int(pos), _ptr(M), _ptr(z), _ptr(out),
                                        _ptr(workspace), ws_bytes, _stream(stream))


def infini_attn_state_ws(shape, k, v, seg_len, M_tot, z_tot, workspace, workspace_bytes,
                         path=INFINI_PATH_AUTO, stream=None) -> int:
    return _lib.infini_attn_state_ws(ctypes.byref(shape), _ptr(k), _ptr(v), seg_len, _ptr(M_tot), _ptr(z_tot),
                                     _ptr(workspace), workspace_bytes, path, _stream(stream))


def infini_attn_finish_ws(shape, q, k, v, beta, M_in, z_in, seg_len, out, M_out, z_out, workspace,
                          workspace_bytes, path=INFINI_PATH_AUTO, stream=None) -> int:
    return _lib.infini_attn_finish_ws(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(M_in),
                                      _ptr(z_in), seg_len, _ptr(out), _ptr(M_out), _ptr(z_out), _ptr(workspace),
                                      workspace_bytes, path, _stream(stream))


def infini_attn_exscan_parts(n_M, n_z, n_parts, part, totals_M, totals_z, M_in, z_in, off_M, off_z,
                             stream=None) -> int:
    return _lib.infini_attn_exscan_parts(n_M, n_z, n_parts, part, _ptr(totals_M), _ptr(totals_z), _ptr(M_in),
                                         _ptr(z_in), _ptr(off_M), _ptr(off_z), _stream(stream))


def infini_attn_backward_workspace_size(shape, seg_len) -> int:
    return _lib.infini_attn_backward_workspace_size(ctypes.byref(shape), seg_len)


def infini_attn_backward(shape, q, k, v, beta, M_in, z_in, seg_len, dout, dM_out, dz_out, dq, dk, dv, dbeta,
                         dM_in, dz_in, workspace, workspace_bytes, stream=None) -> int:
    return _lib.infini_attn_backward(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(M_in),
                                     _ptr(z_in), seg_len, _ptr(dout), _ptr(dM_out), _ptr(dz_out), _ptr(dq),
                                     _ptr(dk), _ptr(dv), _ptr(dbeta), _ptr(dM_in), _ptr(dz_in), _ptr(workspace),
                                     workspace_bytes, _stream(stream))


def infini_attn_backward_path(shape, q, k, v, beta, M_in, z_in, seg_len, dout, dM_out, dz_out, dq, dk, dv, dbeta,
                              dM_in, dz_in, workspace, workspace_bytes, path, stream=None) -> int:
    return _lib.infini_attn_backward_path(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(M_in),
                                          _ptr(z_in), seg_len, _ptr(dout), _ptr(dM_out), _ptr(dz_out), _ptr(dq),
                                          _ptr(dk), _ptr(dv), _ptr(dbeta), _ptr(dM_in), _ptr(dz_in),
                                          _ptr(workspace), workspace_bytes, path, _stream(stream))


class InfiniError(RuntimeError):
    def __init__(self, code: int):
        super().__init__("infini_attn error %d: %s" % (code, infini_attn_strerror(code)))
        self.code = code


def check(code: int) -> None:
    if code != INFINI_OK:
        raise InfiniError(code)


def shape_of(q) -> infini_shape:
    import torch
    if q.dim() != 4:
        raise ValueError("q must be [B, H, L, d]")
    dt = {torch.float32: INFINI_F32, torch.bfloat16: INFINI_BF16}.get(q.dtype)
    if dt is None:
        raise TypeError("q, k, v must be float32 or bfloat16")
    B, H, L, d = q.shape
    return infini_shape(B, H, L, d, dt)


def workspace_for(q, seg_len: int):
    """Allocate (torch, on q's device) a workspace for this shape."""
    import torch
    n = infini_attn_workspace_size(shape_of(q), seg_len)
    if n == 0:
        raise InfiniError(INFINI_ERR_SHAPE)
    return torch.empty(n, dtype=torch.uint8, device=q.device)


def forward(q, k, v, beta, seg_len: int, M_in=None, z_in=None, out=None, M_out=None, z_out=None,
            workspace=None, path: int = INFINI_PATH_AUTO, stream=None):
    """Run the layer on device tensors q, k, v [B, H, L, d] (fp32 or bf16),
    beta [H] fp32, optional incoming state M_in [B, H, d, d], z_in [B, H, d]
    fp32. Returns (out, M_out, z_out); outputs are allocated when not given."""
    import torch
    shp = shape_of(q)
    B, H, L, d = q.shape
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous")
    if out is None:
        out = torch.empty_like(q)
    if M_out is None:
        M_out = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device)
    if z_out is None:
        z_out = torch.empty((B, H, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = workspace_for(q, seg_len)
    check(infini_attn_forward_ws(shp, q, k, v, beta, M_in, z_in, seg_len, out, M_out, z_out,
                                 workspace, workspace.numel() * workspace.element_size(), path, stream))
    return out, M_out, z_out


def decode_step(q, k, v, beta, k_cache, v_cache, pos: int, M, z, out=None, workspace=None, stream=None):
    """One decode step on device tensors: q, k, v [B, H, d] (this token),
    k_cache, v_cache [B, H, N, d] (rows 0..pos-1 filled; row pos is written),
    M [B, H, d, d] and z [B, H, d] fp32 (updated in place when pos == N - 1).
    Returns out [B, H, d]."""
    import torch
    B, H, N, d = k_cache.shape
    dt = {torch.float32: INFINI_F32, torch.bfloat16: INFINI_BF16}.get(q.dtype)
    if dt is None:
        raise TypeError("q, k, v must be float32 or bfloat16")
    shp = infini_shape(B, H, N, d, dt)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = torch.empty(infini_attn_decode_workspace_size(shp), dtype=torch.uint8, device=q.device)
    nbytes = workspace.numel() * workspace.element_size()
    check(infini_attn_decode_step(shp, q, k, v, beta, k_cache, v_cache, pos, M, z, out, workspace, nbytes, stream))
    return out


def backward(q, k, v, beta, seg_len: int, dout, M_in=None, z_in=None, dM_out=None, dz_out=None, workspace=None,
             stream=None, path: int = 0):
    """Gradients of the forward on device tensors. Returns (dq, dk, dv, dbeta,
    dM_in, dz_in), all fp32; dq, dk, dv have q's shape. path: INFINI_PATH_AUTO
    (0), _SIMT or _TC."""
    import torch
    shp = shape_of(q)
    B, H, L, d = q.shape
    f32 = dict(dtype=torch.float32, device=q.device)
    dq, dk, dv = (torch.empty((B, H, L, d), **f32) for _ in range(3))
    dbeta = torch.empty((H,), **f32)
    dM_in = torch.empty((B, H, d, d), **f32)
    dz_in = torch.empty((B, H, d), **f32)
    if workspace is None:
        workspace = torch.empty(infini_attn_backward_workspace_size(shp, seg_len), dtype=torch.uint8,
                                device=q.device)
    check(infini_attn_backward_path(shp, q, k, v, beta, M_in, z_in, seg_len, dout, dM_out, dz_out, dq, dk, dv, dbeta,
                                    dM_in, dz_in, workspace, workspace.numel() * workspace.element_size(), path,
                                    stream))
    return dq, dk, dv, dbeta, dM_in, dz_in
