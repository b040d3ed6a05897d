"""Double-precision CPU oracle for the Infini-attention layer forward.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the product path
(the CUDA library and its Python binding) never does.

The arithmetic lives in ``oracle.cpp`` (plain C++, double accumulation, no
code shared with the CUDA library). This module only compiles it with g++ and
marshals numpy arrays through ctypes. See ``oracle.cpp`` for the definition
and the passages it follows ("Hugging Face Infini-Attention reproduction
analysis", section "Infini-Attention mechanism"; "KV linear-addition
Infini-attention").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

IN_F32, IN_BF16, IN_F64 = 0, 1, 2

_lib = None

_CXXFLAGS = ["-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
             "-fno-fast-math", "-ffp-contract=off"]


def _compile(src: str, lib: str) -> None:
    tmp = lib + ".tmp%d" % os.getpid()
    subprocess.check_call(["g++", *_CXXFLAGS, src, "-o", tmp])
    os.replace(tmp, lib)


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so (beside the source)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        _compile(_SRC, _LIB)
    return _LIB


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _bind(path: str):
    lib = ctypes.CDLL(path)
    i64, vp, dp, ip = ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int
    lib.oracle_infini_forward.argtypes = [i64, i64, i64, i64, i64, vp, vp, vp, ip,
                                          dp, dp, dp, dp, dp, dp, ip]
    lib.oracle_infini_forward.restype = ctypes.c_int
    lib.oracle_infini_forward_segments.argtypes = [i64, i64, i64, i64, i64, vp, vp, vp, ip,
                                                   dp, dp, dp, vp, i64, dp, dp, dp, ip]
    lib.oracle_infini_forward_segments.restype = ctypes.c_int
    lib.oracle_infini_decode_step.argtypes = [i64, i64, i64, i64, i64, vp, vp, vp, vp, vp, ip,
                                              dp, dp, dp, dp]
    lib.oracle_infini_decode_step.restype = ctypes.c_int
    lib.oracle_infini_backward.argtypes = [i64, i64, i64, i64, i64, vp, vp, vp, ip, dp, dp, dp, dp, dp, dp,
                                           dp, dp, dp, dp, dp, dp, ip]
    lib.oracle_infini_backward.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _bind(_LIB)
    return _lib


def compile_variant(src_text: str, workdir: str):
    """Compile an edited copy of the oracle source (used by the tests that
    plant mistakes to show the pins catch them) and return a forward function
    bound to it."""
    src = os.path.join(workdir, "oracle_variant.cpp")
    lib = os.path.join(workdir, "liboracle_variant.so")
    with open(src, "w") as f:
        f.write(src_text)
    _compile(src, lib)
    bound = _bind(lib)
    fwd = lambda *a, **kw: forward(*a, _lib_override=bound, **kw)  # noqa: E731
    fwd.decode = lambda *a, **kw: decode_step(*a, _lib_override=bound, **kw)
    fwd.backward = lambda *a, **kw: backward(*a, _lib_override=bound, **kw)
    return fwd


def _as_input(x: np.ndarray) -> Tuple[np.ndarray, int]:
    """Accept fp32, double or bf16 bit patterns (uint16/int16) without copying
    the data into a wider type."""
    if x.dtype == np.float32:
        return np.ascontiguousarray(x), IN_F32
    if x.dtype == np.float64:
        return np.ascontiguousarray(x), IN_F64
    if x.dtype in (np.uint16, np.int16):
        return np.ascontiguousarray(x.view(np.uint16)), IN_BF16
    raise TypeError("oracle inputs must be float32, float64 or bf16 bits (uint16), got %s" % x.dtype)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def forward(q: np.ndarray, k: np.ndarray, v: np.ndarray, beta, M_in=None, z_in=None,
            seg_len: int = 1, nthreads: int = 1, segments: Optional[Sequence[int]] = None,
            _lib_override=None):
    """Run the oracle.

    q, k, v: [B, H, L, d] arrays (float32, float64 or bf16 bits as uint16),
    all the same dtype. beta: [H]. M_in: [B, H, d, d], z_in: [B, H, d] or None
    for the zero state. Returns (out, M_out, z_out) as float64 arrays; with
    ``segments`` given, out is [B, H, len(segments), N, d] holding only those
    segments' rows (the state chain still covers every segment).
    """
    lib = _lib_override if _lib_override is not None else _load()
    q, dt = _as_input(q)
    k, dtk = _as_input(k)
    v, dtv = _as_input(v)
    if not (dt == dtk == dtv):
        raise TypeError("q, k, v must share a dtype")
    if q.ndim != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must be [B, H, L, d] with equal shapes")
    B, H, L, d = q.shape
    N = int(seg_len)
    beta = np.ascontiguousarray(np.asarray(beta, dtype=np.float64).reshape(H))
    if (M_in is None) != (z_in is None):
        raise ValueError("M_in and z_in must both be given or both be None")
    if M_in is not None:
        M_in = np.ascontiguousarray(np.asarray(M_in, dtype=np.float64).reshape(B, H, d, d))
        z_in = np.ascontiguousarray(np.asarray(z_in, dtype=np.float64).reshape(B, H, d))
    M_out = np.empty((B, H, d, d), np.float64)
    z_out = np.empty((B, H, d), np.float64)
    if segments is None:
        out = np.empty((B, H, L, d), np.float64)
        rc = lib.oracle_infini_forward(B, H, L, d, N, _ptr(q), _ptr(k), _ptr(v), dt,
                                       _ptr(beta), _ptr(M_in), _ptr(z_in),
                                       _ptr(out), _ptr(M_out), _ptr(z_out), int(nthreads))
    else:
        seg = np.ascontiguousarray(np.asarray(segments, dtype=np.int64))
        out = np.empty((B, H, len(seg), N, d), np.float64)
        rc = lib.oracle_infini_forward_segments(B, H, L, d, N, _ptr(q), _ptr(k), _ptr(v), dt,
                                                _ptr(beta), _ptr(M_in), _ptr(z_in),
                                                _ptr(seg), len(seg),
                                                _ptr(out), _ptr(M_out), _ptr(z_out), int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments (code %d)" % rc)
    return out, M_out, z_out


def decode_step(q, k, v, k_cache, v_cache, pos: int, beta, M, z, _lib_override=None):
    """One decode step of the oracle.

    q, k, v: [B, H, d] (this token); k_cache, v_cache: [B, H, N, d] whose rows
    0..pos-1 hold the current segment's earlier keys and values (same dtype as
    q). beta: [H]. M: [B, H, d, d], z: [B, H, d], the memory of earlier
    segments. Returns (out [B, H, d], M_new, z_new) as float64 arrays; M_new and
    z_new include the segment when pos == N - 1 and equal M, z otherwise.
    """
    lib = _lib_override if _lib_override is not None else _load()
    q, dt = _as_input(q)
    k, dtk = _as_input(k)
    v, dtv = _as_input(v)
    kc, dkc = _as_input(k_cache)
    vc, dvc = _as_input(v_cache)
    if not (dt == dtk == dtv == dkc == dvc):
        raise TypeError("q, k, v and the caches must share a dtype")
    B, H, d = q.shape
    N = kc.shape[2]
    if kc.shape != (B, H, N, d) or vc.shape != kc.shape or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v: [B, H, d]; caches: [B, H, N, d]")
    beta = np.ascontiguousarray(np.asarray(beta, dtype=np.float64).reshape(H))
    M = np.array(np.asarray(M, dtype=np.float64).reshape(B, H, d, d), copy=True)
    z = np.array(np.asarray(z, dtype=np.float64).reshape(B, H, d), copy=True)
    out = np.empty((B, H, d), np.float64)
    rc = lib.oracle_infini_decode_step(B, H, d, N, int(pos), _ptr(q), _ptr(k), _ptr(v), _ptr(kc), _ptr(vc),
                                       dt, _ptr(beta), _ptr(M), _ptr(z), _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected the arguments (code %d)" % rc)
    return out, M, z


def backward(q, k, v, beta, dout, M_in=None, z_in=None, dM_out=None, dz_out=None, seg_len: int = 1,
             nthreads: int = 1, _lib_override=None):
    """Gradients of the forward (the oracle's backward, in double).

    q, k, v: [B, H, L, d] (float32, float64 or bf16 bits); beta [H]; M_in, z_in
    the incoming state or None; dout [B, H, L, d] the gradient of out; dM_out,
    dz_out the gradient of the output state or None. Returns (dq, dk, dv, dbeta
    [H], dM_in, dz_in) as float64 arrays.
    """
    lib = _lib_override if _lib_override is not None else _load()
    q, dt = _as_input(q)
    k, dtk = _as_input(k)
    v, dtv = _as_input(v)
    if not (dt == dtk == dtv):
        raise TypeError("q, k, v must share a dtype")
    B, H, L, d = q.shape
    beta = np.ascontiguousarray(np.asarray(beta, dtype=np.float64).reshape(H))
    dout = np.ascontiguousarray(np.asarray(dout, dtype=np.float64).reshape(B, H, L, d))
    def st(x, shape):
        return None if x is None else np.ascontiguousarray(np.asarray(x, dtype=np.float64).reshape(shape))
    M_in, z_in = st(M_in, (B, H, d, d)), st(z_in, (B, H, d))
    dM_out, dz_out = st(dM_out, (B, H, d, d)), st(dz_out, (B, H, d))
    dq, dk, dv = (np.empty((B, H, L, d), np.float64) for _ in range(3))
    dbeta_bh = np.empty((B, H), np.float64)
    dM_in, dz_in = np.empty((B, H, d, d), np.float64), np.empty((B, H, d), np.float64)
    rc = lib.oracle_infini_backward(B, H, L, d, int(seg_len), _ptr(q), _ptr(k), _ptr(v), dt, _ptr(beta),
                                    _ptr(M_in), _ptr(z_in), _ptr(dout), _ptr(dM_out), _ptr(dz_out),
                                    _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dbeta_bh), _ptr(dM_in), _ptr(dz_in),
                                    int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected the arguments (code %d)" % rc)
    return dq, dk, dv, dbeta_bh.sum(axis=0), dM_in, dz_in
