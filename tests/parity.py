"""Helpers for GPU-vs-oracle parity: run the CUDA library through the C ABI on
seeded inputs, run the CPU oracle on the same bits, compare.

Error metric (the specification states "max relative error" without a norm;
elementwise relative error is ill-posed for entries near zero):
    err(X) = max_i |X_i - R_i| / max_i |R_i|
per (b, h) slice, worst slice reported. Bounds: fp32 I/O 1e-4 for out, M, z;
bf16 I/O 2e-2 for out and 5e-3 for M and z. The bound is normwise per slice:
an element whose reference is small against the slice's largest may be off by
more than the tolerance relative to itself. So the elementwise relative error
    elem(X) = max_i |X_i - R_i| / (|R_i| + 1e-3 max_j |R_j|)
is reported beside it for every comparison (REPORT, printed at the end of the
pytest run); it is a reported figure, not asserted.
"""
import os

import numpy as np
import torch

import oracle
from compressive_memory_segment_b200 import binding as bd
from compressive_memory_segment_b200 import synth

TOL = {"f32": dict(out=1e-4, M=1e-4, z=1e-4), "bf16": dict(out=2e-2, M=5e-3, z=5e-3)}
NTHREADS = max(1, min(32, os.cpu_count() or 1))


def host_bits(t: torch.Tensor):
    """Tensor -> numpy array the oracle accepts (bf16 as uint16 bits)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def slice_err(x: np.ndarray, r: np.ndarray, lead: int = 2) -> float:
    """Worst over the leading `lead` dims of max|x - r| / max|r|."""
    x = x.reshape(int(np.prod(x.shape[:lead])), -1).astype(np.float64)
    r = r.reshape(int(np.prod(r.shape[:lead])), -1)
    num = np.max(np.abs(x - r), axis=1)
    den = np.maximum(np.max(np.abs(r), axis=1), 1e-30)
    return float(np.max(num / den))


def elem_err(x: np.ndarray, r: np.ndarray, lead: int = 2) -> float:
    """Worst over the leading `lead` dims of max |x - r| / (|r| + 1e-3 max|r|)."""
    x = x.reshape(int(np.prod(x.shape[:lead])), -1).astype(np.float64)
    r = r.reshape(int(np.prod(r.shape[:lead])), -1)
    floor = 1e-3 * np.maximum(np.max(np.abs(r), axis=1, keepdims=True), 1e-30)
    return float(np.max(np.abs(x - r) / (np.abs(r) + floor)))


# (what, normwise errors, elementwise errors) of every assert_close call.
REPORT = []


def record(what: str, norm, elem):
    REPORT.append((what, tuple(norm), tuple(elem)))


def run_gpu(q, k, v, beta, seg_len, M_in=None, z_in=None, path=bd.INFINI_PATH_AUTO, inplace=False):
    """One forward call through infini_attn_forward_ws; returns (out, M, z)."""
    B, H, L, d = q.shape
    out = torch.empty_like(q)
    if inplace and M_in is not None:
        M_out, z_out = M_in, z_in
    else:
        M_out = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device)
        z_out = torch.empty((B, H, d), dtype=torch.float32, device=q.device)
    ws = bd.workspace_for(q, seg_len)
    rc = bd.infini_attn_forward_ws(bd.shape_of(q), q, k, v, beta, M_in, z_in, seg_len, out, M_out,
                                   z_out, ws, ws.numel(), path, None)
    assert rc == bd.INFINI_OK, bd.infini_attn_strerror(rc)
    assert bd.infini_attn_device_status(None) == bd.INFINI_OK
    return out, M_out, z_out


def run_oracle(q, k, v, beta, seg_len, M_in=None, z_in=None, segments=None):
    Mi = None if M_in is None else M_in.detach().cpu().double().numpy()
    zi = None if z_in is None else z_in.detach().cpu().double().numpy()
    return oracle.forward(host_bits(q), host_bits(k), host_bits(v), beta.detach().cpu().double().numpy(),
                          Mi, zi, seg_len=seg_len, nthreads=NTHREADS, segments=segments)


def assert_close(gpu, ref, kind: str, what: str = ""):
    tol = TOL[kind]
    out, M, z = gpu
    ro, rM, rz = ref
    xo, xM, xz = out.float().cpu().numpy(), M.cpu().numpy(), z.cpu().numpy()
    eo, eM, ez = slice_err(xo, ro), slice_err(xM, rM), slice_err(xz, rz)
    el = (elem_err(xo, ro), elem_err(xM, rM), elem_err(xz, rz))
    record(what, (eo, eM, ez), el)
    assert np.isfinite(xo).all(), what + ": non-finite output"
    assert eo <= tol["out"] and eM <= tol["M"] and ez <= tol["z"], \
        "%s: err out %.3e (<= %.1e) M %.3e (<= %.1e) z %.3e (<= %.1e); elementwise %.2e %.2e %.2e" % (
            what, eo, tol["out"], eM, tol["M"], ez, tol["z"], *el)
    return eo, eM, ez
