"""The C ABI on the host (no GPU needed): the library loads, exports every
symbol the header declares, and rejects bad arguments before launching
anything. Fake pointers are only ever passed together with an argument error
that the library catches before any CUDA call."""
import ctypes
import os
import re

import pytest

from compressive_memory_segment_b200 import binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"INFINI_API\s+[\w\s\*]+?\b(infini_\w+)\s*\(", txt)
    return sorted(set(names))


def test_exports_every_declared_symbol():
    lib = ctypes.CDLL(bd.LIB_PATH)
    declared = _declared_symbols()
    assert len(declared) >= 8
    for name in declared:
        assert hasattr(lib, name), name
    assert set(bd.EXPORTED) <= set(declared)


def test_version_and_strerror():
    assert bd.infini_attn_version() >= 100
    for code in range(-9, 1):
        assert len(bd.infini_attn_strerror(code)) > 5
    assert "unknown" in bd.infini_attn_strerror(-1000)


def shp(B=1, H=2, L=256, d=128, dt=bd.INFINI_BF16):
    return bd.make_shape(B, H, L, d, dt)


def test_workspace_size():
    # dM + dz + Mp + zp, each rounded to 256 bytes.
    B, H, L, d, N = 2, 3, 512, 128, 128
    S = L // N
    mat = B * H * S * d * d * 4
    vec = B * H * S * d * 4
    rnd = lambda x: (x + 255) // 256 * 256
    want = rnd(mat) + rnd(vec) + rnd(mat) + rnd(vec)
    assert bd.infini_attn_workspace_size(shp(B, H, L, d), N) == want
    assert bd.infini_attn_workspace_size(shp(L=100), 64) == 0   # L % N != 0
    assert bd.infini_attn_workspace_size(shp(d=96), 64) == 0    # unsupported d


def test_select_path():
    from compressive_memory_segment_b200.binding import infini_attn_select_path as sel
    assert sel(shp(dt=bd.INFINI_F32), 128) == bd.INFINI_PATH_SIMT
    assert sel(shp(d=64), 64) == bd.INFINI_PATH_TC              # bf16, d = 64, 64-token segments
    assert sel(shp(d=64), 128) == bd.INFINI_PATH_SIMT
    assert sel(shp(d=64, dt=bd.INFINI_F32), 64) == bd.INFINI_PATH_SIMT
    assert sel(shp(L=192), 64) == bd.INFINI_PATH_SIMT           # seg_len not a multiple of 128
    assert sel(shp(), 0) == bd.INFINI_ERR_SHAPE
    assert sel(shp(L=512), 256) == bd.INFINI_PATH_TC                # bf16, d = 128, N % 128 == 0
    assert bd.infini_attn_launch_count(shp(L=512), 256, bd.INFINI_PATH_TC) == 3
    assert bd.infini_attn_launch_count(shp(), 128, bd.INFINI_PATH_SIMT) == 3
    # The paired-query-tile attention kernel: bf16, d = 128, seg_len % 256 == 0, never AUTO.
    assert bd.infini_attn_launch_count(shp(L=512), 256, bd.INFINI_PATH_TC_PAIRED) == 3
    assert bd.infini_attn_launch_count(shp(L=512), 128, bd.INFINI_PATH_TC_PAIRED) == bd.INFINI_ERR_UNSUPPORTED
    assert bd.infini_attn_launch_count(shp(d=64), 64, bd.INFINI_PATH_TC_PAIRED) == bd.INFINI_ERR_UNSUPPORTED
    # d = 64 with 64-token segments: one single-pass kernel per forward.
    assert bd.infini_attn_launch_count(shp(d=64), 64, bd.INFINI_PATH_TC) == 1
    assert bd.infini_attn_launch_count(shp(d=64), 64, bd.INFINI_PATH_SIMT) == 3
    assert bd.infini_attn_launch_count(shp(dt=bd.INFINI_F32), 128, bd.INFINI_PATH_TC) == bd.INFINI_ERR_UNSUPPORTED


# Distinct, 16-byte aligned fake device addresses, far apart.
A = [0x7f0000000000 + i * (1 << 32) for i in range(16)]


def call(shape, seg_len=128, q=A[0], k=A[1], v=A[2], beta=A[3], M_in=None, z_in=None,
         out=A[4], M_out=A[5], z_out=A[6], ws=A[7], ws_bytes=None, path=0):
    if ws_bytes is None:
        ws_bytes = max(bd.infini_attn_workspace_size(shape, seg_len), 1)
    return bd.infini_attn_forward_ws(shape, q, k, v, beta, M_in, z_in, seg_len, out, M_out, z_out,
                                     ws, ws_bytes, path, 0)


@pytest.mark.parametrize("field", ["q", "k", "v", "beta", "out", "M_out", "z_out", "ws"])
def test_null_pointers(field):
    assert call(shp(), **{field: None}) == bd.INFINI_ERR_NULL


def test_half_state_is_null_error():
    assert call(shp(), M_in=A[8]) == bd.INFINI_ERR_NULL
    assert call(shp(), z_in=A[9]) == bd.INFINI_ERR_NULL
    assert bd.infini_attn_forward(shp(), A[0], A[1], A[2], A[3], A[8], None, 128, A[4], A[5], A[6], 0) \
        == bd.INFINI_ERR_NULL


@pytest.mark.parametrize("shape,seg", [
    (dict(B=0), 128), (dict(H=0), 128), (dict(L=0), 128), (dict(), 0), (dict(), -4),
    (dict(L=300), 128), (dict(L=256), 96)])
def test_shape_errors(shape, seg):
    assert call(shp(**shape), seg_len=seg) == bd.INFINI_ERR_SHAPE


@pytest.mark.parametrize("shape", [dict(d=32), dict(d=96), dict(d=256), dict(dt=7)])
def test_unsupported(shape):
    assert call(shp(**shape)) == bd.INFINI_ERR_UNSUPPORTED


def test_forced_tc_path_on_uncovered_shape():
    assert call(shp(dt=bd.INFINI_F32), path=bd.INFINI_PATH_TC) == bd.INFINI_ERR_UNSUPPORTED
    assert call(shp(d=64), path=bd.INFINI_PATH_TC) == bd.INFINI_ERR_UNSUPPORTED
    assert call(shp(), path=9) == bd.INFINI_ERR_UNSUPPORTED


@pytest.mark.parametrize("field", ["q", "k", "v", "beta", "out", "M_out", "z_out"])
def test_misaligned(field):
    base = dict(q=A[0], k=A[1], v=A[2], beta=A[3], out=A[4], M_out=A[5], z_out=A[6])
    assert call(shp(), **{field: base[field] + 8}) == bd.INFINI_ERR_ALIGN


def test_misaligned_workspace_and_state():
    assert call(shp(), ws=A[7] + 16) == bd.INFINI_ERR_ALIGN
    assert call(shp(), M_in=A[8] + 4, z_in=A[9]) == bd.INFINI_ERR_ALIGN


def test_workspace_too_small():
    s = shp()
    assert call(s, ws_bytes=bd.infini_attn_workspace_size(s, 128) - 256) == bd.INFINI_ERR_WORKSPACE


def test_aliasing():
    s = shp()
    assert call(s, out=A[0]) == bd.INFINI_ERR_ALIAS                   # out == q
    assert call(s, out=A[1] + 1024) == bd.INFINI_ERR_ALIAS            # out inside k
    assert call(s, M_out=A[2] + 4096) == bd.INFINI_ERR_ALIAS          # M_out inside v
    assert call(s, z_out=A[5] + 16) == bd.INFINI_ERR_ALIAS            # z_out inside M_out
    assert call(s, M_in=A[8], z_in=A[9], M_out=A[8] + 64) == bd.INFINI_ERR_ALIAS  # partial overlap


def test_size_limit():
    assert call(shp(B=1, H=1 << 10, L=1 << 21, d=64), seg_len=1 << 11) == bd.INFINI_ERR_SIZE


def test_forward_validates_before_allocating():
    # The allocating entry point checks everything before cudaMallocAsync.
    assert bd.infini_attn_forward(shp(L=300), A[0], A[1], A[2], A[3], None, None, 128,
                                  A[4], A[5], A[6], 0) == bd.INFINI_ERR_SHAPE
    assert bd.infini_attn_forward(shp(), A[0], A[1], A[2], A[3], None, None, 128,
                                  A[0], A[5], A[6], 0) == bd.INFINI_ERR_ALIAS


def test_selftest_timeout_validates_limit():
    # Out-of-range limits are rejected on the host; nothing is launched.
    assert bd.infini_attn_selftest_timeout(0, 0) == bd.INFINI_ERR_SHAPE
    assert bd.infini_attn_selftest_timeout(999, 0) == bd.INFINI_ERR_SHAPE
    assert bd.infini_attn_selftest_timeout(100_000_001, 0) == bd.INFINI_ERR_SHAPE


# ------------------------------------------------------------------ decode step

def dcall(B=1, H=2, N=8, d=128, dt=bd.INFINI_BF16, pos=3, ws=A[9], ws_bytes=None, **kw):
    shape = bd.make_shape(B, H, N, d, dt)
    p = dict(q=A[0], k=A[1], v=A[2], beta=A[3], kc=A[4], vc=A[5], M=A[6], z=A[7], out=A[8])
    p.update(kw)
    if ws_bytes is None:
        ws_bytes = max(bd.infini_attn_decode_workspace_size(shape), 1)
    return bd.infini_attn_decode_step(shape, p["q"], p["k"], p["v"], p["beta"], p["kc"], p["vc"], pos,
                                      p["M"], p["z"], p["out"], ws, ws_bytes, 0)


def test_decode_workspace_size():
    # The one-segment forward workspace (for the fold), then per (b, h) the
    # chunk partials (m, l, acc[d]) of ceil(N / 128) chunks and (den, num[d]).
    B, H, N, d = 2, 3, 600, 128
    s = bd.make_shape(B, H, N, d, bd.INFINI_BF16)
    rnd = lambda x: (x + 255) // 256 * 256
    chunks = (N + 127) // 128
    want = rnd(rnd(bd.infini_attn_workspace_size(s, N)) + B * H * (chunks * (d + 2) + d + 1) * 4)
    assert bd.infini_attn_decode_workspace_size(s) == want
    assert bd.infini_attn_decode_workspace_size(bd.make_shape(1, 1, 65536, 64, bd.INFINI_F32)) == 0  # N too long


@pytest.mark.parametrize("field", ["q", "k", "v", "beta", "kc", "vc", "M", "z", "out"])
def test_decode_null(field):
    assert dcall(**{field: None}) == bd.INFINI_ERR_NULL


def test_decode_workspace_checks():
    assert dcall(pos=2, ws=None) == bd.INFINI_ERR_NULL
    assert dcall(pos=7, ws=None) == bd.INFINI_ERR_NULL
    assert dcall(pos=7, ws=A[9] + 16) == bd.INFINI_ERR_ALIGN
    assert dcall(pos=7, ws_bytes=16) == bd.INFINI_ERR_WORKSPACE
    assert dcall(pos=7, ws=A[0]) == bd.INFINI_ERR_ALIAS  # workspace over q


@pytest.mark.parametrize("pos", [-1, 8, 100])
def test_decode_position_range(pos):
    assert dcall(pos=pos) == bd.INFINI_ERR_SHAPE


def test_decode_shape_and_alignment_errors():
    assert dcall(d=96) == bd.INFINI_ERR_UNSUPPORTED
    assert dcall(dt=5) == bd.INFINI_ERR_UNSUPPORTED
    assert dcall(B=0) == bd.INFINI_ERR_SHAPE
    assert dcall(N=40000, pos=1) == bd.INFINI_ERR_SIZE
    assert dcall(q=A[0] + 8) == bd.INFINI_ERR_ALIGN
    assert dcall(kc=A[4] + 4) == bd.INFINI_ERR_ALIGN


def test_decode_aliasing():
    assert dcall(out=A[0]) == bd.INFINI_ERR_ALIAS          # out == q
    assert dcall(kc=A[5]) == bd.INFINI_ERR_ALIAS           # the two caches
    assert dcall(M=A[4] + 256) == bd.INFINI_ERR_ALIAS      # M inside the key cache
    assert dcall(z=A[6] + 64) == bd.INFINI_ERR_ALIAS       # z inside M


# ------------------------------------------------------------------ backward

def bcall(shape=None, **kw):
    shape = shape or shp()
    p = dict(q=A[0], k=A[1], v=A[2], beta=A[3], M_in=None, z_in=None, dout=A[4], dM_out=None, dz_out=None,
             dq=A[5], dk=A[6], dv=A[7], dbeta=A[8], dM_in=A[9], dz_in=A[10], ws=A[11])
    p.update(kw)
    n = max(bd.infini_attn_backward_workspace_size(shape, 128), 1)
    return bd.infini_attn_backward(shape, p["q"], p["k"], p["v"], p["beta"], p["M_in"], p["z_in"], 128, p["dout"],
                                   p["dM_out"], p["dz_out"], p["dq"], p["dk"], p["dv"], p["dbeta"], p["dM_in"],
                                   p["dz_in"], p["ws"], kw.get("ws_bytes", n), 0)


def test_backward_workspace_covers_forward_workspace():
    s = shp(B=2, H=3, L=512)
    assert bd.infini_attn_backward_workspace_size(s, 128) > bd.infini_attn_workspace_size(s, 128)
    assert bd.infini_attn_backward_workspace_size(shp(L=300), 128) == 0


@pytest.mark.parametrize("field", ["q", "k", "v", "beta", "dout", "dq", "dk", "dv", "dbeta", "dM_in", "dz_in", "ws"])
def test_backward_null(field):
    assert bcall(**{field: None}) == bd.INFINI_ERR_NULL


def test_backward_half_state_and_errors():
    assert bcall(M_in=A[12]) == bd.INFINI_ERR_NULL
    assert bcall(dM_out=A[12]) == bd.INFINI_ERR_NULL
    assert bcall(shp(L=300)) == bd.INFINI_ERR_SHAPE
    assert bcall(q=A[0] + 8) == bd.INFINI_ERR_ALIGN
    assert bcall(ws=A[11] + 16) == bd.INFINI_ERR_ALIGN
    assert bcall(ws_bytes=256) == bd.INFINI_ERR_WORKSPACE


def test_backward_aliasing():
    assert bcall(dq=A[0]) == bd.INFINI_ERR_ALIAS          # gradient over q
    assert bcall(dk=A[5] + 64) == bd.INFINI_ERR_ALIAS     # dk inside dq
    assert bcall(dbeta=A[3]) == bd.INFINI_ERR_ALIAS       # dbeta over beta
    assert bcall(ws=A[4]) == bd.INFINI_ERR_ALIAS          # workspace over dout


def test_backward_path_choice():
    """An explicit backward path that the shape does not allow is refused
    before anything runs; the tensor-core backward covers bf16 with d = 128
    and segments of whole 128-row tiles, and bf16 with d = 64, 64-token
    segments and an even number of them."""
    def pcall(shape, path, N=128, **kw):
        p = dict(q=A[0], k=A[1], v=A[2], beta=A[3], dout=A[4], dq=A[5], dk=A[6], dv=A[7], dbeta=A[8], dM_in=A[9],
                 dz_in=A[10], ws=A[11])
        p.update(kw)
        n = max(bd.infini_attn_backward_workspace_size(shape, N), 1)
        return bd.infini_attn_backward_path(shape, p["q"], p["k"], p["v"], p["beta"], None, None, N, p["dout"], None,
                                            None, p["dq"], p["dk"], p["dv"], p["dbeta"], p["dM_in"], p["dz_in"],
                                            p["ws"], n, path, 0)
    U = bd.INFINI_ERR_UNSUPPORTED
    assert pcall(shp(dt=bd.INFINI_F32), bd.INFINI_PATH_TC) == U
    assert pcall(shp(d=64, L=192), bd.INFINI_PATH_TC, 64) == U     # d = 64: an odd number of segments
    assert pcall(shp(d=64), bd.INFINI_PATH_TC, 128) == U           # d = 64: segments of 128 tokens
    assert pcall(shp(L=192), bd.INFINI_PATH_TC, 64) == U          # seg_len not a multiple of 128
    assert pcall(shp(), bd.INFINI_PATH_TC_PAIRED) == U
    assert pcall(shp(), 9) == U
    assert pcall(shp(), bd.INFINI_PATH_TC, q=None) == bd.INFINI_ERR_NULL
    assert pcall(shp(), bd.INFINI_PATH_SIMT, dq=None) == bd.INFINI_ERR_NULL


def _trace_symbols():
    txt = open(os.path.join(ROOT, "include", "infini_attn_trace.h")).read()
    return sorted(set(re.findall(r"INFINI_TRACE_API\s+[\w\s\*]+?\b(infini_\w+)\s*\(", txt)))


def test_trace_entry_points_only_in_the_tracing_build():
    """The regular library records no trace and exports no trace entry point;
    the tracing build (compiled here, for sm_100a) exports every one the trace
    header declares and checks its arguments on the host."""
    from compressive_memory_segment_b200 import build as b
    names = _trace_symbols()
    assert names == ["infini_attn_trace_read", "infini_attn_trace_reset"]
    lib = ctypes.CDLL(bd.LIB_PATH)
    for name in names:
        assert not hasattr(lib, name), name
    tlib = ctypes.CDLL(b.build(trace=True))
    for name in names:
        assert hasattr(tlib, name), name
    tlib.infini_attn_trace_read.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_int]
    assert tlib.infini_attn_trace_read(-1, None, 0) == bd.INFINI_ERR_SHAPE
    assert tlib.infini_attn_trace_read(8, None, 0) == bd.INFINI_ERR_SHAPE  # channels 0 .. 7
    assert tlib.infini_attn_trace_read(0, None, -1) == bd.INFINI_ERR_SHAPE
    assert tlib.infini_attn_trace_read(0, None, 4) == bd.INFINI_ERR_NULL
