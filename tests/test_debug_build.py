"""The debug build of the library (INFINI_DEBUG): the same kernels with
device-side index checks on their global stores and TMA coordinates, which
record INFINI_ERR_BOUNDS in the status word instead of trapping (the regular
build compiles them away). On the CPU: the debug build compiles for sm_100a
and exports the same entry points. On a GPU: small and odd shapes on every
path, and a decode step, leave the status clean and match the CPU oracle.
"""
import ctypes

import pytest
import torch

from compressive_memory_segment_b200 import binding as bd
from compressive_memory_segment_b200 import build as b
from compressive_memory_segment_b200 import synth
from tests.parity import assert_close, run_oracle


def _debug_lib():
    return bd.open_library(b.build(debug=True))


def test_debug_build_exports_the_same_entry_points():
    lib = _debug_lib()
    for name in bd.EXPORTED:
        assert hasattr(lib, name), name
    assert lib.infini_attn_strerror(bd.INFINI_ERR_BOUNDS).decode().startswith("a device-side index check")
    # Host-side argument checks are the same as the regular build's.
    shp = bd.make_shape(1, 1, 100, 128, bd.INFINI_BF16)
    assert lib.infini_attn_workspace_size(ctypes.byref(shp), 30) == 0


CASES = [
    # B, H, L, d, N, dtype, path
    (1, 1, 128, 128, 128, "bf16", bd.INFINI_PATH_TC),
    (1, 2, 512, 128, 256, "bf16", bd.INFINI_PATH_TC),
    (2, 1, 1152, 128, 384, "bf16", bd.INFINI_PATH_TC),
    (1, 1, 192, 64, 64, "bf16", bd.INFINI_PATH_TC),
    (1, 1, 192, 64, 64, "bf16", bd.INFINI_PATH_SIMT),
    (1, 2, 200, 128, 100, "bf16", bd.INFINI_PATH_SIMT),
    (1, 1, 65, 64, 65, "f32", bd.INFINI_PATH_SIMT),
]


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,L,d,N,dt,path", CASES)
def test_debug_build_index_checks_stay_clean(cuda_ok, B, H, L, d, N, dt, path):
    lib = _debug_lib()
    w = synth.Workload("debug", B, H, d, L, 1, dt, 500 + L + d + N, beta="normal")
    q, k, v = synth.make_qkv(w, "cuda")
    beta = synth.make_beta(w, "cuda")
    out = torch.empty_like(q)
    M = torch.empty((B, H, d, d), device="cuda")
    z = torch.empty((B, H, d), device="cuda")
    shp = bd.shape_of(q)
    n = bd.infini_attn_workspace_size(shp, N)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    rc = lib.infini_attn_forward_ws(ctypes.byref(shp), q.data_ptr(), k.data_ptr(), v.data_ptr(), beta.data_ptr(),
                                    None, None, N, out.data_ptr(), M.data_ptr(), z.data_ptr(), ws.data_ptr(), n, path,
                                    torch.cuda.current_stream().cuda_stream)
    assert rc == bd.INFINI_OK
    st = lib.infini_attn_device_status(torch.cuda.current_stream().cuda_stream)
    assert st == bd.INFINI_OK, lib.infini_attn_strerror(st).decode()
    assert_close((out, M, z), run_oracle(q, k, v, beta, N), dt, "debug build %s path %d" % ((B, H, L, d, N), path))
