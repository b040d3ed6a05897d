"""The allocation-free entry point, infini_attn_forward_noalloc.

It serves callers that cannot allocate device memory (all of it already
reserved by another allocator, or a code path that must not enter the CUDA
allocator because cudaMalloc/cudaFree can block or synchronise the device).
Its scratch is a fixed buffer compiled into the library, shared by every call.
These tests call it through the C ABI and compare it with the workspace entry
point, infini_attn_forward_ws, within the same tolerances the parity tests
use. This file is named to be collected last; it must pass both on its own in
a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

from compressive_memory_segment_b200 import binding as bd
from compressive_memory_segment_b200 import synth
from tests.parity import TOL, slice_err


def _inputs(B, H, L, d, N, dtype, seed, state):
    w = synth.Workload("noalloc", B, H, d, N, L // N, dtype, seed, beta="normal")
    q, k, v = synth.make_qkv(w, "cuda")
    beta = synth.make_beta(w, "cuda")
    M = z = None
    if state:
        M, z = synth.make_state(w, "cuda", scale=2.0)
    return q, k, v, beta, M, z


def _outputs(q):
    B, H, L, d = q.shape
    return (torch.empty_like(q), torch.empty((B, H, d, d), dtype=torch.float32, device=q.device),
            torch.empty((B, H, d), dtype=torch.float32, device=q.device))


def _with_workspace(q, k, v, beta, M, z, N):
    out, Mo, zo = _outputs(q)
    ws = bd.workspace_for(q, N)
    rc = bd.infini_attn_forward_ws(bd.shape_of(q), q, k, v, beta, M, z, N, out, Mo, zo, ws, ws.numel(),
                                   bd.INFINI_PATH_AUTO, None)
    assert rc == bd.INFINI_OK, bd.infini_attn_strerror(rc)
    return out, Mo, zo


def _close(got, ref, kind):
    tol = TOL[kind]
    eo = slice_err(got[0].float().cpu().numpy(), ref[0].double().cpu().numpy())
    eM = slice_err(got[1].cpu().numpy(), ref[1].double().cpu().numpy())
    ez = slice_err(got[2].cpu().numpy(), ref[2].double().cpu().numpy())
    assert eo <= tol["out"] and eM <= tol["M"] and ez <= tol["z"], (kind, eo, eM, ez)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(cuda_ok):
    cases = [
        # B, H, L, d, N, dtype, seed, incoming state
        (1, 2, 1024, 128, 256, "bf16", 11, False),
        (2, 3, 384, 64, 128, "f32", 12, True),
        (1, 2, 1024, 128, 256, "bf16", 13, True),
    ]
    prepared = []
    for B, H, L, d, N, dt, seed, state in cases:
        q, k, v, beta, M, z = _inputs(B, H, L, d, N, dt, seed, state)
        ref = _with_workspace(q, k, v, beta, M, z, N)
        prepared.append((q, k, v, beta, M, z, N, dt, ref))
    torch.cuda.synchronize()
    # Back-to-back calls on one stream, no synchronisation in between: each
    # call must only see its own scratch contents.
    results = []
    for q, k, v, beta, M, z, N, dt, ref in prepared:
        out, Mo, zo = _outputs(q)
        rc = bd.infini_attn_forward_noalloc(bd.shape_of(q), q, k, v, beta, M, z, N, out, Mo, zo, None)
        assert rc == bd.INFINI_OK, bd.infini_attn_strerror(rc)
        results.append((out, Mo, zo))
    assert bd.infini_attn_device_status(None) == bd.INFINI_OK
    for (q, k, v, beta, M, z, N, dt, ref), got in zip(prepared, results):
        _close(got, ref, dt)


@pytest.mark.gpu
def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_ok):
    q = torch.zeros((1, 64, 2048, 128), dtype=torch.bfloat16, device="cuda")
    shp = bd.shape_of(q)
    assert bd.infini_attn_workspace_size(shp, 128) > bd.INFINI_NOALLOC_SCRATCH_BYTES
    out, Mo, zo = _outputs(q)
    beta = torch.zeros(64, device="cuda")
    rc = bd.infini_attn_forward_noalloc(shp, q, q, q, beta, None, None, 128, out, Mo, zo, None)
    assert rc == bd.INFINI_ERR_SCRATCH
    assert "scratch" in bd.infini_attn_strerror(rc)
