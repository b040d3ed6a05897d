"""GPU parity: the CUDA library (through the C ABI) against the CPU oracle on
seeded inputs. Small cases compare every element; the full-size workloads
compare the final state exactly-in-tolerance and sampled segments' outputs.

Tolerances (in tests/parity.py): fp32 I/O 1e-4 on out, M, z; bf16 I/O 2e-2 on
out and 5e-3 on M and z, as max|x - ref| / max|ref| per (b, h) slice.
"""
import math

import numpy as np
import pytest
import torch

from compressive_memory_segment_b200 import binding as bd
from compressive_memory_segment_b200 import synth
from tests.parity import assert_close, elem_err, record, run_gpu, run_oracle, slice_err, TOL

pytestmark = pytest.mark.gpu

DEV = "cuda"


def paths_for(q, seg_len):
    """The SIMT path always; the tensor-core path where it covers the shape,
    and its paired-query-tile attention kernel where that covers it."""
    shp = bd.shape_of(q)
    ps = [bd.INFINI_PATH_SIMT]
    for p in (bd.INFINI_PATH_TC, bd.INFINI_PATH_TC_PAIRED):
        if bd.infini_attn_launch_count(shp, seg_len, p) > 0:
            ps.append(p)
    return ps


def inputs(B, H, L, d, dtype, seed, scale=1.0, beta="normal", state=False):
    w = synth.Workload("case", B, H, d, L, 1, "f32" if dtype == torch.float32 else "bf16", seed,
                       qkv_scale=scale, beta=beta)
    q, k, v = synth.make_qkv(w, DEV)
    b = synth.make_beta(w, DEV)
    M = z = None
    if state:
        M, z = synth.make_state(w, DEV, scale=4.0)
    return q, k, v, b, M, z


# --------------------------------------------------------------- workloads 1, 2

def test_tiny_f32_full(cuda_ok):
    w = synth.WORKLOADS["tiny_f32"]
    q, k, v = synth.make_qkv(w, DEV)
    beta = synth.make_beta(w, DEV)
    ref = run_oracle(q, k, v, beta, w.N)
    for path in paths_for(q, w.N):
        assert_close(run_gpu(q, k, v, beta, w.N, path=path), ref, "f32", "tiny_f32 path %d" % path)


def test_hf_repro_bf16_full(cuda_ok):
    w = synth.WORKLOADS["hf_repro_bf16"]
    q, k, v = synth.make_qkv(w, DEV)
    beta = synth.make_beta(w, DEV)
    ref = run_oracle(q, k, v, beta, w.N)
    for path in paths_for(q, w.N):
        assert_close(run_gpu(q, k, v, beta, w.N, path=path), ref, "bf16", "hf_repro path %d" % path)


# --------------------------------------------------------------- small shapes, every element

CASES = [
    # B, H, L, d, N, dtype
    (1, 2, 1152, 128, 384, torch.bfloat16),   # 3 segments x 3 q-tiles of 128
    (2, 1, 1024, 128, 256, torch.bfloat16),
    (1, 1, 512, 128, 512, torch.bfloat16),    # S = 1
    (1, 3, 640, 128, 128, torch.bfloat16),    # one tile per segment
    (1, 2, 600, 128, 200, torch.bfloat16),    # N not a multiple of 128 (ragged tail)
    (2, 2, 300, 64, 100, torch.bfloat16),
    (1, 2, 192, 64, 64, torch.bfloat16),      # d = 64, 64-token segments: an odd count (3)
    (2, 3, 64, 64, 64, torch.bfloat16),       # one segment per (b, h)
    (1, 1, 1024, 64, 64, torch.bfloat16),     # 16 segments, one (b, h)
    (1, 2, 576, 64, 192, torch.float32),
    (1, 1, 96, 128, 1, torch.float32),        # every token its own segment
    (1, 1, 130, 128, 65, torch.float32),
]


@pytest.mark.parametrize("B,H,L,d,N,dtype", CASES)
def test_small_shapes(cuda_ok, B, H, L, d, N, dtype):
    q, k, v, beta, _, _ = inputs(B, H, L, d, dtype, seed=7 + L + d + N)
    ref = run_oracle(q, k, v, beta, N)
    kind = "f32" if dtype == torch.float32 else "bf16"
    for path in paths_for(q, N):
        assert_close(run_gpu(q, k, v, beta, N, path=path), ref, kind, "case %s path %d" % ((B, H, L, d, N), path))


@pytest.mark.parametrize("dtype,d,N", [(torch.bfloat16, 128, 256), (torch.float32, 64, 64), (torch.bfloat16, 64, 64)])
def test_incoming_state_and_in_place(cuda_ok, dtype, d, N):
    q, k, v, beta, M, z = inputs(1, 2, 4 * N, d, dtype, seed=99, state=True)
    ref = run_oracle(q, k, v, beta, N, M, z)
    kind = "f32" if dtype == torch.float32 else "bf16"
    for path in paths_for(q, N):
        assert_close(run_gpu(q, k, v, beta, N, M, z, path=path), ref, kind, "state path %d" % path)
        Mi, zi = M.clone(), z.clone()
        got = run_gpu(q, k, v, beta, N, Mi, zi, path=path, inplace=True)
        assert got[1].data_ptr() == Mi.data_ptr()
        assert_close(got, ref, kind, "in-place path %d" % path)


@pytest.mark.parametrize("dtype,d,N", [(torch.bfloat16, 128, 256), (torch.float32, 64, 32), (torch.bfloat16, 64, 64)])
def test_gate_limits(cuda_ok, dtype, d, N):
    """beta = -inf: pure local attention; beta = +inf: pure memory retrieval
    (segment 0 from the zero state is then exactly 0)."""
    q, k, v, _, _, _ = inputs(1, 2, 3 * N, d, dtype, seed=5)
    kind = "f32" if dtype == torch.float32 else "bf16"
    for val in (-math.inf, math.inf):
        beta = torch.full((2,), val, dtype=torch.float32, device=DEV)
        ref = run_oracle(q, k, v, beta, N)
        for path in paths_for(q, N):
            got = run_gpu(q, k, v, beta, N, path=path)
            assert_close(got, ref, kind, "beta=%s path %d" % (val, path))
            if val > 0:
                assert torch.count_nonzero(got[0][:, :, :N]) == 0


def test_streaming_calls_match_one_call_on_gpu(cuda_ok):
    q, k, v, beta, _, _ = inputs(1, 2, 2048, 128, torch.bfloat16, seed=17)
    N = 256
    for path in paths_for(q, N):
        o1, M1, z1 = run_gpu(q, k, v, beta, N, path=path)
        M = z = None
        parts = []
        for c in range(4):
            sl = slice(c * 512, (c + 1) * 512)
            o, M, z = run_gpu(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(), v[:, :, sl].contiguous(),
                              beta, N, M, z, path=path)
            parts.append(o)
        o4 = torch.cat(parts, dim=2)
        assert slice_err(o4.float().cpu().numpy(), o1.double().cpu().numpy()) < 1e-2
        assert slice_err(M.cpu().numpy(), M1.double().cpu().numpy()) < 1e-5
        assert slice_err(z.cpu().numpy(), z1.double().cpu().numpy()) < 1e-5


def test_repeat_calls_are_deterministic(cuda_ok):
    q, k, v, beta, _, _ = inputs(1, 2, 1024, 128, torch.bfloat16, seed=23)
    for path in paths_for(q, 256):
        a = run_gpu(q, k, v, beta, 256, path=path)
        b = run_gpu(q, k, v, beta, 256, path=path)
        for x, y in zip(a, b):
            assert torch.equal(x, y)


def test_allocating_entry_point(cuda_ok):
    q, k, v, beta, _, _ = inputs(1, 2, 512, 128, torch.bfloat16, seed=31)
    B, H, L, d = q.shape
    out = torch.empty_like(q)
    M = torch.empty((B, H, d, d), device=DEV)
    z = torch.empty((B, H, d), device=DEV)
    rc = bd.infini_attn_forward(bd.shape_of(q), q, k, v, beta, None, None, 128, out, M, z, None)
    assert rc == 0
    ref = run_oracle(q, k, v, beta, 128)
    assert_close((out, M, z), ref, "bf16", "allocating entry point")


def test_tc_state_is_split_precision(cuda_ok):
    """The tensor-core state kernel feeds sigma(K) to bf16 MMAs as hi + lo
    parts, so M and z come out near fp32 accuracy (the bf16 tolerance above is
    for a single bf16 rounding of sigma(K))."""
    q, k, v, beta, _, _ = inputs(1, 2, 8 * 256, 128, torch.bfloat16, seed=41)
    ref = run_oracle(q, k, v, beta, 256)
    out, M, z = run_gpu(q, k, v, beta, 256, path=bd.INFINI_PATH_TC)
    eM = slice_err(M.cpu().numpy(), ref[1])
    ez = slice_err(z.cpu().numpy(), ref[2])
    assert eM <= 2e-5 and ez <= 2e-5, (eM, ez)


# --------------------------------------------------------------- many units per CTA, every element

# Shapes whose tensor-core attention launch gives every persistent CTA several
# work units, so the pipeline across units (the Q buffers, the O / retrieval
# hand-off, the schedule's segment groups, units short enough that a slot
# finishes one before the previous one's retrieval) runs here element by
# element, not only in the sampled full-size workloads below.
@pytest.mark.parametrize("B,H,L,N,state", [
    (1, 8, 8192, 2048, False),   # 256 units of 2 query tiles
    (2, 4, 4096, 1024, True),
    (4, 8, 4096, 1024, True),    # 512 units: ~3.5 per CTA, every pair length of a 1024-token segment
    (2, 8, 8192, 256, False),    # 512 units, all with the shortest tiles (2 and 4 key tiles of 64)
])
def test_many_units_per_cta_every_element(cuda_ok, B, H, L, N, state):
    q, k, v, beta, M, z = inputs(B, H, L, 128, torch.bfloat16, seed=57 + N, state=state)
    ref = run_oracle(q, k, v, beta, N, M, z)
    got = run_gpu(q, k, v, beta, N, M, z, path=bd.INFINI_PATH_TC)
    assert_close(got, ref, "bf16", "many units B%d H%d L%d N%d" % (B, H, L, N))


# --------------------------------------------------------------- full-size workloads (sampled)

def _full_workload(name, segments, head_subset=None):
    w = synth.WORKLOADS[name]
    q, k, v = synth.make_qkv(w, DEV)
    beta = synth.make_beta(w, DEV)
    N = w.N
    # GPU: the sequence in `calls` streamed calls, on the path AUTO selects.
    per = w.L // w.calls
    M = z = None
    outs = []
    for c in range(w.calls):
        sl = slice(c * per, (c + 1) * per)
        qs, ks, vs = (t[:, :, sl].contiguous() if w.calls > 1 else t for t in (q, k, v))
        o, M, z = run_gpu(qs, ks, vs, beta, N, M, z)
        outs.append(o)
    out = torch.cat(outs, dim=2) if w.calls > 1 else outs[0]
    if head_subset is not None:
        bsel, hsel = head_subset
        q, k, v = (t[bsel][:, hsel].contiguous() for t in (q, k, v))
        out, M, z = out[bsel][:, hsel], M[bsel][:, hsel], z[bsel][:, hsel]
        beta = beta[hsel]
    ro, rM, rz = run_oracle(q, k, v, beta, N, segments=segments)
    B, H = q.shape[:2]
    got = out.view(B, H, w.S, N, w.d)[:, :, segments]
    tol = TOL["bf16"]
    xo, xM, xz = got.float().cpu().numpy(), M.cpu().numpy(), z.cpu().numpy()
    eo, eM, ez = slice_err(xo, ro), slice_err(xM, rM), slice_err(xz, rz)
    record(name + " (sampled)", (eo, eM, ez), (elem_err(xo, ro), elem_err(xM, rM), elem_err(xz, rz)))
    assert eo <= tol["out"] and eM <= tol["M"] and ez <= tol["z"], (name, eo, eM, ez)


@pytest.mark.slow
def test_llama8b_32k_streamed(cuda_ok):
    _full_workload("llama8b_32k_bf16", [0, 3, 4, 9, 15], head_subset=([0], list(range(0, 32, 4))))


@pytest.mark.slow
def test_mid_8k_outlier_keys(cuda_ok):
    _full_workload("mid_8k_outlier_bf16", [0, 1, 7], head_subset=([0, 9, 15], [0, 5, 11, 15]))


@pytest.mark.slow
def test_stream_1m(cuda_ok):
    _full_workload("stream_1m_bf16", [0, 1, 255, 511], head_subset=([0], [0, 3, 7]))
