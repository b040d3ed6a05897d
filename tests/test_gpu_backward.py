"""GPU parity of the backward (through the C ABI) against the oracle's
backward (itself pinned by finite differences of the forward): every gradient
element on small cases spanning several tiles, segments and a ragged tail,
both dtypes, d in {64, 128}, with and without incoming state and output-state
gradient, and saturated gates."""
import numpy as np
import pytest
import torch

import oracle
from compressive_memory_segment_b200 import binding as bd
from compressive_memory_segment_b200 import synth
from tests.parity import host_bits, slice_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
# fp32 I/O: the gradients are fp32 sums of fp32 products; bf16 I/O: the same
# arithmetic on bf16 inputs (the oracle widens the same bits), so the bound is
# the fp32 one with headroom for the longer sums.
TOL = {"f32": 2e-4, "bf16": 2e-3}


def _case(B, H, d, N, S, dtype, seed, state, beta="normal"):
    kind = "f32" if dtype == torch.float32 else "bf16"
    w = synth.Workload("bwd", B, H, d, N, S, kind, seed, beta=beta)
    q, k, v = synth.make_qkv(w, DEV)
    b = synth.make_beta(w, DEV)
    g = torch.Generator(device="cpu").manual_seed(seed)
    dout = torch.randn((B, H, N * S, d), generator=g).to(dtype).to(DEV)
    M = z = dM = dz = None
    if state:
        M, z = synth.make_state(w, DEV, scale=2.0)
        dM = torch.randn((B, H, d, d), generator=g).to(DEV)
        dz = torch.randn((B, H, d), generator=g).to(DEV)
    return kind, q, k, v, b, dout, M, z, dM, dz


def _np(x):
    return None if x is None else x.detach().double().cpu().numpy()


@pytest.mark.parametrize("B,H,d,N,S,dtype,state", [
    (1, 2, 64, 32, 3, torch.float32, False),
    (1, 1, 64, 45, 2, torch.float32, True),     # ragged tail (45 = 32 + 13)
    (2, 2, 128, 64, 3, torch.float32, True),
    (1, 2, 128, 100, 2, torch.bfloat16, True),
    (1, 1, 64, 1, 5, torch.float32, True),       # one-token segments
])
def test_backward_matches_oracle(cuda_ok, B, H, d, N, S, dtype, state):
    kind, q, k, v, beta, dout, M, z, dM, dz = _case(B, H, d, N, S, dtype, 300 + N, state)
    got = bd.backward(q, k, v, beta, N, dout, M, z, dM, dz)
    torch.cuda.synchronize()
    ref = oracle.backward(host_bits(q), host_bits(k), host_bits(v), _np(beta), host_bits(dout).astype(np.float64)
                          if dtype == torch.float32 else _np(dout), _np(M), _np(z), _np(dM), _np(dz), seg_len=N)
    names = ["dq", "dk", "dv", "dbeta", "dM_in", "dz_in"]
    for name, g_, r_ in zip(names, got, ref):
        gn = g_.double().cpu().numpy()
        if name == "dbeta":
            err = float(np.max(np.abs(gn - r_)) / max(np.max(np.abs(r_)), 1e-30))
        else:
            err = slice_err(gn, r_)
        assert err <= TOL[kind], (name, err)
    assert bd.infini_attn_device_status(None) == bd.INFINI_OK


# The tensor-core backward (bf16, d = 128, seg_len % 128 == 0) rounds the MMA
# operands P, dS, sigma(K), G_s, dnum and M_{s-1} to bf16 (relative error
# <= 2^-9 each) and accumulates in fp32; the bound allows for the sums of up
# to seg_len such products against the slice maximum.
TOL_TC = 2e-2


def _oracle_bwd(q, k, v, beta, dout, M, z, dM, dz, N):
    return oracle.backward(host_bits(q), host_bits(k), host_bits(v), _np(beta), _np(dout), _np(M), _np(z), _np(dM),
                           _np(dz), seg_len=N)


@pytest.mark.parametrize("B,H,d,N,S,state", [
    (1, 2, 128, 128, 3, True),     # one tile per segment
    (1, 1, 128, 256, 2, True),     # two tiles: a full tile below the diagonal one
    (2, 1, 128, 384, 2, False),    # three tiles, no incoming state
    (1, 2, 128, 512, 3, True),     # four tiles, 24 CTAs per kernel
    (1, 2, 64, 64, 4, True),       # d = 64: two pairs of 64-token segments per head
    (2, 3, 64, 64, 2, False),      # one pair per head, no incoming state
    (1, 1, 64, 64, 16, True),      # the reproduction shape's 16 segments
])
def test_backward_tc_matches_oracle(cuda_ok, B, H, d, N, S, state):
    kind, q, k, v, beta, dout, M, z, dM, dz = _case(B, H, d, N, S, torch.bfloat16, 700 + N + d, state)
    got = bd.backward(q, k, v, beta, N, dout, M, z, dM, dz, path=bd.INFINI_PATH_TC)
    torch.cuda.synchronize()
    assert bd.infini_attn_device_status(None) == bd.INFINI_OK
    ref = _oracle_bwd(q, k, v, beta, dout, M, z, dM, dz, N)
    errs = {}
    for name, g_, r_ in zip(["dq", "dk", "dv", "dbeta", "dM_in", "dz_in"], got, ref):
        gn = g_.double().cpu().numpy()
        if name == "dbeta":
            errs[name] = float(np.max(np.abs(gn - r_)) / max(np.max(np.abs(r_)), 1e-30))
        else:
            errs[name] = slice_err(gn, r_)
    print("tc backward errors", (B, H, d, N, S, state), {n: "%.2e" % e for n, e in errs.items()})
    for name, e in errs.items():
        assert e <= TOL_TC, (name, e)


@pytest.mark.parametrize("B,H,d,N,S,heads", [
    (2, 8, 128, 1024, 2, [(0, 0), (1, 5)]),    # 256 CTAs per backward kernel: several waves
    (4, 12, 64, 64, 16, [(0, 3), (3, 11)]),    # 384 pair CTAs
])
def test_backward_tc_many_ctas(cuda_ok, B, H, d, N, S, heads):
    """The tensor-core backward on grids of more CTAs than SMs: sampled heads
    element by element against the oracle (heads are independent, so a head's
    slice is the oracle's whole problem), every head against the CUDA-core
    backward."""
    kind, q, k, v, beta, dout, M, z, dM, dz = _case(B, H, d, N, S, torch.bfloat16, 900 + d, True)
    got = bd.backward(q, k, v, beta, N, dout, M, z, dM, dz, path=bd.INFINI_PATH_TC)
    simt = bd.backward(q, k, v, beta, N, dout, M, z, dM, dz, path=bd.INFINI_PATH_SIMT)
    torch.cuda.synchronize()
    assert bd.infini_attn_device_status(None) == bd.INFINI_OK
    for name, g_, s_ in zip(["dq", "dk", "dv", "dM_in", "dz_in"], got[:3] + got[4:], simt[:3] + simt[4:]):
        e = slice_err(g_.double().cpu().numpy(), s_.double().cpu().numpy())
        assert e <= TOL_TC, (name, e)
    for b, h in heads:
        sl = lambda x: None if x is None else x[b:b + 1, h:h + 1]
        ref = _oracle_bwd(sl(q), sl(k), sl(v), beta[h:h + 1], sl(dout), sl(M), sl(z), sl(dM), sl(dz), N)
        for name, g_, r_ in zip(["dq", "dk", "dv"], got[:3], ref[:3]):
            e = slice_err(g_[b:b + 1, h:h + 1].double().cpu().numpy(), r_)
            assert e <= TOL_TC, (b, h, name, e)
        for name, g_, r_ in zip(["dM_in", "dz_in"], got[4:], ref[4:]):
            e = slice_err(g_[b:b + 1, h:h + 1].double().cpu().numpy(), r_)
            assert e <= TOL_TC, (b, h, name, e)


@pytest.mark.parametrize("name,heads", [
    ("mid_8k_outlier_bf16", [(0, 0), (15, 11)]),   # 16 x 16 heads of 8 segments of 1024: 16,384 CTAs per kernel
    ("hf_repro_bf16", [(0, 0), (7, 11)]),           # 8 x 12 heads of 16 segments of 64: 768 pair CTAs
])
def test_backward_tc_full_size_sampled(cuda_ok, name, heads):
    """The backward on the exact workloads bench.py times (same seeded inputs
    and dout), on the default path: two heads element by element against the
    oracle, every head against the CUDA-core backward."""
    w = synth.WORKLOADS[name]
    q, k, v = synth.make_qkv(w, DEV)
    beta = synth.make_beta(w, DEV)
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    dout = torch.randn(q.shape, generator=g).to(q.dtype).to(DEV)
    got = bd.backward(q, k, v, beta, w.N, dout)
    simt = bd.backward(q, k, v, beta, w.N, dout, path=bd.INFINI_PATH_SIMT)
    torch.cuda.synchronize()
    assert bd.infini_attn_device_status(None) == bd.INFINI_OK
    for nm, g_, s_ in zip(["dq", "dk", "dv", "dM_in", "dz_in"], got[:3] + got[4:], simt[:3] + simt[4:]):
        e = slice_err(g_.double().cpu().numpy(), s_.double().cpu().numpy())
        assert e <= TOL_TC, (nm, e)
    for b, h in heads:
        sl = lambda x: x[b:b + 1, h:h + 1]
        ref = _oracle_bwd(sl(q), sl(k), sl(v), beta[h:h + 1], sl(dout), None, None, None, None, w.N)
        for nm, g_, r_ in zip(["dq", "dk", "dv", "dM_in", "dz_in"], got[:3] + got[4:], ref[:3] + ref[4:]):
            e = slice_err(g_[b:b + 1, h:h + 1].double().cpu().numpy(), r_)
            assert e <= TOL_TC, (b, h, nm, e)


@pytest.mark.parametrize("d,N,S", [(128, 256, 2), (64, 64, 4)])
def test_backward_tc_is_the_default_and_deterministic(cuda_ok, d, N, S):
    """AUTO takes the tensor-core backward for bf16 with d = 128 and
    N % 128 == 0, and with d = 64, N = 64 and an even segment count; dq, dk
    and dv are the same bits on every call. (With one query tile per segment,
    as here, one CTA adds into G[s]; with several, dk takes their shares in
    arrival order and may differ in the last bits.)"""
    kind, q, k, v, beta, dout, M, z, dM, dz = _case(1, 2, d, N, S, torch.bfloat16, 77, True)
    a = bd.backward(q, k, v, beta, N, dout, M, z, dM, dz)
    b = bd.backward(q, k, v, beta, N, dout, M, z, dM, dz, path=bd.INFINI_PATH_TC)
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)
    torch.testing.assert_close(a[3], b[3], rtol=1e-5, atol=1e-7)


@pytest.mark.parametrize("d,N,S", [(128, 128, 3), (64, 64, 4)])
def test_backward_tc_saturated_gates(cuda_ok, d, N, S):
    """beta = +-inf on the tensor-core backward: dbeta = 0, and with g = 1 the
    local attention passes no gradient (g = 0: the retrieval none)."""
    kind, q, k, v, beta, dout, M, z, dM, dz = _case(1, 2, d, N, S, torch.bfloat16, 9, True)
    beta = torch.tensor([float("inf"), float("-inf")], device=DEV)
    got = bd.backward(q, k, v, beta, N, dout, M, z, dM, dz, path=bd.INFINI_PATH_TC)
    ref = _oracle_bwd(q, k, v, beta, dout, M, z, dM, dz, N)
    assert torch.all(got[3] == 0)
    for g_, r_ in zip(got[:3], ref[:3]):
        assert slice_err(g_.double().cpu().numpy(), r_) <= TOL_TC


def test_backward_saturated_gates(cuda_ok):
    """beta = +-inf: dbeta = 0 and one branch carries no gradient."""
    kind, q, k, v, beta, dout, M, z, dM, dz = _case(1, 2, 64, 32, 3, torch.float32, 5, True)
    beta = torch.tensor([float("inf"), float("-inf")], device=DEV)
    got = bd.backward(q, k, v, beta, 32, dout, M, z, dM, dz)
    ref = oracle.backward(host_bits(q), host_bits(k), host_bits(v), _np(beta), _np(dout), _np(M), _np(z), _np(dM),
                          _np(dz), seg_len=32)
    assert torch.all(got[3] == 0)
    for g_, r_ in zip(got[:3], ref[:3]):
        assert slice_err(g_.double().cpu().numpy(), r_) <= TOL[kind]
