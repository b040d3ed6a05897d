"""GPU parity of the decode step (through the C ABI): every step against the
oracle's decode step fed the same inputs (the GPU's cache rows and fp32
state), the fold at each segment end against the oracle's fold, and a whole
sequence decoded token by token against the forward."""
import numpy as np
import pytest
import torch

import oracle
from compressive_memory_segment_b200 import binding as bd
from compressive_memory_segment_b200 import synth
from tests.parity import TOL, host_bits, run_gpu, run_oracle, slice_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _seq(B, H, N, S, d, dtype, seed, beta="normal"):
    w = synth.Workload("dec", B, H, d, N, S, "f32" if dtype == torch.float32 else "bf16", seed, beta=beta)
    q, k, v = synth.make_qkv(w, DEV)
    return w, q, k, v, synth.make_beta(w, DEV)


def _err(x, ref):
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-30))


@pytest.mark.parametrize("B,H,N,S,d,dtype", [
    (2, 3, 5, 3, 64, torch.float32),
    (1, 2, 33, 2, 128, torch.float32),
    (2, 2, 40, 2, 64, torch.bfloat16),
    (1, 2, 128, 2, 128, torch.bfloat16),   # the fold runs on the tensor-core state kernel
])
def test_decode_steps_match_oracle(cuda_ok, B, H, N, S, d, dtype):
    kind = "f32" if dtype == torch.float32 else "bf16"
    w, q, k, v, beta = _seq(B, H, N, S, d, dtype, seed=90 + N)
    kc = torch.zeros((B, H, N, d), dtype=dtype, device=DEV)
    vc = torch.zeros_like(kc)
    M = torch.zeros((B, H, d, d), device=DEV)
    z = torch.zeros((B, H, d), device=DEV)
    beta_h = beta.double().cpu().numpy()
    worst_out = worst_state = 0.0
    for t in range(N * S):
        pos = t % N
        qt, kt, vt = (x[:, :, t].contiguous() for x in (q, k, v))
        M_before = M.double().cpu().numpy()
        z_before = z.double().cpu().numpy()
        kc_before, vc_before = host_bits(kc), host_bits(vc)
        out = bd.decode_step(qt, kt, vt, beta, kc, vc, pos, M, z)
        torch.cuda.synchronize()
        ro, rM, rz = oracle.decode_step(host_bits(qt), host_bits(kt), host_bits(vt), kc_before, vc_before, pos,
                                        beta_h, M_before, z_before)
        worst_out = max(worst_out, _err(out.float().cpu().numpy(), ro))
        # The cache row was written from this token's key and value.
        assert torch.equal(kc[:, :, pos], kt) and torch.equal(vc[:, :, pos], vt)
        if pos == N - 1:
            worst_state = max(worst_state, _err(M.cpu().numpy(), rM), _err(z.cpu().numpy(), rz))
        else:
            assert np.array_equal(M.double().cpu().numpy(), M_before)
    tol = TOL[kind]
    assert worst_out <= tol["out"], worst_out
    assert worst_state <= tol["M"], worst_state
    assert bd.infini_attn_device_status(None) == bd.INFINI_OK


@pytest.mark.parametrize("N,d,dtype", [(64, 64, torch.float32), (128, 128, torch.bfloat16)])
def test_decode_sequence_matches_forward(cuda_ok, N, d, dtype):
    """Token-by-token decoding of 3 segments (with an incoming state) gives the
    forward's outputs and final state, both against the oracle and against the
    GPU forward."""
    kind = "f32" if dtype == torch.float32 else "bf16"
    B, H, S = 1, 2, 3
    w, q, k, v, beta = _seq(B, H, N, S, d, dtype, seed=7 + d)
    M0, z0 = synth.make_state(w, DEV, scale=2.0)
    M, z = M0.clone(), z0.clone()
    kc = torch.empty((B, H, N, d), dtype=dtype, device=DEV)
    vc = torch.empty_like(kc)
    outs = []
    for t in range(N * S):
        outs.append(bd.decode_step(q[:, :, t].contiguous(), k[:, :, t].contiguous(), v[:, :, t].contiguous(), beta,
                                   kc, vc, t % N, M, z))
    out = torch.stack(outs, dim=2)
    ref = run_oracle(q, k, v, beta, N, M0, z0)
    tol = TOL[kind]
    assert slice_err(out.float().cpu().numpy(), ref[0]) <= tol["out"]
    assert slice_err(M.cpu().numpy(), ref[1]) <= tol["M"] and slice_err(z.cpu().numpy(), ref[2]) <= tol["z"]
    fo, fM, fz = run_gpu(q, k, v, beta, N, M0, z0)
    assert float((out.float() - fo.float()).abs().max()) <= 2 * tol["out"] * float(fo.float().abs().max())
