"""The forward split into blocks of consecutive segments, through the library's
phase entry points (state, exclusive sum of the block totals, finish), run
block after block on one GPU: the concatenated outputs and the final state
must match the oracle on the whole sequence and the single-call forward. This
is the decomposition the sequence-sharded multi-GPU mode runs, minus the
all-gather (covered by the gloo test on CPU)."""
import pytest
import torch

from compressive_memory_segment_b200 import binding as bd
from compressive_memory_segment_b200 import sharded, synth
from tests.parity import TOL, assert_close, run_gpu, run_oracle, slice_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("B,H,d,N,S,parts,dtype", [
    (1, 2, 128, 256, 8, 2, torch.bfloat16),   # tensor-core path
    (1, 2, 128, 128, 8, 4, torch.bfloat16),
    (2, 1, 64, 64, 6, 3, torch.float32),      # CUDA-core path
    (2, 3, 64, 64, 10, 2, torch.bfloat16),    # d = 64: the phases run the three-kernel tensor-core path,
                                              # the single call the single-pass kernel
    (1, 2, 64, 64, 7, 1, torch.bfloat16),     # an odd number of segments in one block
])
def test_blocks_match_whole_sequence(cuda_ok, B, H, d, N, S, parts, dtype):
    kind = "f32" if dtype == torch.float32 else "bf16"
    w = synth.Workload("blocks", B, H, d, N, S, kind, 123 + parts, beta="normal")
    q, k, v = synth.make_qkv(w, DEV)
    beta = synth.make_beta(w, DEV)
    M0, z0 = synth.make_state(w, DEV, scale=2.0)
    L = N * S
    blk = L // parts
    blocks = [tuple(t[:, :, r * blk:(r + 1) * blk].contiguous() for t in (q, k, v)) for r in range(parts)]
    outs, M, z = sharded.forward_blocks_one_device(blocks, beta, N, M0, z0)
    out = torch.cat(outs, dim=2)
    ref = run_oracle(q, k, v, beta, N, M0, z0)
    assert_close((out, M, z), ref, kind, "blocks=%d" % parts)
    fo, fM, fz = run_gpu(q, k, v, beta, N, M0, z0)
    tol = TOL[kind]
    assert float((out.float() - fo.float()).abs().max()) <= tol["out"] * float(fo.float().abs().max())
    assert slice_err(M.cpu().numpy(), fM.double().cpu().numpy()) <= 1e-5


def test_state_then_finish_equals_forward(cuda_ok):
    """One block: phase 1 then phase 3 with the caller's state is the forward."""
    w = synth.Workload("phases", 1, 2, 128, 256, 4, "bf16", 9, beta="normal")
    q, k, v = synth.make_qkv(w, DEV)
    beta = synth.make_beta(w, DEV)
    M0, z0 = synth.make_state(w, DEV)
    ph = sharded.CudaPhases()
    ws = ph.workspace(q, w.N)
    M_tot, z_tot = ph.state(k, v, w.N, ws)
    out, M, z = ph.finish(q, k, v, beta, M0, z0, w.N, ws)
    fo, fM, fz = run_gpu(q, k, v, beta, w.N, M0, z0)
    assert torch.equal(out, fo)
    assert torch.equal(M, fM) and torch.equal(z, fz)
    assert torch.allclose(M, M0 + M_tot, rtol=1e-5, atol=1e-3)
