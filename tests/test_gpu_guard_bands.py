"""Guard bands: every buffer the library writes (out, M_out, z_out, the
workspace; for the decode step also the caches and M, z) sits inside a larger
allocation whose bytes outside the buffer hold a sentinel, and after the call
the sentinel must be intact. This stands in for a memory checker, which this
environment does not provide: a kernel whose index arithmetic is off for
small or odd shapes (one segment, two segments, one (b, h), a ragged last
tile, an odd number of 64-token segments, an output that is only 16-byte
aligned) writes into a band and fails here. The results are also compared
with the CPU oracle, so the calls did real work.
"""
import numpy as np
import pytest
import torch

from compressive_memory_segment_b200 import binding as bd
from compressive_memory_segment_b200 import synth
from tests.parity import TOL, assert_close, host_bits, run_oracle

pytestmark = pytest.mark.gpu

DEV = "cuda"
SENTINEL = 0xA5
BAND = 4096  # bytes on each side


class Guarded:
    """A tensor of `shape` and `dtype` inside a sentinel-filled byte buffer.
    `skew` shifts the tensor by that many bytes (16 keeps 16-byte alignment
    while breaking 32-byte alignment)."""

    def __init__(self, shape, dtype, skew=0, fill=None):
        nbytes = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        self.lo = BAND + skew
        self.nbytes = nbytes
        self.raw = torch.full((BAND + skew + nbytes + BAND,), SENTINEL, dtype=torch.uint8, device=DEV)
        self.t = self.raw[self.lo:self.lo + nbytes].view(dtype).view(shape)
        if fill is not None:
            self.t.copy_(fill)

    def intact(self):
        raw = self.raw.cpu().numpy()
        return bool((raw[:self.lo] == SENTINEL).all() and (raw[self.lo + self.nbytes:] == SENTINEL).all())


def _inputs(B, H, L, d, dtype, seed, state):
    w = synth.Workload("guard", B, H, d, L, 1, dtype, seed, beta="normal")
    q, k, v = synth.make_qkv(w, DEV)
    beta = synth.make_beta(w, DEV)
    M = z = None
    if state:
        M, z = synth.make_state(w, DEV, scale=2.0)
    return q, k, v, beta, M, z


CASES = [
    # B, H, L, d, N, dtype, incoming state
    (1, 1, 128, 128, 128, "bf16", False),   # one segment, one (b, h)
    (1, 1, 256, 128, 128, "bf16", True),    # two segments
    (1, 2, 512, 128, 256, "bf16", False),   # paired-tile kernel, S = 2
    (2, 1, 768, 128, 384, "bf16", True),    # single-tile kernel (odd tile count)
    (1, 1, 192, 64, 64, "bf16", False),     # d = 64, three 64-token segments
    (1, 1, 64, 64, 64, "bf16", True),       # d = 64, one segment
    (1, 2, 200, 128, 100, "bf16", False),   # CUDA-core path, ragged tile
    (1, 1, 65, 64, 65, "f32", True),        # fp32, one odd segment
]


@pytest.mark.parametrize("B,H,L,d,N,dt,state", CASES)
@pytest.mark.parametrize("skew", [0, 16])
def test_forward_writes_stay_inside_their_buffers(cuda_ok, B, H, L, d, N, dt, state, skew):
    q, k, v, beta, M, z = _inputs(B, H, L, d, dt, seed=300 + L + d + N, state=state)
    torch_dt = torch.float32 if dt == "f32" else torch.bfloat16
    out = Guarded((B, H, L, d), torch_dt, skew=skew)
    Mo = Guarded((B, H, d, d), torch.float32, skew=skew)
    zo = Guarded((B, H, d), torch.float32, skew=skew)
    ws_bytes = bd.infini_attn_workspace_size(bd.shape_of(q), N)
    ws = Guarded((ws_bytes,), torch.uint8)  # the workspace must stay 256-byte aligned
    rc = bd.infini_attn_forward_ws(bd.shape_of(q), q, k, v, beta, M, z, N, out.t, Mo.t, zo.t, ws.t, ws_bytes,
                                   bd.INFINI_PATH_AUTO, None)
    assert rc == bd.INFINI_OK, bd.infini_attn_strerror(rc)
    assert bd.infini_attn_device_status(None) == bd.INFINI_OK
    for name, g in (("out", out), ("M_out", Mo), ("z_out", zo), ("workspace", ws)):
        assert g.intact(), "write outside %s" % name
    ref = run_oracle(q, k, v, beta, N, M, z)
    assert_close((out.t, Mo.t, zo.t), ref, dt, "guarded %s skew %d" % ((B, H, L, d, N, dt), skew))


@pytest.mark.parametrize("B,H,N,d,dt", [(1, 1, 64, 64, "bf16"), (2, 1, 128, 128, "bf16"), (1, 2, 33, 64, "f32")])
def test_decode_writes_stay_inside_their_buffers(cuda_ok, B, H, N, d, dt):
    torch_dt = torch.float32 if dt == "f32" else torch.bfloat16
    q, k, v, beta, _, _ = _inputs(B, H, N, d, dt, seed=77 + N, state=False)
    kc = Guarded((B, H, N, d), torch_dt, fill=torch.zeros((B, H, N, d), dtype=torch_dt))
    vc = Guarded((B, H, N, d), torch_dt, fill=torch.zeros((B, H, N, d), dtype=torch_dt))
    M = Guarded((B, H, d, d), torch.float32, fill=torch.zeros((B, H, d, d)))
    z = Guarded((B, H, d), torch.float32, fill=torch.zeros((B, H, d)))
    shp = bd.make_shape(B, H, N, d, bd.INFINI_F32 if dt == "f32" else bd.INFINI_BF16)
    ws_bytes = bd.infini_attn_decode_workspace_size(shp)
    ws = Guarded((ws_bytes,), torch.uint8)
    for t in range(N):  # a whole segment, so the last step folds it into (M, z)
        out = Guarded((B, H, d), torch_dt)
        qt, kt, vt = (x[:, :, t].contiguous() for x in (q, k, v))
        rc = bd.infini_attn_decode_step(shp, qt, kt, vt, beta, kc.t, vc.t, t, M.t, z.t, out.t, ws.t, ws_bytes, None)
        assert rc == bd.INFINI_OK, bd.infini_attn_strerror(rc)
        assert out.intact(), "write outside out at position %d" % t
    assert bd.infini_attn_device_status(None) == bd.INFINI_OK
    for name, g in (("k_cache", kc), ("v_cache", vc), ("M", M), ("z", z), ("workspace", ws)):
        assert g.intact(), "write outside %s" % name
    # The fold left (M, z) equal to the forward's final state of the segment.
    ref = run_oracle(q, k, v, beta, N)
    tol = TOL[dt]
    eM = float(np.max(np.abs(M.t.cpu().numpy() - ref[1])) / np.max(np.abs(ref[1])))
    assert eM <= tol["M"], eM
