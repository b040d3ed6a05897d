"""Failure detection on the GPU without a GPU fault: every device-side wait of
the library is bounded. A self-test kernel waits on an mbarrier that nothing
arrives on; the wait must give up after its limit, the host must read
INFINI_ERR_TIMEOUT from the device status word, and the CUDA context must stay
usable (a forward right after it is still correct)."""
import pytest
import torch

from compressive_memory_segment_b200 import binding as bd
from compressive_memory_segment_b200 import synth
from tests.parity import assert_close, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(cuda_ok):
    stream = torch.cuda.current_stream()
    assert bd.infini_attn_device_status(stream) == bd.INFINI_OK
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    assert bd.infini_attn_selftest_timeout(2_000_000, stream) == bd.INFINI_OK  # 2 ms
    ev1.record(stream)
    assert bd.infini_attn_device_status(stream) == bd.INFINI_ERR_TIMEOUT
    assert bd.infini_attn_device_status(stream) == bd.INFINI_OK  # read-and-clear
    # The wait lasted about its limit (it polls the global timer), not forever.
    ms = ev0.elapsed_time(ev1)
    assert 1.5 <= ms < 1000.0, ms
    # The context still runs the layer, on both paths.
    w = synth.Workload("after_timeout", 1, 2, 128, 256, 2, "bf16", 77, beta="normal")
    q, k, v = synth.make_qkv(w, "cuda")
    beta = synth.make_beta(w, "cuda")
    ref = run_oracle(q, k, v, beta, w.N)
    for path in (bd.INFINI_PATH_SIMT, bd.INFINI_PATH_TC):
        assert_close(run_gpu(q, k, v, beta, w.N, path=path), ref, "bf16", "after timeout, path %d" % path)
    assert bd.infini_attn_device_status(stream) == bd.INFINI_OK
