"""The multi-rank host logic of bench.py on CPU: two gloo ranks, launched the
way torchrun would (RANK / WORLD_SIZE / MASTER_ADDR=127.0.0.1 in the
environment). Each rank runs its own replica of the workload, the step time is
the max over ranks and the job throughput counts every rank's tokens; the
reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, results):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import bench
    dist = bench.init_dist("gloo", timeout_s=60)
    assert dist is not None and dist.get_world_size() == world
    # Rank r "measured" a step time of 10 + r ms; everyone reports the slowest.
    ms = bench.max_over_ranks(10.0 + rank, dist, torch.device("cpu"))
    tok = bench.job_tokens_per_s(world, 1 << 20, ms)
    # Replicas: every rank builds the same seeded inputs (weak scaling, no
    # collective on the data path); check that by comparing a checksum.
    from compressive_memory_segment_b200 import synth
    w = synth.WORKLOADS["tiny_f32"]
    q, k, v = synth.make_qkv(w, "cpu")
    cs = torch.tensor([float(q.double().sum() + 2 * k.double().sum() + 3 * v.double().sum())], dtype=torch.float64)
    all_cs = [torch.zeros_like(cs) for _ in range(world)]
    dist.all_gather(all_cs, cs)
    # The reference arm: ranks other than 0 return at once without work.
    class A:
        steps, warmup, gpus = 1, 3, world
    ref_rc = bench.reference_arm(A, w) if rank != 0 else 0
    results[rank] = (ms, tok, [float(x) for x in all_cs], ref_rc)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        results = m.dict()
        ctx = mp.get_context("spawn")
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(150)
        for p in procs:
            if p.is_alive():
                p.kill()
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(results)
    assert sorted(res) == [0, 1]
    for r in range(world):
        ms, tok, all_cs, ref_rc = res[r]
        assert ms == 11.0                                  # max over ranks
        assert tok == pytest.approx(world * (1 << 20) / 0.011)
        assert all_cs[0] == all_cs[1]                       # identical replicas
        assert ref_rc == 0


# ------------------------------------------------------------------ sequence-sharded forward

class _NumpyPhases:
    """Stand-in for the library's three phases on CPU, so the orchestration
    (all-gather in rank order, exclusive sum of the lower ranks' totals, the
    final state from the last rank) runs under gloo without a GPU. The block
    totals come from a plain sum written here; the finish phase is the oracle
    started from the offset state."""

    def workspace(self, q, seg_len):
        return None

    def state(self, k, v, seg_len, ws):
        import torch
        kk = k.double()
        sk = torch.where(kk > 0, kk + 1.0, torch.exp(kk))        # ELU + 1
        M = torch.einsum("bhtc,bhtj->bhcj", sk, v.double())
        return M.float(), sk.sum(dim=2).float()

    def exscan(self, totals_M, totals_z, part, M_in, z_in):
        off_M = totals_M[:part].sum(dim=0) if part > 0 else torch.zeros_like(totals_M[0])
        off_z = totals_z[:part].sum(dim=0) if part > 0 else torch.zeros_like(totals_z[0])
        if M_in is not None:
            off_M, off_z = off_M + M_in, off_z + z_in
        return off_M, off_z

    def finish(self, q, k, v, beta, M_in, z_in, seg_len, ws, out=None):
        import oracle
        o, M, z = oracle.forward(q.numpy(), k.numpy(), v.numpy(), beta.double().numpy(), M_in.double().numpy(),
                                 z_in.double().numpy(), seg_len=seg_len)
        return torch.from_numpy(o), torch.from_numpy(M).float(), torch.from_numpy(z).float()


import torch  # noqa: E402  (used by _NumpyPhases in the spawned ranks)


def _sharded_rank(rank, world, port, results):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import numpy as np
    import bench
    from compressive_memory_segment_b200 import sharded
    dist = bench.init_dist("gloo", timeout_s=60)
    r = np.random.default_rng(5)
    B, H, N, S, d = 1, 2, 4, 6, 8
    q, k, v = (torch.from_numpy(r.standard_normal((B, H, N * S, d))).float() for _ in range(3))
    beta = torch.from_numpy(r.standard_normal(H)).float()
    M0 = torch.from_numpy(r.standard_normal((B, H, d, d))).float()
    z0 = torch.from_numpy(np.abs(r.standard_normal((B, H, d))) + 1.0).float()
    blk = N * S // world
    sl = slice(rank * blk, (rank + 1) * blk)
    out, M, z = sharded.forward_sequence_sharded(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(),
                                                 v[:, :, sl].contiguous(), beta, N, M0, z0,
                                                 phases=_NumpyPhases())
    results[rank] = (out.numpy(), M.numpy(), z.numpy())
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_sequence_sharded_two_gloo_ranks():
    import numpy as np
    import oracle
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        results = m.dict()
        ctx = mp.get_context("spawn")
        procs = [ctx.Process(target=_sharded_rank, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(150)
        for p in procs:
            if p.is_alive():
                p.kill()
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(results)
    # The whole sequence on one process, through the oracle.
    r = np.random.default_rng(5)
    B, H, N, S, d = 1, 2, 4, 6, 8
    q, k, v = (r.standard_normal((B, H, N * S, d)).astype(np.float32) for _ in range(3))
    beta = r.standard_normal(H).astype(np.float32)
    M0 = r.standard_normal((B, H, d, d)).astype(np.float32)
    z0 = (np.abs(r.standard_normal((B, H, d))) + 1.0).astype(np.float32)
    ro, rM, rz = oracle.forward(q, k, v, beta.astype(np.float64), M0.astype(np.float64), z0.astype(np.float64),
                                seg_len=N)
    out = np.concatenate([res[0][0], res[1][0]], axis=2)
    assert np.max(np.abs(out - ro)) <= 1e-5 * np.max(np.abs(ro))
    for rk in range(world):  # every rank holds the state after the whole sequence
        assert np.max(np.abs(res[rk][1] - rM)) <= 1e-5 * np.max(np.abs(rM))
        assert np.max(np.abs(res[rk][2] - rz)) <= 1e-5 * np.max(np.abs(rz))
