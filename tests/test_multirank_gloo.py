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
