"""Multi-process host logic of the benchmark on CPU: two gloo ranks on
127.0.0.1, each with its own replica workload; the job time is the slowest
rank's, the throughput counts every rank's tokens."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    import bench
    from compressed_kv_cache_routing_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        spec = bench.replica_spec(W.SPECS["tiny"], rank)
        w = W.generate(spec)
        ms = 1.0 + rank  # rank 1 is the slow one
        value, ms_max = bench.aggregate(w.context_tokens, ms, world)
        bench.barrier(world)
        results[rank] = (spec.seed, int(w.seq_lens.sum()), float(w.q.sum()), value, ms_max)
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    (s0, t0, q0, v0, m0), (s1, t1, q1, v1, m1) = results[0], results[1]
    assert s0 != s1 and q0 != q1          # each rank has its own replica
    assert t0 == t1 == 1024               # same shapes
    assert m0 == m1 == 2.0                # the slowest rank sets the time
    assert v0 == v1 == pytest.approx(2 * 1024 / 2e-3)
