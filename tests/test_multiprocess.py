"""Host logic of the multi-GPU bench on the CPU: world size 2 over gloo.

The attention block shards by batch with no exchange, so the only collectives
are the bench's timing barrier and the max over ranks; each rank draws its own
batch. These run here as two gloo processes on 127.0.0.1.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    r, w, local = bench.dist_setup(world)
    try:
        assert (r, w, local) == (rank, world, rank)
        assert dist.get_backend() == "gloo"
        bench.barrier(w)
        # every rank reports a different elapsed time; all must agree on the max
        m = bench.max_over_ranks(10.0 + rank, w)
        seed = bench.shard_seed(1, rank)
        # each rank draws its own batch from its own seed
        import workloads
        q = workloads.training_inputs(1, 4, 2, 1, 64, seed)[0]
        results[rank] = (m, seed, float(q.float().sum()))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_shards():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_worker, args=(world, port, results), nprocs=world, start_method="spawn", join=True)
    assert set(results.keys()) == {0, 1}
    assert results[0][0] == results[1][0] == 11.0          # max over ranks
    assert results[0][1] != results[1][1]                  # distinct shard seeds
    assert results[0][2] != results[1][2]                  # distinct shard data


def test_reference_arm_runs_on_rank0_only(monkeypatch):
    """bench.run_reference: rank 0 prints the oracle line, other ranks return None."""
    import bench

    class A:
        steps, warmup = 2, 1

    class Units:  # stands in for the oracle: a fixed amount of work per unit
        calls = 0

        def __init__(self, seed_offset=0):
            pass

        def run_one(self):
            Units.calls += 1
            return 1e9
    monkeypatch.setattr(bench, "OracleUnits", Units)
    assert bench.run_reference(A, 1, 2) is None
    assert Units.calls == 0
    res = bench.run_reference(A, 0, 2)
    assert Units.calls == 3  # warm-up + timed steps, one unit each
    assert res["impl"] == "reference" and res["cpu_baseline"]["kind"] == "oracle"
    assert res["e2e"]["h2d_bytes_per_step"] == 0 and res["value"] > 0
    assert res["e2e"]["value"] == res["value"] == res["cpu_baseline"]["value"]
    assert "per step" in res["config"]["workload"]
