"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The DSA step shards by sequence with no data-path collective: each rank runs
its own replica of the workload, and the job's step time is the slowest
rank's.  These tests run that logic as two gloo processes on the host.
"""

import json
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import dsa_inputs as di


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        wl = bench.replica_workload(di.CONFIGS["tiny_decode"], rank)
        inp = di.make_inputs(wl)
        # a rank-dependent "step time": the slowest rank must win everywhere
        my_ms = 1.0 + 0.25 * rank
        ms = bench.max_over_ranks(my_ms, dist, "cpu")
        # a second reduction in the same order on every rank, as the bench does
        e2e_ms = bench.max_over_ranks(10.0 - rank, dist, "cpu")
        res = {"rank": rank, "seed": wl.seed, "ms": ms, "e2e_ms": e2e_ms,
               "value": bench.job_rows_per_s(wl.n_q, world, ms),
               "q_sum": int(inp["q"].astype(np.int64).sum()),
               "shapes": {k: list(v.shape) for k, v in inp.items() if hasattr(v, "shape")}}
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run_two_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    return [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]


def test_replicas_and_max_over_ranks_gloo(tmp_path):
    res = _run_two_ranks(tmp_path)
    base = di.CONFIGS["tiny_decode"]
    # every rank sees the slowest rank's time, for each reduction
    assert [r["ms"] for r in res] == [1.25, 1.25]
    assert [r["e2e_ms"] for r in res] == [10.0, 10.0]
    # whole-job throughput counts the rows of both replicas
    assert res[0]["value"] == pytest.approx(base.n_q * 2 / 1.25e-3)
    # rank 0 runs the workload as named; other ranks run same-shaped, different batches
    assert res[0]["seed"] == base.seed and res[1]["seed"] != base.seed
    assert res[0]["shapes"] == res[1]["shapes"]
    assert res[0]["q_sum"] != res[1]["q_sum"]


def test_single_rank_helpers_without_a_process_group():
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    wl = di.CONFIGS["glm5_decode_8k"]
    assert bench.replica_workload(wl, 0) is wl
    r3 = bench.replica_workload(wl, 3)
    assert r3.seed == wl.seed + 3000 and r3.seq_lens == wl.seq_lens
    assert bench.job_rows_per_s(32, 4, 2.0) == pytest.approx(64000.0)
