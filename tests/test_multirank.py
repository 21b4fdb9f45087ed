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


# ---------------------------------------------------------------- context-parallel exchange

def _oracle_ops(inp_shard, wl):
    """The per-rank steps as the float64 oracle (CPU tensors)."""
    import torch
    from oracle import dsa_oracle as orc
    from sparse_attention_scores_b200.context_parallel import CpOps

    def local_topk(shard, k):
        s = shard.local
        n_q = s["q_idx"].shape[0]
        lens = s["seq_lens"]
        ld = max(1, int(lens.max()))
        scores = np.full((n_q, ld), np.nan)
        idx = np.full((n_q, k), -1, np.int64)
        for b in range(n_q):
            n = int(lens[b])
            keys = orc.bf16_to_f64(orc.gather_paged_rows(s["k_pages"], s["block_table"][b], range(n)))
            sc = orc.indexer_scores(orc.bf16_to_f64(s["q_idx"][b]), s["w"][b], keys)
            scores[b, :n] = sc
            idx[b] = orc.topk_select(sc, k)
        return torch.from_numpy(scores), torch.from_numpy(idx)

    def candidates(scores, idx, offsets):
        sc, ix, off = scores.numpy(), idx.numpy(), offsets.numpy()
        cs = np.where(ix >= 0, np.take_along_axis(sc, np.maximum(ix, 0), 1), -np.inf)
        ci = np.where(ix >= 0, ix + off[:, None], -1)
        return torch.from_numpy(cs), torch.from_numpy(ci)

    def select(all_s, all_i, offsets, lens):
        a_s, a_i = all_s.numpy(), all_i.numpy()
        n_q, k = a_s.shape[1], a_s.shape[2]
        g = np.stack([orc.cp_merge_candidates(a_s[:, b], a_i[:, b], k) for b in range(n_q)])
        off, ln = offsets.numpy()[:, None], lens.numpy()[:, None]
        own = np.where((g >= off) & (g < off + ln), g - off, -1)
        return torch.from_numpy(g), torch.from_numpy(own)

    def attend(shard, own):
        s = shard.local
        outs, lses = [], []
        for b in range(own.shape[0]):
            o = own[b].numpy()
            sel = o[o >= 0]
            if len(sel) == 0:
                outs.append(np.zeros((wl.H, wl.R)))
                lses.append(np.full(wl.H, -np.inf))
                continue
            rows = orc.bf16_to_f64(orc.gather_paged_rows(s["latent_pages"], s["block_table"][b], sel))
            out, lse, _ = orc.mla_attention(orc.bf16_to_f64(s["q"][b]), rows, wl.R, wl.scale)
            outs.append(out)
            lses.append(lse)
        return torch.from_numpy(np.stack(outs)), torch.from_numpy(np.stack(lses))

    def merge(outs, lses):
        o, l = outs.numpy(), lses.numpy()
        res = [orc.cp_merge_partials(o[:, b], l[:, b]) for b in range(o.shape[1])]
        return (torch.from_numpy(np.stack([r[0] for r in res])),
                torch.from_numpy(np.stack([r[1] for r in res])))

    return CpOps(local_topk, candidates, select, attend, merge)


def _cp_rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    import cp_testutil as cpt
    from sparse_attention_scores_b200.context_parallel import RankShard, cp_decode_step
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    try:
        wl = di.small_decode([900, 301, 64], H_I=4, D_I=32, topk=100, H=3, R=16, P=8, seed=71)
        inp = di.make_inputs(wl)
        lo = np.array([cpt.shard_bounds(n, world)[rank] for n in wl.seq_lens])
        hi = np.array([cpt.shard_bounds(n, world)[rank + 1] for n in wl.seq_lens])
        sh = cpt.make_shard(inp, wl, lo, hi)
        shard = RankShard(offsets=torch.from_numpy(sh["offsets"].astype(np.int64)),
                          lens=torch.from_numpy(sh["seq_lens"].astype(np.int64)), local=sh)
        gidx, out, lse = cp_decode_step(shard, wl.topk, _oracle_ops(sh, wl), dist=dist)
        np.save(os.path.join(out_dir, f"cp{rank}.npy"),
                {"gidx": gidx.numpy(), "out": out.numpy(), "lse": lse.numpy()}, allow_pickle=True)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_exchange_gloo(tmp_path, world):
    from oracle import dsa_oracle as orc
    mp.start_processes(_cp_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [np.load(tmp_path / f"cp{r}.npy", allow_pickle=True).item() for r in range(world)]
    wl = di.small_decode([900, 301, 64], H_I=4, D_I=32, topk=100, H=3, R=16, P=8, seed=71)
    ref = orc.dsa_decode(di.make_inputs(wl))
    for r in range(world):
        for b in range(len(wl.seq_lens)):
            assert np.array_equal(res[r]["gidx"][b], ref[b]["idx"]), (r, b)
            np.testing.assert_allclose(res[r]["out"][b], ref[b]["out"], rtol=1e-9, atol=1e-12)
            np.testing.assert_allclose(res[r]["lse"][b], ref[b]["lse"], rtol=1e-12)
