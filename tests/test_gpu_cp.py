"""Context-parallel decode on one GPU: R ranks emulated one after another in
one process (each rank's shard, the library's per-rank steps, the all-gathers
as stacks), against the oracle's one-device step over whole sequences.  No
rank waits on another, so nothing here needs more than one GPU."""

import numpy as np
import pytest
import torch

import cp_testutil as cpt
import dsa_inputs as di
import sparse_attention_scores_b200 as dsa
from oracle import dsa_oracle as orc
from sparse_attention_scores_b200.context_parallel import RankShard, cuda_ops
from dsa_testutil import upload, cache_of, dims_of, assert_row_matches

pytestmark = pytest.mark.gpu


def _run_emulated(wl, ranks):
    inp = di.make_inputs(wl)
    dims = dims_of(inp)
    ops = cuda_ops(dims)
    shards = []
    for r in range(ranks):
        lo = np.array([cpt.shard_bounds(n, ranks)[r] for n in wl.seq_lens])
        hi = np.array([cpt.shard_bounds(n, ranks)[r + 1] for n in wl.seq_lens])
        sh = cpt.make_shard(inp, wl, lo, hi)
        t = upload(sh)
        t["cache"] = cache_of(sh, t)
        shards.append(RankShard(offsets=torch.from_numpy(sh["offsets"]).cuda(),
                                lens=torch.from_numpy(sh["seq_lens"]).cuda(), local=t))
    cand = [ops.candidates(*ops.local_topk(s, wl.topk), s.offsets) for s in shards]
    all_s = torch.stack([c[0] for c in cand])
    all_i = torch.stack([c[1] for c in cand])
    sel = [ops.select(all_s, all_i, s.offsets, s.lens) for s in shards]
    for g, _ in sel[1:]:                       # every rank computes the same global indices
        assert torch.equal(g, sel[0][0])
    part = [ops.attend(s, own) for s, (_, own) in zip(shards, sel)]
    out, lse = ops.merge(torch.stack([p[0] for p in part]), torch.stack([p[1] for p in part]))
    torch.cuda.synchronize()
    return inp, sel[0][0].cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("ranks", [2, 4])
def test_context_parallel_matches_one_device_step(ranks):
    wl = di.small_decode([9000, 3000, 2100], H_I=32, D_I=128, topk=2048, H=64, R=512, P=64,
                         seed=81, scale=1 / 192 ** 0.5)
    inp, gidx, out, lse = _run_emulated(wl, ranks)
    for b, res in orc.dsa_decode(inp).items():
        assert_row_matches(b, res, gidx, out, lse)


def test_context_parallel_long_row_8_ranks():
    # one 131,072-token row over 8 ranks (16,384 keys each)
    wl = di.small_decode([131072], H_I=32, D_I=128, topk=2048, H=64, R=512, P=64, seed=82,
                         scale=1 / 192 ** 0.5)
    inp, gidx, out, lse = _run_emulated(wl, 8)
    assert_row_matches(0, orc.dsa_decode(inp)[0], gidx, out, lse)
