"""Indexer work order on the GPU.

With enough work units per CTA the indexer splits part of them statically
over the CTAs (half for grouped causal prefill, three quarters for decode
with bf16 keys)
and hands out the rest in chunks from a counter in the workspace status
block; the last CTA to stop taking chunks puts the counter back to zero.
Every launch on the same workspace must therefore score every key of every
row, in whatever order the CTAs take the chunks, and leave the counter at
zero for the next launch.
"""

import numpy as np
import pytest
import torch

import dsa_inputs as di
import sparse_attention_scores_b200 as dsa
from oracle import dsa_oracle as orc
from dsa_testutil import cache_of, dims_of, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dsa.lib()


def _counter_words(ws):
    # DevStatus: flags, first, count, then the two counter words
    return ws[12:20].clone().view(torch.int32).tolist()


@pytest.mark.parametrize("k8", [False, True], ids=["bf16_keys", "fp8_keys"])
def test_prefill_indexer_repeated_launches_cover_every_unit(k8):
    # 1,600 rows after 300 cached tokens: 400 row groups and 3,636 128-key
    # units, half of them handed out in chunks of six on 148 CTAs
    wl = di.small_prefill(1600, q_pos0=300, H_I=32, D_I=128, topk=64, H=4, R=64, P=16, seed=71,
                          shuffle_pages=True)
    inp = di.make_inputs(wl)
    if k8:
        inp = di.with_fp8_keys(inp, seed=71)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    T, q_pos0 = wl.n_q, wl.q_pos0
    ld = (q_pos0 + T + 3) // 4 * 4
    op = dsa.OP_INDEXER_SCORES_K8 if k8 else dsa.OP_INDEXER_SCORES
    ws = dsa.workspace(op, dims, cache)
    if k8:
        k8_pages = torch.from_numpy(inp["k8_pages"]).cuda()
        k_scale = torch.from_numpy(inp["k_scale"]).cuda()
    runs = []
    for _ in range(3):
        scores = torch.full((T, ld), float("nan"), device="cuda")
        if k8:
            dsa.dsa_indexer_scores_k8(t["q_idx"], t["w"], k8_pages, k_scale, cache, dims, scores, ws)
        else:
            dsa.dsa_indexer_scores(t["q_idx"], t["w"], t["k_pages"], cache, dims, scores, ws)
        st, info = dsa.workspace_check(ws)
        assert st == 0, (st, hex(info))
        assert _counter_words(ws) == [0, 0]
        runs.append(scores.cpu().numpy())
    for r in range(T):
        n = q_pos0 + r + 1
        # every key of the row written (scores are finite), nothing past it
        assert np.isfinite(runs[0][r, :n]).all(), f"row {r}"
        assert np.isnan(runs[0][r, n:]).all(), f"row {r}"
    for other in runs[1:]:
        np.testing.assert_array_equal(np.nan_to_num(other, nan=-1.0), np.nan_to_num(runs[0], nan=-1.0))
    # sampled rows (spread over the row groups, last rows included) against the oracle
    rows = list(range(0, T, 97)) + [T - 2, T - 1]
    ref = orc.dsa_prefill(inp, rows=rows)
    for r in rows:
        n = q_pos0 + r + 1
        np.testing.assert_array_equal(runs[0][r, :n].astype(np.float64), ref[r]["scores"])


@pytest.mark.parametrize("k8", [False, True], ids=["bf16_keys", "fp8_keys"])
def test_decode_indexer_with_counter_exact(k8):
    # 8 rows of about 40K keys: 2,449 128-key units on 296 decode CTAs, enough
    # (8 or more per CTA) for bf16-key decode CTAs to take a quarter of them
    # from the counter (FP8-key decode stays static); every launch on one
    # workspace matches the oracle bit for bit
    lens = [40000, 38001, 39555, 40960, 37000, 40001, 39000, 38500]
    wl = di.small_decode(lens, H_I=32, D_I=128, topk=64, H=4, R=64, P=16, seed=73,
                         shuffle_pages=True)
    inp = di.make_inputs(wl)
    if k8:
        inp = di.with_fp8_keys(inp, seed=73)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    ld = (max(lens) + 3) // 4 * 4
    op = dsa.OP_INDEXER_SCORES_K8 if k8 else dsa.OP_INDEXER_SCORES
    ws = dsa.workspace(op, dims, cache)
    if k8:
        k8_pages = torch.from_numpy(inp["k8_pages"]).cuda()
        k_scale = torch.from_numpy(inp["k_scale"]).cuda()
    ref = orc.dsa_decode(inp)
    for _ in range(2):
        scores = torch.full((len(lens), ld), float("nan"), device="cuda")
        if k8:
            dsa.dsa_indexer_scores_k8(t["q_idx"], t["w"], k8_pages, k_scale, cache, dims, scores, ws)
        else:
            dsa.dsa_indexer_scores(t["q_idx"], t["w"], t["k_pages"], cache, dims, scores, ws)
        st, info = dsa.workspace_check(ws)
        assert st == 0, (st, hex(info))
        assert _counter_words(ws) == [0, 0]
        got = scores.cpu().numpy()
        for b, n in enumerate(lens):
            np.testing.assert_array_equal(got[b, :n].astype(np.float64), ref[b]["scores"])
            assert np.isnan(got[b, n:]).all()
