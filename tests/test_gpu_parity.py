"""GPU path vs the float64 oracle, element by element, through the C ABI.

Indices and (integer-input) indexer scores must match bit-exactly; attention
outputs within 2e-3 max normalised abs error, lse within 2e-3 absolute.
"""

import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import dsa_inputs as di
import sparse_attention_scores_b200 as dsa
from oracle import dsa_oracle as orc
from tests.dsa_testutil import (LSE_TOL, OUT_TOL, assert_row_matches, bf16_tensor, cache_of,
                                dims_of, norm_err, row_lengths, run_forward, upload)

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dsa.lib()


# ---------------------------------------------------------------- step 1

INDEXER_CASES = [
    dict(seq_lens=[1, 63, 64, 65, 127, 128, 129, 1000, 4097], H_I=4, D_I=32),
    dict(seq_lens=[3000, 200, 129], H_I=32, D_I=128),
    dict(seq_lens=[700, 2049], H_I=8, D_I=64),
    dict(seq_lens=[5000], H_I=64, D_I=128),
    dict(seq_lens=[333, 4096, 1], H_I=2, D_I=128),
]


@pytest.mark.parametrize("case", INDEXER_CASES, ids=lambda c: f"HI{c['H_I']}_DI{c['D_I']}")
def test_indexer_scores_exact(case):
    wl = di.small_decode(case["seq_lens"], H_I=case["H_I"], D_I=case["D_I"], topk=64, seed=17)
    inp = di.make_inputs(wl)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    ld = (max(wl.seq_lens) + 3) // 4 * 4
    scores = torch.full((wl.n_q, ld), float("nan"), device="cuda")
    ws = dsa.workspace(dsa.OP_INDEXER_SCORES, dims, cache)
    dsa.dsa_indexer_scores(t["q_idx"], t["w"], t["k_pages"], cache, dims, scores, ws)
    assert dsa.workspace_check(ws)[0] == 0
    got = scores.cpu().numpy()
    for b, n in enumerate(wl.seq_lens):
        k_rows = orc.bf16_to_f64(orc.gather_paged_rows(inp["k_pages"], inp["block_table"][b],
                                                       range(n)))
        ref = orc.indexer_scores(orc.bf16_to_f64(inp["q_idx"][b]), inp["w"][b], k_rows)
        np.testing.assert_array_equal(got[b, :n].astype(np.float64), ref)
        assert np.isnan(got[b, n:]).all()   # entries past the context stay untouched


@pytest.mark.parametrize("T,q_pos0,H_I,D_I", [(300, 0, 32, 128), (130, 77, 4, 32), (257, 5, 64, 128)])
def test_indexer_scores_prefill_exact(T, q_pos0, H_I, D_I):
    wl = di.small_prefill(T, q_pos0=q_pos0, H_I=H_I, D_I=D_I, topk=64, seed=3)
    inp = di.make_inputs(wl)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    ld = (q_pos0 + T + 3) // 4 * 4
    scores = torch.full((T, ld), float("nan"), device="cuda")
    ws = dsa.workspace(dsa.OP_INDEXER_SCORES, dims, cache)
    dsa.dsa_indexer_scores(t["q_idx"], t["w"], t["k_pages"], cache, dims, scores, ws)
    assert dsa.workspace_check(ws)[0] == 0
    got = scores.cpu().numpy()
    k_all = orc.bf16_to_f64(orc.gather_paged_rows(inp["k_pages"], inp["block_table"][0],
                                                  range(q_pos0 + T)))
    for r in range(T):
        n = q_pos0 + r + 1
        ref = orc.indexer_scores(orc.bf16_to_f64(inp["q_idx"][r]), inp["w"][r], k_all[:n])
        np.testing.assert_array_equal(got[r, :n].astype(np.float64), ref)
        assert np.isnan(got[r, n:]).all()


def test_indexer_scores_normal_inputs_within_fp32_bound():
    # N(0,1) bf16 queries and keys and positive real head weights: the scores
    # are no longer exact in fp32.  Each bf16 product is exact in fp32; the
    # D_I-term dot product, the weighting and the H_I-term head sum each add
    # at most one fp32 rounding (2^-23 relative, allowing truncation) per term,
    # so |gpu - exact| <= 2^-23 (D_I + H_I + 2) sum_h w_h sum_d |q_hd k_d|.
    wl = di.small_decode([5000, 1234, 64, 3001], H_I=32, D_I=128, topk=512, H=4, R=64, P=16,
                         seed=61)
    inp = di.make_inputs(wl)
    rng = np.random.default_rng(62)
    inp["q_idx"] = di.f32_to_bf16_bits(rng.standard_normal(inp["q_idx"].shape).astype(np.float32))
    inp["k_pages"] = di.f32_to_bf16_bits(rng.standard_normal(inp["k_pages"].shape).astype(np.float32))
    inp["w"] = np.abs(rng.standard_normal(inp["w"].shape)).astype(np.float32)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    ld = (max(wl.seq_lens) + 3) // 4 * 4
    scores = torch.full((wl.n_q, ld), float("nan"), device="cuda")
    ws = dsa.workspace(dsa.OP_INDEXER_SCORES, dims, cache)
    dsa.dsa_indexer_scores(t["q_idx"], t["w"], t["k_pages"], cache, dims, scores, ws)
    assert dsa.workspace_check(ws)[0] == 0
    got = scores.cpu().numpy()
    # the selection the library makes from those scores
    idx = torch.full((wl.n_q, wl.topk), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(scores, t["seq_lens"], 0, wl.topk, idx, ws)
    assert dsa.workspace_check(ws)[0] == 0
    idx = idx.cpu().numpy()
    D_I, H_I = wl.D_I, wl.H_I
    for b, n in enumerate(wl.seq_lens):
        k_rows = orc.bf16_to_f64(orc.gather_paged_rows(inp["k_pages"], inp["block_table"][b],
                                                       range(n)))
        q = orc.bf16_to_f64(inp["q_idx"][b])
        w = inp["w"][b].astype(np.float64)
        ref = orc.indexer_scores(q, inp["w"][b], k_rows)
        bound = 2.0 ** -23 * (D_I + H_I + 2) * (np.abs(k_rows) @ np.abs(q).T) @ w
        err = np.abs(got[b, :n].astype(np.float64) - ref)
        assert np.all(err <= bound), (b, float(np.max(err / np.maximum(bound, 1e-300))))
        # exact top-k of the GPU's own fp32 scores (both sides decide in fp32)
        want = orc.topk_select(got[b, :n].astype(np.float64), wl.topk)
        np.testing.assert_array_equal(idx[b].astype(np.int64), want)


# ---------------------------------------------------------------- step 2

def _topk_rows(lengths, k, seed, kind):
    rng = np.random.default_rng(seed)
    ld = max(4, (max(lengths) + 3) // 4 * 4)
    s = np.full((len(lengths), ld), np.nan, np.float32)
    for r, n in enumerate(lengths):
        if kind == "ints":
            v = rng.integers(0, 6, n).astype(np.float32)          # heavy ties
        elif kind == "signed":
            v = (rng.integers(-4, 5, n) * 0.5).astype(np.float32)
            v[rng.random(n) < 0.2] = -0.0                          # -0.0 ties with +0.0
        else:
            v = rng.standard_normal(n).astype(np.float32)
        s[r, :n] = v
    return s


@pytest.mark.parametrize("kind", ["ints", "signed", "normal"])
@pytest.mark.parametrize("k", [1, 64, 2048])
def test_topk_exact(kind, k):
    lengths = [0, 1, max(1, k - 1), k, k + 1, 3 * k + 5, 5000, 20000]
    s = _topk_rows(lengths, k, seed=k, kind=kind)
    scores = torch.from_numpy(s).cuda()
    vl = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    idx = torch.full((len(lengths), k), -7, dtype=torch.int32, device="cuda")
    ws = dsa.workspace(dsa.OP_TOPK, dsa.Dims(len(lengths), 1, 32, k, 1, 64, 0), None)
    dsa.dsa_topk(scores, vl, 0, k, idx, ws)
    got = idx.cpu().numpy()
    for r, n in enumerate(lengths):
        want = orc.topk_select(s[r, :n].astype(np.float64), k)
        assert np.array_equal(got[r].astype(np.int64), want), (r, n)


def test_topk_causal_rows():
    # no length array: row r sees causal_base + r + 1 entries
    T, base, k = 300, 20, 64
    s = _topk_rows([base + T] * T, k, seed=5, kind="ints")
    scores = torch.from_numpy(s).cuda()
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    ws = dsa.workspace(dsa.OP_TOPK, dsa.Dims(T, 1, 32, k, 1, 64, 0), None)
    dsa.dsa_topk(scores, None, base, k, idx, ws)
    got = idx.cpu().numpy()
    for r in range(T):
        want = orc.topk_select(s[r, :base + r + 1].astype(np.float64), k)
        assert np.array_equal(got[r].astype(np.int64), want), r


@pytest.mark.parametrize("n", [131072, 400000, 1048576])
def test_topk_long_rows(n):
    # 1,048,576 entries exceed the cluster's shared memory: the re-reading path
    k = 2048
    s = _topk_rows([n, n // 2 + 3], k, seed=n, kind="ints")
    scores = torch.from_numpy(s).cuda()
    vl = torch.tensor([n, n // 2 + 3], dtype=torch.int32, device="cuda")
    idx = torch.empty((2, k), dtype=torch.int32, device="cuda")
    ws = dsa.workspace(dsa.OP_TOPK, dsa.Dims(2, 1, 32, k, 1, 64, 0), None)
    dsa.dsa_topk(scores, vl, 0, k, idx, ws)
    got = idx.cpu().numpy()
    for r, m in enumerate([n, n // 2 + 3]):
        want = np.sort(np.argsort(-s[r, :m].astype(np.float64), kind="stable")[:k])
        assert np.array_equal(got[r].astype(np.int64), want)


@pytest.mark.parametrize("kind", ["ints", "normal"])
@pytest.mark.parametrize("lengths", [
    [4096, 3000, 300],                 # one CTA per row, 4 keys per thread
    [8192, 8191, 2049],                # one CTA per row, 8 keys per thread
    [16384, 9001, 12345],              # clusters of 4, 4 keys per thread
    [16388, 16001],                    # clusters of 5, 4 keys per thread
    [131072, 70001],                   # clusters of 16, 8 keys per thread
    [65536] * 24 + [40000] * 8,        # 32 rows: clusters of 4, 16 keys per thread
], ids=["small4", "small8", "cluster4x4", "cluster5x4", "cluster16x8", "cluster4x16"])
def test_topk_kernel_paths(kind, lengths):
    # each row set lands on one of the top-k kernels (chosen by the row count
    # and the longest row); the ragged rows of a launch share it
    k = 2048
    s = _topk_rows(lengths, k, seed=len(lengths) + lengths[0], kind=kind)
    scores = torch.from_numpy(s).cuda()
    vl = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    idx = torch.full((len(lengths), k), -7, dtype=torch.int32, device="cuda")
    ws = dsa.workspace(dsa.OP_TOPK, dsa.Dims(len(lengths), 1, 32, k, 1, 64, 0), None)
    dsa.dsa_topk(scores, vl, 0, k, idx, ws)
    got = idx.cpu().numpy()
    for r, m in enumerate(lengths):
        want = np.full(k, -1, np.int64)
        sel = np.sort(np.argsort(-s[r, :m].astype(np.float64), kind="stable")[:k])
        want[:len(sel)] = sel
        assert np.array_equal(got[r].astype(np.int64), want), (r, m)


# ---------------------------------------------------------------- step 3

def _random_selection(rng, lengths, k):
    idx = np.full((len(lengths), k), -1, np.int32)
    for r, n in enumerate(lengths):
        m = min(n, k)
        idx[r, :m] = np.sort(rng.choice(n, size=m, replace=False))
    return idx


@pytest.mark.parametrize("shape", [dict(H=4, R=64, P=16, k=256), dict(H=64, R=512, P=64, k=2048),
                                   dict(H=16, R=128, P=32, k=300)])
@pytest.mark.parametrize("batch", [1, 5, 160])
def test_sparse_mla_decode(shape, batch):
    _mla_decode_case(shape, batch)


@pytest.mark.parametrize("batch", [1, 2])
def test_sparse_mla_decode_many_splits(batch):
    # 64 or 32 splits per row: more than one cluster holds, so the partials
    # go through global scratch and the merge kernel
    _mla_decode_case(dict(H=64, R=512, P=64, k=8192), batch)


@pytest.mark.parametrize("shape,batch", [
    (dict(H=64, R=512, P=64, k=2048), 10),   # 8 splits per row, merged in a cluster of 8
    (dict(H=64, R=512, P=64, k=2048), 32),   # clusters of 4
    (dict(H=64, R=512, P=64, k=2048), 74),   # clusters of 2
    (dict(H=4, R=64, P=16, k=256), 40),      # one 128-column block, clusters of 2
    (dict(H=16, R=192, P=32, k=2048), 10),   # a ragged last column block, clusters of 8
], ids=["c8", "c4", "c2", "tiny_c2", "r192_c8"])
def test_sparse_mla_cluster_merge(shape, batch):
    # rows split over 2..8 CTAs merge their partials through distributed shared
    # memory; short rows leave some splits empty and one row selects nothing
    _mla_decode_case(shape, batch, every_row=True, empty_row=batch // 2)


def _mla_decode_case(shape, batch, every_row=False, empty_row=None):
    rng = np.random.default_rng(batch * 7 + shape["k"])
    lengths = rng.integers(1, 3 * shape["k"], size=batch).tolist()
    wl = di.small_decode(lengths, H_I=4, D_I=32, topk=shape["k"], H=shape["H"], R=shape["R"],
                         P=shape["P"], seed=batch)
    inp = di.make_inputs(wl)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    sel = _random_selection(rng, lengths, shape["k"])
    if empty_row is not None:
        sel[empty_row, :] = -1
    idx = torch.from_numpy(sel).cuda()
    out = torch.full((batch, wl.H, wl.R), float("nan"), device="cuda")
    lse = torch.full((batch, wl.H), float("nan"), device="cuda")
    ws = dsa.workspace(dsa.OP_SPARSE_MLA_DECODE, dims, cache)
    dsa.dsa_sparse_mla_decode(t["q"], t["latent_pages"], cache, idx, dims, out, lse, ws)
    assert dsa.workspace_check(ws)[0] == 0
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    if empty_row is not None:
        assert (out[empty_row] == 0).all() and np.isneginf(lse[empty_row]).all()
    for b in range(0, batch, 1 if every_row else max(1, batch // 12)):
        if b == empty_row:
            continue
        s = sel[b][sel[b] >= 0]
        rows = orc.bf16_to_f64(orc.gather_paged_rows(inp["latent_pages"], inp["block_table"][b], s))
        ref_out, ref_lse, _ = orc.mla_attention(orc.bf16_to_f64(inp["q"][b]), rows, wl.R, wl.scale)
        assert norm_err(out[b], ref_out) <= OUT_TOL
        assert np.max(np.abs(lse[b] - ref_lse)) <= LSE_TOL


def test_sparse_mla_prefill_and_empty_rows():
    T, k = 200, 64
    wl = di.small_prefill(T, q_pos0=0, H_I=4, D_I=32, topk=k, H=8, R=64, P=16, seed=2)
    inp = di.make_inputs(wl)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    rng = np.random.default_rng(0)
    sel = _random_selection(rng, [r + 1 for r in range(T)], k)
    sel[7, :] = -1     # a row with no kept token: out = 0, lse = -inf
    idx = torch.from_numpy(sel).cuda()
    out = torch.empty((T, wl.H, wl.R), device="cuda")
    lse = torch.empty((T, wl.H), device="cuda")
    ws = dsa.workspace(dsa.OP_SPARSE_MLA_PREFILL, dims, cache)
    dsa.dsa_sparse_mla_prefill(t["q"], t["latent_pages"], cache, idx, dims, out, lse, ws)
    assert dsa.workspace_check(ws)[0] == 0
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    assert (out[7] == 0).all() and np.isneginf(lse[7]).all()
    for r in [0, 1, 63, 64, 65, 150, 199]:
        s = sel[r][sel[r] >= 0]
        rows = orc.bf16_to_f64(orc.gather_paged_rows(inp["latent_pages"], inp["block_table"][0], s))
        ref_out, ref_lse, _ = orc.mla_attention(orc.bf16_to_f64(inp["q"][r]), rows, wl.R, wl.scale)
        assert norm_err(out[r], ref_out) <= OUT_TOL
        assert np.max(np.abs(lse[r] - ref_lse)) <= LSE_TOL


@pytest.mark.parametrize("T,q_pos0,k,R,P,H", [(40, 0, 256, 64, 16, 4), (12, 3000, 2048, 512, 64, 64)],
                         ids=["short_c2", "long_context_c8"])
def test_sparse_mla_prefill_cluster_merge(T, q_pos0, k, R, P, H):
    # a short prefill chunk splits its rows over 2..8 CTAs, which merge in a cluster
    wl = di.small_prefill(T, q_pos0=q_pos0, H_I=4, D_I=32, topk=k, H=H, R=R, P=P, seed=T + 1)
    inp = di.make_inputs(wl)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    rng = np.random.default_rng(T)
    sel = _random_selection(rng, [q_pos0 + r + 1 for r in range(T)], k)
    idx = torch.from_numpy(sel).cuda()
    out = torch.full((T, wl.H, wl.R), float("nan"), device="cuda")
    lse = torch.full((T, wl.H), float("nan"), device="cuda")
    ws = dsa.workspace(dsa.OP_SPARSE_MLA_PREFILL, dims, cache)
    dsa.dsa_sparse_mla_prefill(t["q"], t["latent_pages"], cache, idx, dims, out, lse, ws)
    assert dsa.workspace_check(ws)[0] == 0
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    for r in range(T):
        s = sel[r][sel[r] >= 0]
        rows = orc.bf16_to_f64(orc.gather_paged_rows(inp["latent_pages"], inp["block_table"][0], s))
        ref_out, ref_lse, _ = orc.mla_attention(orc.bf16_to_f64(inp["q"][r]), rows, wl.R, wl.scale)
        assert norm_err(out[r], ref_out) <= OUT_TOL, r
        assert np.max(np.abs(lse[r] - ref_lse)) <= LSE_TOL, r


# ---------------------------------------------------------------- whole step

FORWARD_CASES = [
    di.small_decode([50, 64, 300, 1000, 4100], H_I=4, D_I=32, topk=128, H=8, R=64, P=16, seed=1),
    di.small_decode([2100, 2048, 5000], H_I=32, D_I=128, topk=2048, H=64, R=512, P=64, seed=2),
    di.small_decode([900, 90], H_I=2, D_I=64, topk=256, H=64, R=512, P=64, seed=3),
    di.small_prefill(260, q_pos0=0, H_I=32, D_I=128, topk=128, H=64, R=512, P=64, seed=4),
    di.small_prefill(150, q_pos0=40, H_I=4, D_I=32, topk=100, H=4, R=64, P=16, seed=5),
]


@pytest.mark.parametrize("wl", FORWARD_CASES, ids=lambda w: f"{w.mode}_{w.n_q}_{w.topk}")
def test_forward_small(wl):
    inp = di.make_inputs(wl)
    idx, out, lse = run_forward(inp)
    ref = orc.dsa_prefill(inp) if wl.mode == "prefill" else orc.dsa_decode(inp)
    for r, res in ref.items():
        assert_row_matches(r, res, idx, out, lse)


def test_fused_equals_composed_and_repeatable():
    wl = di.small_decode([3000, 2500, 70], H_I=32, D_I=128, topk=2048, H=64, R=512, P=64, seed=9)
    inp = di.make_inputs(wl)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    idx_f, out_f, lse_f = run_forward(inp, t)
    idx_f2, out_f2, lse_f2 = run_forward(inp, t)
    assert np.array_equal(idx_f, idx_f2) and np.array_equal(out_f, out_f2)
    assert np.array_equal(lse_f, lse_f2)
    ld = (max(wl.seq_lens) + 3) // 4 * 4
    scores = torch.empty((wl.n_q, ld), device="cuda")
    ws = dsa.workspace(dsa.OP_ATTENTION_FORWARD, dims, cache)
    dsa.dsa_indexer_scores(t["q_idx"], t["w"], t["k_pages"], cache, dims, scores, ws)
    idx = torch.empty((wl.n_q, wl.topk), dtype=torch.int32, device="cuda")
    dsa.dsa_topk(scores, t["seq_lens"], 0, wl.topk, idx, ws)
    out = torch.empty((wl.n_q, wl.H, wl.R), device="cuda")
    lse = torch.empty((wl.n_q, wl.H), device="cuda")
    dsa.dsa_sparse_mla_decode(t["q"], t["latent_pages"], cache, idx, dims, out, lse, ws)
    assert dsa.workspace_check(ws)[0] == 0
    assert np.array_equal(idx.cpu().numpy(), idx_f)
    assert np.array_equal(out.cpu().numpy(), out_f)       # bitwise
    assert np.array_equal(lse.cpu().numpy(), lse_f)


def test_few_indexer_heads_tie_rule():
    # two indexer heads: the ReLU zeroes both heads for many keys, which then
    # tie exactly; the kept set must follow the lower-index rule
    wl = di.small_decode([6000, 3001], H_I=2, D_I=32, topk=512, H=4, R=64, P=16, seed=21)
    inp = di.make_inputs(wl)
    idx, out, lse = run_forward(inp)
    ref = orc.dsa_decode(inp)
    for r, res in ref.items():
        assert (res["scores"] == 0).sum() > 100
        assert_row_matches(r, res, idx, out, lse)


# ---------------------------------------------------------------- device-side checks

def test_bad_page_id_is_reported_not_faulted():
    wl = di.small_decode([700, 300], H_I=4, D_I=32, topk=64, H=4, R=64, P=16, seed=4)
    inp = di.make_inputs(wl)
    bad = dict(inp)
    bt = inp["block_table"].copy()
    bt[0, 3] = inp["k_pages"].shape[0] + 5     # out of the pool
    bad["block_table"] = bt
    t = upload(bad)
    cache, dims = cache_of(bad, t), dims_of(bad)
    idx = torch.empty((2, 64), dtype=torch.int32, device="cuda")
    out = torch.empty((2, 4, 64), device="cuda")
    lse = torch.empty((2, 4), device="cuda")
    ws = dsa.workspace(dsa.OP_ATTENTION_FORWARD, dims, cache)
    dsa.dsa_attention_forward(t["q_idx"], t["w"], t["k_pages"], t["q"], t["latent_pages"], cache,
                              dims, idx, out, lse, ws)
    st, info = dsa.workspace_check(ws)
    assert st == 6      # DSA_ERR_DEVICE_CHECK
    # the context is still usable and a clean call succeeds
    idx2, out2, lse2 = run_forward(inp)
    ref = orc.dsa_decode(inp)
    assert_row_matches(1, ref[1], idx2, out2, lse2)


@pytest.mark.parametrize("kernel", [1, 3], ids=["indexer", "mla"])
def test_bounded_wait_timeout_path(kernel):
    # DSA_DEBUG_STALL makes the chosen kernel wait once on a barrier that
    # nothing arrives at; with a 50 ms limit the wait runs out, the kernel
    # records DSA_ERR_TIMEOUT, drains what is in flight, frees its tensor
    # memory and returns, and the context stays usable (child process: the
    # library reads both variables once, at first use)
    code = r"""
import sys, numpy as np, torch
sys.path.insert(0, %r)
import dsa_inputs as di
import sparse_attention_scores_b200 as dsa
from tests.dsa_testutil import upload, cache_of, dims_of, run_forward
wl = di.small_decode([5000, 3000], H_I=32, D_I=128, topk=2048, H=64, R=512, P=64, seed=1)
inp = di.make_inputs(wl); t = upload(inp)
cache, dims = cache_of(inp, t), dims_of(inp)
idx = torch.empty((2, 2048), dtype=torch.int32, device="cuda")
out = torch.empty((2, 64, 512), device="cuda"); lse = torch.empty((2, 64), device="cuda")
ws = dsa.workspace(dsa.OP_ATTENTION_FORWARD, dims, cache)
dsa.dsa_attention_forward(t["q_idx"], t["w"], t["k_pages"], t["q"], t["latent_pages"], cache,
                          dims, idx, out, lse, ws)
st, info = dsa.workspace_check(ws)
x = torch.ones(1000, device="cuda").sum().item()
print("STATUS", st, hex(info), x)
""" % ROOT
    env = dict(os.environ, DSA_WAIT_LIMIT_NS="50000000", DSA_DEBUG_STALL=str(kernel))
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env,
                         timeout=300, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    line = [l for l in res.stdout.splitlines() if l.startswith("STATUS")][0]
    st, info = int(line.split()[1]), int(line.split()[2], 16)
    assert st == 5, line     # DSA_ERR_TIMEOUT
    assert info >> 24 == kernel, line
    assert line.endswith("1000.0")
