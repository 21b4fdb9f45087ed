"""FP8 (E4M3 + per-token scale) index keys on the GPU: scores, selections and
the whole step against the oracle, and against the bf16-key path on keys that
stand for the same values."""

import numpy as np
import pytest
import torch

import dsa_inputs as di
import sparse_attention_scores_b200 as dsa
from oracle import dsa_oracle as orc
from dsa_testutil import upload, cache_of, dims_of, row_lengths, run_forward, assert_row_matches

pytestmark = pytest.mark.gpu


def _k8_tensors(inp):
    return (torch.from_numpy(inp["k8_pages"]).cuda(), torch.from_numpy(inp["k_scale"]).cuda())


def _scores(inp, t, k8=None):
    cache, dims = cache_of(inp, t), dims_of(inp)
    ld = max(4, (int(row_lengths(inp).max()) + 3) // 4 * 4)
    scores = torch.full((dims.n_q, ld), float("nan"), device="cuda")
    ws = dsa.workspace(dsa.OP_INDEXER_SCORES if k8 is None else dsa.OP_INDEXER_SCORES_K8, dims,
                       cache)
    if k8 is None:
        dsa.dsa_indexer_scores(t["q_idx"], t["w"], t["k_pages"], cache, dims, scores, ws)
    else:
        dsa.dsa_indexer_scores_k8(t["q_idx"], t["w"], k8[0], k8[1], cache, dims, scores, ws)
    st, info = dsa.workspace_check(ws)
    assert st == 0, (st, hex(info))
    return scores.cpu().numpy()


CASES = [
    di.small_decode([300, 129, 64, 2000, 1], H_I=32, D_I=128, topk=64, H=64, R=512, P=64, seed=51,
                    shuffle_pages=True),
    di.small_decode([1000, 4097], H_I=4, D_I=128, topk=256, H=4, R=64, P=16, seed=52),
    di.small_prefill(400, q_pos0=90, H_I=32, D_I=128, topk=128, H=64, R=512, P=64, seed=53,
                     shuffle_pages=True),
]


@pytest.mark.parametrize("wl", CASES, ids=["decode_ragged", "decode_4heads", "prefill_grouped"])
def test_k8_scores_exact(wl):
    inp = di.make_inputs(wl)
    k8 = di.with_fp8_keys(inp, seed=wl.seed)
    t = upload(inp)
    got = _scores(inp, t, _k8_tensors(k8))
    ref = orc.dsa_prefill(k8) if wl.mode == "prefill" else orc.dsa_decode(k8)
    lens = row_lengths(inp)
    for r, res in ref.items():
        n = int(lens[r])
        assert np.array_equal(got[r, :n].astype(np.float64), res["scores"]), f"row {r}"
    # the same keys held as bf16 give the same scores, bit for bit
    bf = _scores(inp, t)
    for r in range(len(lens)):
        n = int(lens[r])
        assert np.array_equal(got[r, :n], bf[r, :n])


@pytest.mark.parametrize("wl", CASES[:2], ids=["decode_ragged", "decode_4heads"])
def test_k8_forward_matches_oracle_and_bf16_path(wl):
    inp = di.make_inputs(wl)
    k8 = di.with_fp8_keys(inp, seed=wl.seed + 1)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    n_q, k, H, R = dims.n_q, dims.topk, dims.H, dims.R
    idx = torch.full((n_q, k), -7, dtype=torch.int32, device="cuda")
    out = torch.full((n_q, H, R), float("nan"), device="cuda")
    lse = torch.full((n_q, H), float("nan"), device="cuda")
    ws = dsa.workspace(dsa.OP_ATTENTION_FORWARD_K8, dims, cache)
    k8p, ks = _k8_tensors(k8)
    dsa.dsa_attention_forward_k8(t["q_idx"], t["w"], k8p, ks, t["q"], t["latent_pages"], cache,
                                 dims, idx, out, lse, ws)
    st, info = dsa.workspace_check(ws)
    assert st == 0, (st, hex(info))
    idx, out, lse = idx.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy()
    for r, res in orc.dsa_decode(k8).items():
        assert_row_matches(r, res, idx, out, lse)
    bidx, bout, blse = run_forward(inp, t)
    assert np.array_equal(idx, bidx) and np.array_equal(out, bout) and np.array_equal(lse, blse)


def test_k8_long_rows_full_size():
    # the 4 x 131,072 decode with FP8 keys: every index and sampled outputs
    wl = di.CONFIGS["glm5_decode_4x128k"]
    inp = di.make_inputs(wl)
    k8 = di.with_fp8_keys(inp, seed=7)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    idx = torch.empty((dims.n_q, dims.topk), dtype=torch.int32, device="cuda")
    out = torch.empty((dims.n_q, dims.H, dims.R), device="cuda")
    lse = torch.empty((dims.n_q, dims.H), device="cuda")
    ws = dsa.workspace(dsa.OP_ATTENTION_FORWARD_K8, dims, cache)
    k8p, ks = _k8_tensors(k8)
    dsa.dsa_attention_forward_k8(t["q_idx"], t["w"], k8p, ks, t["q"], t["latent_pages"], cache,
                                 dims, idx, out, lse, ws)
    assert dsa.workspace_check(ws)[0] == 0
    idx, out, lse = idx.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy()
    for r in (0, 3):
        res = orc.dsa_decode(k8, rows=[r])[r]
        assert_row_matches(r, res, idx, out, lse)


def test_k8_query_terms_carry_bf16_queries():
    # normal (non-integer) bf16 queries within the carried range: the FP8-key
    # scores equal the oracle's to fp32 rounding, and the selection is the same
    wl = di.small_decode([3000, 777], H_I=32, D_I=128, topk=256, H=4, R=64, P=16, seed=54)
    inp = di.make_inputs(wl)
    rng = np.random.default_rng(9)
    q = rng.standard_normal(inp["q_idx"].shape).astype(np.float32)
    q = np.where(np.abs(q) < 2.0 ** -8, 0.0, q).astype(np.float32)   # inside the carried range
    inp = dict(inp, q_idx=di.f32_to_bf16_bits(q))
    k8 = di.with_fp8_keys(inp, seed=4)
    t = upload(inp)
    got = _scores(inp, t, _k8_tensors(k8))
    for r, res in orc.dsa_decode(k8).items():
        n = int(inp["seq_lens"][r])
        ref = res["scores"]
        assert np.max(np.abs(got[r, :n] - ref)) <= 1e-5 * np.max(np.abs(ref)), r
