"""Pins of the float64 oracle to facts outside itself (no GPU needed).

Each test checks the oracle against something its own code does not restate:
hand-derived golden values, closed forms, brute force over every subset on
tiny inputs, the stable-argsort rule the pages name, algebraic identities
(dense == sparse below the top-k size, absorbed == non-absorbed attention),
and special cases.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import dsa_oracle as orc
import dsa_inputs as di


def _num(x):
    table = {"ln3": math.log(3.0), "ln4": math.log(4.0), "ln2": math.log(2.0),
             "ln5": math.log(5.0), "ln(1+e2)": math.log(1.0 + math.e ** 2),
             "2e2/(1+e2)": 2.0 * math.e ** 2 / (1.0 + math.e ** 2)}
    return table[x] if isinstance(x, str) else float(x)


def _arr(v):
    return np.array([[_num(x) for x in row] for row in v], dtype=np.float64)


# ---------------------------------------------------------------- indexer

def test_indexer_hand_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "indexer_hand.json")))
    s = orc.indexer_scores(np.array(g["q_idx"], float), np.array(g["w"], float),
                           np.array(g["keys"], float))
    assert s.tolist() == [float(x) for x in g["scores"]]
    for k, want in g["topk"].items():
        assert orc.topk_select(s, int(k)).tolist() == want


def test_indexer_relu_odd_part_identity():
    # relu(x) - relu(-x) = x, so score(q) - score(-q) = sum_h w_h (q_h . k):
    # a dropped ReLU, a wrong sign or a transposed operand breaks it.
    rng = np.random.default_rng(11)
    q = rng.standard_normal((5, 9))
    w = rng.standard_normal(5)
    k = rng.standard_normal((13, 9))
    lhs = orc.indexer_scores(q, w, k) - orc.indexer_scores(-q, w, k)
    rhs = np.array([sum(w[h] * sum(q[h, d] * k[s, d] for d in range(9)) for h in range(5))
                    for s in range(13)])
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-12)


def test_indexer_one_hot_weight_selects_head():
    rng = np.random.default_rng(12)
    q = rng.integers(-3, 4, (4, 6)).astype(float)
    k = rng.integers(-3, 4, (10, 6)).astype(float)
    for h in range(4):
        w = np.zeros(4)
        w[h] = 1.0
        want = [max(0.0, float(np.dot(q[h], k[s]))) for s in range(10)]
        assert orc.indexer_scores(q, w, k).tolist() == want


def test_indexer_positive_homogeneity_and_nonnegativity():
    rng = np.random.default_rng(13)
    q = rng.standard_normal((3, 8))
    k = rng.standard_normal((20, 8))
    w = rng.uniform(0, 2, 3)
    s = orc.indexer_scores(q, w, k)
    assert (s >= 0).all()          # w >= 0 and ReLU >= 0
    np.testing.assert_allclose(orc.indexer_scores(2.5 * q, w, k), 2.5 * s, rtol=1e-13)


# ---------------------------------------------------------------- top-k

def _brute_force_topk(scores, k):
    """The unique size-k subset S with: every kept token beats every dropped one
    (higher score, or equal score and lower index)."""
    n = len(scores)
    if n <= k:
        return list(range(n))
    hits = []
    for sub in itertools.combinations(range(n), k):
        kept = set(sub)
        ok = all(scores[s] > scores[t] or (scores[s] == scores[t] and s < t)
                 for s in kept for t in range(n) if t not in kept)
        if ok:
            hits.append(list(sub))
    assert len(hits) == 1
    return hits[0]


@pytest.mark.parametrize("seed", range(40))
def test_topk_brute_force_tiny(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 11))
    k = int(rng.integers(1, 9))
    scores = rng.integers(0, 4, n).astype(float)   # few values -> many ties
    want = _brute_force_topk(scores.tolist(), k)
    got = orc.topk_select(scores, k)
    assert got[got >= 0].tolist() == want
    assert (got[len(want):] == -1).all()


@pytest.mark.parametrize("seed", range(10))
def test_topk_matches_stable_argsort(seed):
    # the exact library rule the pages name: argsort(-scores, kind='stable')
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(300, 3000))
    k = int(rng.integers(1, 400))
    scores = rng.integers(-5, 6, n).astype(float) * 0.25
    want = np.sort(np.argsort(-scores, kind="stable")[:k]).tolist()
    want += [-1] * (k - len(want))
    assert orc.topk_select(scores, k).tolist() == want


def test_topk_invariants_and_special_cases():
    rng = np.random.default_rng(7)
    scores = rng.standard_normal(5000)
    scores[::7] = 0.0
    sel = orc.topk_select(scores, 300)
    assert len(sel) == 300 and (np.diff(sel) > 0).all()
    kept = set(sel.tolist())
    lo_kept = min(scores[s] for s in kept)
    hi_drop = max(scores[t] for t in range(5000) if t not in kept)
    assert lo_kept >= hi_drop
    # N <= K keeps everything, ascending, padded with -1
    assert orc.topk_select([3.0, 1.0, 2.0], 5).tolist() == [0, 1, 2, -1, -1]
    assert orc.topk_select([], 3).tolist() == [-1, -1, -1]
    # -0.0 and +0.0 are equal scores: the lower index wins
    assert orc.topk_select([-0.0, 0.0, -1.0], 1).tolist() == [0]
    assert orc.topk_select([-1.0, 0.0, -0.0], 1).tolist() == [1]
    # all equal: the first k
    assert orc.topk_select([1.5] * 10, 4).tolist() == [0, 1, 2, 3]


def test_topk_few_indexer_heads_tie_case():
    # two indexer heads whose ReLU zeroes every head for many keys: many exact
    # ties at score 0 (the failure the pages describe); ties go to lower index
    rng = np.random.default_rng(5)
    q = rng.integers(-3, 4, (2, 16)).astype(float)
    k = rng.integers(-3, 4, (400, 16)).astype(float)
    w = np.array([1.0, 2.0])
    s = orc.indexer_scores(q, w, k)
    assert (s == 0).sum() > 50
    want = np.sort(np.argsort(-s, kind="stable")[:200])
    assert orc.topk_select(s, 200).tolist() == want.tolist()


# ---------------------------------------------------------------- attention

def test_mla_hand_golden(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "mla_hand.json")))
    for case in g["cases"]:
        out, lse, p = orc.mla_attention(_arr(case["q"]), _arr(case["rows"]), case["R"],
                                        case["scale"])
        np.testing.assert_allclose(out, _arr(case["out"]), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse, [_num(x) for x in case["lse"]], rtol=1e-12)
        np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=1e-14)


def test_mla_softmax_sums_to_one_and_bounds():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((6, 40)) * 3
    rows = rng.standard_normal((77, 40))
    out, lse, p = orc.mla_attention(q, rows, 32, 0.3)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=1e-13)
    assert (p >= 0).all()
    # a convex combination stays inside the per-column range of the values
    assert (out <= rows[:, :32].max(axis=0) + 1e-12).all()
    assert (out >= rows[:, :32].min(axis=0) - 1e-12).all()
    # lse >= max logit and <= max logit + log n
    z = 0.3 * q @ rows.T
    assert (lse >= z.max(axis=1) - 1e-12).all()
    assert (lse <= z.max(axis=1) + math.log(77) + 1e-12).all()


def test_mla_single_key_and_zero_query():
    rng = np.random.default_rng(4)
    rows = rng.standard_normal((1, 12))
    q = rng.standard_normal((3, 12))
    out, lse, _ = orc.mla_attention(q, rows, 8, 0.7)
    np.testing.assert_allclose(out, np.repeat(rows[:, :8], 3, axis=0), rtol=1e-14)
    np.testing.assert_allclose(lse, 0.7 * (q @ rows[0]), rtol=1e-13)
    rows = rng.standard_normal((9, 12))
    out, lse, _ = orc.mla_attention(np.zeros((2, 12)), rows, 8, 0.7)
    np.testing.assert_allclose(out, np.repeat(rows[:, :8].mean(axis=0, keepdims=True), 2, 0),
                               rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(lse, math.log(9), rtol=1e-14)


def test_sparse_equals_dense_below_k():
    # below K tokens the selection keeps everything, so the sparse step must
    # equal dense MLA attention computed by an independent routine
    wl = di.small_decode([40, 63, 64, 100], H_I=2, D_I=16, topk=128, H=3, R=16, P=8,
                         seed=9)
    inp = di.make_inputs(wl)
    res = orc.dsa_decode(inp)
    for b, n in enumerate(wl.seq_lens):
        lat = orc.bf16_to_f64(orc.gather_paged_rows(inp["latent_pages"],
                                                    inp["block_table"][b], range(n)))
        out, lse = orc.dense_mla_attention(orc.bf16_to_f64(inp["q"][b]), lat, wl.R, wl.scale)
        assert res[b]["idx"][:n].tolist() == list(range(n))
        np.testing.assert_allclose(res[b]["out"], out, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(res[b]["lse"], lse, rtol=1e-12)


def test_absorbed_equals_nonabsorbed():
    rng = np.random.default_rng(21)
    H, R, P, d_nope, d_v, n = 4, 32, 8, 16, 12, 50
    W_UK = rng.standard_normal((H, d_nope, R)) / math.sqrt(R)
    W_UV = rng.standard_normal((H, R, d_v)) / math.sqrt(R)
    q_nope = rng.standard_normal((H, d_nope))
    q_rope = rng.standard_normal((H, P))
    c_kv = rng.standard_normal((n, R))
    k_rope = rng.standard_normal((n, P))
    scale = 1.0 / math.sqrt(d_nope + P)
    ref_out, ref_lse = orc.mla_attention_nonabsorbed(q_nope, q_rope, c_kv, k_rope,
                                                     W_UK, W_UV, scale)
    q_abs = orc.absorb_query(q_nope, q_rope, W_UK)
    lat_out, lse, _ = orc.mla_attention(q_abs, np.concatenate([c_kv, k_rope], 1), R, scale)
    out = orc.project_values(lat_out, W_UV)
    np.testing.assert_allclose(out, ref_out, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12)


def test_sparse_attends_only_selected_rows():
    # perturbing a latent row that was not selected leaves the output unchanged;
    # perturbing a selected one changes it
    wl = di.small_decode([700], H_I=2, D_I=16, topk=32, H=2, R=16, P=8, seed=4,
                         shuffle_pages=False)
    inp = di.make_inputs(wl)
    base = orc.dsa_decode(inp)[0]
    sel = set(base["idx"].tolist())
    drop = next(t for t in range(700) if t not in sel)
    keep = next(iter(sel))
    for tok, changes in ((drop, False), (keep, True)):
        mod = dict(inp)
        lat = inp["latent_pages"].copy()
        lat[tok // 64, tok % 64, :] = di.f32_to_bf16_bits(np.full(wl.W, 3.0, np.float32))
        mod["latent_pages"] = lat
        r = orc.dsa_decode(mod)[0]
        assert np.array_equal(r["idx"], base["idx"])
        assert (not np.array_equal(r["out"], base["out"])) == changes


# ---------------------------------------------------------------- cache append

def _new_rows(n, width, seed):
    rng = np.random.default_rng(seed)
    return di.f32_to_bf16_bits(rng.standard_normal((n, width)).astype(np.float32))


def test_append_reads_back_through_the_block_table():
    wl = di.small_decode([300, 129, 64, 1000], H_I=2, D_I=16, topk=32, H=2, R=16, P=8, seed=3,
                         shuffle_pages=True)
    inp = di.make_inputs(wl)
    pos = orc.append_positions(inp)
    assert pos == [(b, n - 1) for b, n in enumerate(wl.seq_lens)]
    k_new, l_new = _new_rows(4, wl.D_I, 1), _new_rows(4, wl.W, 2)
    kp, lp = orc.cache_append(inp["k_pages"], inp["latent_pages"], inp["block_table"], pos,
                              k_new, l_new)
    for b, n in enumerate(wl.seq_lens):
        old = orc.gather_paged_rows(inp["latent_pages"], inp["block_table"][b], range(n))
        new = orc.gather_paged_rows(lp, inp["block_table"][b], range(n))
        assert np.array_equal(new[:n - 1], old[:n - 1])   # earlier tokens untouched
        assert np.array_equal(new[n - 1], l_new[b])       # the new token at its position
        newk = orc.gather_paged_rows(kp, inp["block_table"][b], [n - 1])
        assert np.array_equal(newk[0], k_new[b])
    # exactly one row per appended token changed in each pool
    assert (kp != inp["k_pages"]).any(axis=2).sum() == 4
    assert (lp != inp["latent_pages"]).any(axis=2).sum() == 4


def test_append_round_trip_restores_the_step():
    # blank the current tokens' rows, append them again: the pools and the
    # step's result are what they were
    wl = di.small_decode([200, 65], H_I=2, D_I=16, topk=16, H=2, R=16, P=8, seed=5,
                         shuffle_pages=True)
    inp = di.make_inputs(wl)
    pos = orc.append_positions(inp)
    k_cur = np.stack([orc.gather_paged_rows(inp["k_pages"], inp["block_table"][b], [p])[0]
                      for b, p in pos])
    l_cur = np.stack([orc.gather_paged_rows(inp["latent_pages"], inp["block_table"][b], [p])[0]
                      for b, p in pos])
    blank = dict(inp)
    blank["k_pages"], blank["latent_pages"] = orc.cache_append(
        inp["k_pages"], inp["latent_pages"], inp["block_table"], pos,
        np.zeros_like(k_cur), np.zeros_like(l_cur))
    kp, lp = orc.cache_append(blank["k_pages"], blank["latent_pages"], inp["block_table"], pos,
                              k_cur, l_cur)
    assert np.array_equal(kp, inp["k_pages"]) and np.array_equal(lp, inp["latent_pages"])
    again = dict(inp, k_pages=kp, latent_pages=lp)
    r0, r1 = orc.dsa_decode(inp), orc.dsa_decode(again)
    for b in r0:
        assert np.array_equal(r0[b]["idx"], r1[b]["idx"])
        np.testing.assert_array_equal(r0[b]["out"], r1[b]["out"])


def test_append_prefill_positions_and_checks():
    wl = di.small_prefill(70, q_pos0=10, H_I=2, D_I=16, topk=16, H=2, R=16, P=8, seed=2)
    inp = di.make_inputs(wl)
    pos = orc.append_positions(inp)
    assert pos == [(0, 10 + t) for t in range(70)]
    k_new, l_new = _new_rows(70, wl.D_I, 3), _new_rows(70, wl.W, 4)
    kp, lp = orc.cache_append(inp["k_pages"], inp["latent_pages"], inp["block_table"], pos,
                              k_new, l_new)
    got = orc.gather_paged_rows(lp, inp["block_table"][0], range(10, 80))
    assert np.array_equal(got, l_new)
    with pytest.raises(ValueError):
        orc.cache_append(inp["k_pages"], inp["latent_pages"], inp["block_table"],
                         [(0, inp["block_table"].shape[1] * 64)], k_new[:1], l_new[:1])
    bad = inp["block_table"].copy()
    bad[0, 0] = inp["k_pages"].shape[0]
    with pytest.raises(ValueError):
        orc.cache_append(inp["k_pages"], inp["latent_pages"], bad, [(0, 0)], k_new[:1],
                         l_new[:1])


# ---------------------------------------------------------------- whole step

def test_step_keeps_the_best_scored_tokens():
    # the whole step: the kept set is the stable-argsort head of its own
    # indexer scores, and the output is dense attention over exactly those rows
    wl = di.small_decode([300, 97], H_I=3, D_I=16, topk=64, H=2, R=16, P=8, seed=14)
    inp = di.make_inputs(wl)
    res = orc.dsa_decode(inp)
    for b, n in enumerate(wl.seq_lens):
        r = res[b]
        want = np.sort(np.argsort(-r["scores"], kind="stable")[:wl.topk]).tolist()
        got = r["idx"][r["idx"] >= 0].tolist()
        assert got == want
        lat = orc.bf16_to_f64(orc.gather_paged_rows(inp["latent_pages"],
                                                    inp["block_table"][b], want))
        out, lse = orc.dense_mla_attention(orc.bf16_to_f64(inp["q"][b]), lat, wl.R, wl.scale)
        np.testing.assert_allclose(r["out"], out, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(r["lse"], lse, rtol=1e-12)


def test_prefill_row_equals_decode_at_same_position():
    # cached decode == full-prefix forward: prefill row t must equal a decode
    # query at position t over the same cache
    wl = di.small_prefill(150, q_pos0=10, H_I=2, D_I=16, topk=48, H=2, R=16, P=8, seed=6)
    inp = di.make_inputs(wl)
    rows = [0, 37, 38, 100, 149]
    pre = orc.dsa_prefill(inp, rows)
    for t in rows:
        dec = dict(inp)
        dec["q_idx"] = inp["q_idx"][t:t + 1]
        dec["w"] = inp["w"][t:t + 1]
        dec["q"] = inp["q"][t:t + 1]
        dec["seq_lens"] = np.array([wl.q_pos0 + t + 1], np.int32)
        d = orc.dsa_decode(dec)[0]
        assert np.array_equal(d["idx"], pre[t]["idx"])
        np.testing.assert_array_equal(d["out"], pre[t]["out"])


def test_paging_is_transparent():
    # the same logical token data through a shuffled block table gives the
    # same result as through the identity table
    wl = di.small_decode([300, 129], H_I=2, D_I=16, topk=40, H=2, R=16, P=8, seed=8,
                         shuffle_pages=True)
    inp = di.make_inputs(wl)
    res = orc.dsa_decode(inp)
    flat = dict(inp)
    kp, lp, bt = [], [], np.full_like(inp["block_table"], -1)
    nxt = 0
    for b, n in enumerate(wl.seq_lens):
        for j in range(di.pages_needed(n)):
            kp.append(inp["k_pages"][inp["block_table"][b, j]])
            lp.append(inp["latent_pages"][inp["block_table"][b, j]])
            bt[b, j] = nxt
            nxt += 1
    flat.update(k_pages=np.stack(kp), latent_pages=np.stack(lp), block_table=bt)
    res2 = orc.dsa_decode(flat)
    for b in range(2):
        assert np.array_equal(res[b]["idx"], res2[b]["idx"])
        np.testing.assert_array_equal(res[b]["out"], res2[b]["out"])


def test_integer_config_scores_are_exact_integers():
    wl = di.CONFIGS["tiny_decode"]
    inp = di.make_inputs(wl)
    r = orc.dsa_decode(inp)[0]
    s = r["scores"]
    assert np.array_equal(s, np.round(s)) and s.max() < 2 ** 24
    assert (r["idx"] >= 0).all() and len(r["idx"]) == wl.topk


# ---------------------------------------------------------------- bf16

def test_bf16_widening_all_encodings():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mine = orc.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(mine[ok], ref[ok])
    np.testing.assert_array_equal(np.signbit(mine[ok]), np.signbit(ref[ok]))


# ---------------------------------------------------------------- FP8 index keys

def test_e4m3_decoding_all_encodings():
    codes = np.arange(256, dtype=np.uint8)
    mine = orc.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(mine[ok], ref[ok])
    np.testing.assert_array_equal(np.signbit(mine[ok]), np.signbit(ref[ok]))
    # a few by hand: 1.0, -2.0, 448 (largest), 2^-9 (smallest subnormal)
    assert orc.e4m3_to_f64(np.array([0x38, 0xC0, 0x7E, 0x01], np.uint8)).tolist() == \
        [1.0, -2.0, 448.0, 2.0 ** -9]


def test_fp8_keys_stand_for_the_same_keys_and_scores():
    wl = di.small_decode([300, 129], H_I=4, D_I=64, topk=32, H=2, R=16, P=8, seed=31,
                         shuffle_pages=True)
    inp = di.make_inputs(wl)
    k8 = di.with_fp8_keys(inp, seed=3)
    assert k8["k8_pages"].dtype == np.uint8 and k8["k_scale"].shape == (inp["k_pages"].shape[0] * 64,)
    assert len(set(k8["k_scale"].tolist())) > 1          # the scales vary per token
    deq = orc.dequantize_keys(k8["k8_pages"].reshape(-1, wl.D_I), k8["k_scale"])
    np.testing.assert_array_equal(deq, orc.bf16_to_f64(inp["k_pages"]).reshape(-1, wl.D_I))
    r_bf, r_k8 = orc.dsa_decode(inp), orc.dsa_decode(k8)
    for b in r_bf:
        np.testing.assert_array_equal(r_bf[b]["scores"], r_k8[b]["scores"])
        assert np.array_equal(r_bf[b]["idx"], r_k8[b]["idx"])


def test_fp8_key_scale_is_a_factor_of_the_score():
    # a positive per-token scale comes out of the ReLU and the head sum
    rng = np.random.default_rng(41)
    q = rng.standard_normal((3, 16))
    w = rng.uniform(0, 2, 3)
    codes = rng.integers(0, 256, (20, 16)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0                      # no NaN codes
    scale = rng.uniform(0.1, 4.0, 20)
    s1 = orc.indexer_scores(q, w, orc.dequantize_keys(codes, np.ones(20)))
    s2 = orc.indexer_scores(q, w, orc.dequantize_keys(codes, scale))
    np.testing.assert_allclose(s2, scale * s1, rtol=1e-12)


# ---------------------------------------------------------------- FP8 latent cache

def test_fp8_latent_stands_for_the_same_latent_and_attention():
    # codes of x * 2^j with scale 2^-j stand for the latent x exactly, so the
    # whole step over the FP8 cache equals the step over the bf16 cache
    wl = di.small_decode([300, 129], H_I=4, D_I=32, topk=64, H=3, R=64, P=16, seed=33,
                         shuffle_pages=True)
    inp = di.with_fp8_latent(di.make_inputs(wl), seed=5)
    assert inp["latent8_pages"].dtype == np.uint8
    assert inp["latent_scale"].shape == (inp["latent_pages"].shape[0] * 64,)
    assert len(set(inp["latent_scale"].tolist())) > 1      # the scales vary per token
    W = wl.R + wl.P
    deq = orc.dequantize_latent(inp["latent8_pages"].reshape(-1, W), inp["latent_scale"])
    np.testing.assert_array_equal(deq, orc.bf16_to_f64(inp["latent_pages"]).reshape(-1, W))
    bf = {k: v for k, v in inp.items() if k not in ("latent8_pages", "latent_scale")}
    r_bf, r_l8 = orc.dsa_decode(bf), orc.dsa_decode(inp)
    for b in r_bf:
        assert np.array_equal(r_bf[b]["idx"], r_l8[b]["idx"])
        np.testing.assert_array_equal(r_bf[b]["out"], r_l8[b]["out"])
        np.testing.assert_array_equal(r_bf[b]["lse"], r_l8[b]["lse"])


def test_fp8_latent_single_token_closed_form():
    # one selected token: out is its dequantized c_kv part, lse its logit
    rng = np.random.default_rng(43)
    codes = rng.integers(0, 256, (1, 40)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0                      # no NaN codes
    scale = np.array([0.375])
    q = rng.standard_normal((2, 40))
    row = orc.dequantize_latent(codes, scale)
    out, lse, p = orc.mla_attention(q, row, 32, 0.5)
    np.testing.assert_array_equal(out, np.repeat(0.375 * orc.e4m3_to_f64(codes[:, :32]), 2, axis=0))
    np.testing.assert_allclose(lse, 0.5 * (q @ (0.375 * orc.e4m3_to_f64(codes[0]))), rtol=1e-12)
    assert np.all(p == 1.0)


# ---------------------------------------------------------------- context-parallel decode

@pytest.mark.parametrize("ranks", [2, 3, 5])
def test_context_parallel_equals_one_gpu_decode(ranks):
    # split one sequence's keys over ranks: local top-k, global merge of the
    # candidates, each rank's attention over its own kept keys, LSE merge ==
    # the one-device step (indices exactly)
    wl = di.small_decode([1500], H_I=4, D_I=32, topk=200, H=3, R=16, P=8, seed=61)
    inp = di.make_inputs(wl)
    ref = orc.dsa_decode(inp)[0]
    n = wl.seq_lens[0]
    bounds = np.linspace(0, n, ranks + 1).astype(int)
    cs, ci = [], []
    for r in range(ranks):
        s_r, i_r = orc.cp_local_candidates(ref["scores"][bounds[r]:bounds[r + 1]], wl.topk,
                                           int(bounds[r]))
        cs.append(s_r)
        ci.append(i_r)
    gidx = orc.cp_merge_candidates(np.stack(cs), np.stack(ci), wl.topk)
    assert np.array_equal(gidx, ref["idx"])
    q = orc.bf16_to_f64(inp["q"][0])
    outs, lses = [], []
    for r in range(ranks):
        own = gidx[(gidx >= bounds[r]) & (gidx < bounds[r + 1])]
        if len(own) == 0:
            outs.append(np.zeros((wl.H, wl.R)))
            lses.append(np.full(wl.H, -np.inf))
            continue
        rows = orc.bf16_to_f64(orc.gather_paged_rows(inp["latent_pages"], inp["block_table"][0], own))
        o, l, _ = orc.mla_attention(q, rows, wl.R, wl.scale)
        outs.append(o)
        lses.append(l)
    out, lse = orc.cp_merge_partials(outs, lses)
    np.testing.assert_allclose(out, ref["out"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, ref["lse"], rtol=1e-12)


def test_cp_merge_candidates_tie_rule_across_ranks():
    # equal scores on two ranks: the lower global index (the earlier rank) wins
    s = np.array([[5.0, 3.0, -np.inf], [5.0, 3.0, 3.0]])
    i = np.array([[2, 7, -1], [10, 11, 12]])
    assert orc.cp_merge_candidates(s, i, 3).tolist() == [2, 7, 10]
    assert orc.cp_merge_candidates(s, i, 4).tolist() == [2, 7, 10, 11]
    assert orc.cp_merge_candidates(s, i, 9).tolist() == [2, 7, 10, 11, 12, -1, -1, -1, -1]
