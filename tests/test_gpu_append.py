"""Cache append on the GPU against the oracle's append (byte-exact), and the
appended caches through the whole step."""

import numpy as np
import pytest
import torch

import dsa_inputs as di
import sparse_attention_scores_b200 as dsa
from oracle import dsa_oracle as orc
from dsa_testutil import bf16_tensor, upload, cache_of, dims_of, run_forward, assert_row_matches

pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _new_rows(n, width, seed):
    rng = np.random.default_rng(seed)
    return di.f32_to_bf16_bits(rng.standard_normal((n, width)).astype(np.float32))


def _append(inp, t, k_new, l_new):
    cache, dims = cache_of(inp, t), dims_of(inp)
    ws = dsa.workspace(dsa.OP_CACHE_APPEND, dims, cache)
    dsa.dsa_cache_append(bf16_tensor(k_new), bf16_tensor(l_new), t["k_pages"], t["latent_pages"],
                         cache, dims, ws)
    return dsa.workspace_check(ws)


@pytest.mark.parametrize("wl", [
    di.small_decode([300, 129, 64, 1000, 1], H_I=32, D_I=128, topk=64, H=64, R=512, P=64,
                    seed=11, shuffle_pages=True),
    di.small_decode([4096], H_I=4, D_I=32, topk=256, H=4, R=64, P=16, seed=12),
    di.small_prefill(300, q_pos0=37, H_I=32, D_I=128, topk=128, H=64, R=512, P=64, seed=13,
                     shuffle_pages=True),
], ids=["decode_ragged_shuffled", "decode_tiny_widths", "prefill"])
def test_append_matches_oracle_bytes(wl):
    inp = di.make_inputs(wl)
    t = upload(inp)
    n = wl.n_q
    k_new, l_new = _new_rows(n, wl.D_I, 1), _new_rows(n, wl.W, 2)
    st, info = _append(inp, t, k_new, l_new)
    assert st == 0, (st, hex(info))
    kp, lp = orc.cache_append(inp["k_pages"], inp["latent_pages"], inp["block_table"],
                              orc.append_positions(inp), k_new, l_new)
    assert np.array_equal(_bits(t["k_pages"]).reshape(kp.shape), kp)
    assert np.array_equal(_bits(t["latent_pages"]).reshape(lp.shape), lp)


def test_append_then_forward_matches_oracle():
    wl = di.small_decode([700, 2100, 64], H_I=32, D_I=128, topk=512, H=64, R=512, P=64, seed=14,
                         shuffle_pages=True)
    inp = di.make_inputs(wl)
    t = upload(inp)
    # integer-valued index keys keep the scores exact
    k_new = di.f32_to_bf16_bits(
        np.random.default_rng(5).integers(-3, 4, (3, wl.D_I)).astype(np.float32))
    l_new = _new_rows(3, wl.W, 4)
    st, info = _append(inp, t, k_new, l_new)
    assert st == 0, (st, hex(info))
    kp, lp = orc.cache_append(inp["k_pages"], inp["latent_pages"], inp["block_table"],
                              orc.append_positions(inp), k_new, l_new)
    ref_inp = dict(inp, k_pages=kp, latent_pages=lp)
    idx, out, lse = run_forward(ref_inp, t)
    for r, res in orc.dsa_decode(ref_inp).items():
        assert_row_matches(r, res, idx, out, lse)


def test_append_bad_page_is_reported_and_skipped():
    wl = di.small_decode([200, 300], H_I=4, D_I=32, topk=64, H=4, R=64, P=16, seed=15)
    inp = di.make_inputs(wl)
    bt = inp["block_table"].copy()
    bt[1, (300 - 1) // 64] = inp["k_pages"].shape[0]   # row 1's append page is out of range
    inp = dict(inp, block_table=bt)
    t = upload(inp)
    before_k, before_l = _bits(t["k_pages"]).copy(), _bits(t["latent_pages"]).copy()
    k_new, l_new = _new_rows(2, wl.D_I, 6), _new_rows(2, wl.W, 7)
    st, info = _append(inp, t, k_new, l_new)
    assert st == 6 and (info >> 24) == 5, (st, hex(info))
    # row 0 written, row 1 skipped
    kp, lp = orc.cache_append(inp["k_pages"], inp["latent_pages"], bt, [(0, 199)], k_new[:1],
                              l_new[:1])
    assert np.array_equal(_bits(t["k_pages"]).reshape(kp.shape), kp)
    assert np.array_equal(_bits(t["latent_pages"]).reshape(lp.shape), lp)
    assert (_bits(t["k_pages"]) != before_k).any() and (_bits(t["latent_pages"]) != before_l).any()
