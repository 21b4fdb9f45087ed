"""FP8 latent cache on the GPU: the sparse MLA step (decode, prefill) and the
whole step with both caches in FP8, against the float64 oracle over the
dequantized rows (scale * e4m3(code)), within the step's tolerances."""

import numpy as np
import pytest
import torch

import dsa_inputs as di
import sparse_attention_scores_b200 as dsa
from oracle import dsa_oracle as orc
from tests.dsa_testutil import LSE_TOL, OUT_TOL, assert_row_matches, cache_of, dims_of, norm_err, upload

pytestmark = pytest.mark.gpu


def _l8_tensors(inp):
    return (torch.from_numpy(inp["latent8_pages"]).cuda(),
            torch.from_numpy(inp["latent_scale"]).cuda())


def _random_codes_and_scales(inp, seed):
    """An FP8 latent cache with arbitrary (not power-of-two) per-token scales:
    random valid E4M3 codes (no NaN) and scales in [0.002, 0.05]."""
    rng = np.random.default_rng(seed)
    shape = inp["latent_pages"].shape
    codes = rng.integers(0, 256, shape).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x00
    out = dict(inp)
    out["latent8_pages"] = codes
    out["latent_scale"] = rng.uniform(0.002, 0.05, shape[0] * shape[1]).astype(np.float32)
    return out


def _selection(rng, lengths, k):
    idx = np.full((len(lengths), k), -1, np.int32)
    for r, n in enumerate(lengths):
        m = min(n, k)
        idx[r, :m] = np.sort(rng.choice(n, size=m, replace=False))
    return idx


def _check_rows(inp, sel, out, lse, rows, table_row_of, R, scale):
    q = orc.bf16_to_f64(inp["q"])
    W = inp["latent8_pages"].shape[2]
    for r in rows:
        s = sel[r][sel[r] >= 0]
        if len(s) == 0:
            assert (out[r] == 0).all() and np.isneginf(lse[r]).all()
            continue
        tr = table_row_of(r)
        codes = orc.gather_paged_rows(inp["latent8_pages"], tr, s)
        scales = orc.gather_paged_rows(inp["latent_scale"].reshape(-1, 64, 1), tr, s)
        rows_f = orc.dequantize_latent(codes.reshape(-1, W), scales.reshape(-1))
        ref_out, ref_lse, _ = orc.mla_attention(q[r], rows_f, R, scale)
        assert norm_err(out[r], ref_out) <= OUT_TOL, r
        assert np.max(np.abs(lse[r] - ref_lse)) <= LSE_TOL, r


# Both MLA kernels take E4M3 rows; the batch decides which one runs (the
# per-chunk kernel for a few rows, the pipelined one for many).
@pytest.mark.parametrize("shape,batch", [
    (dict(H=64, R=512, P=64, k=2048), 5),    # per-chunk: 16 splits through the merge kernel
    (dict(H=64, R=512, P=64, k=1024), 12),   # per-chunk: 8 splits merged in a cluster
    (dict(H=64, R=512, P=64, k=2048), 32),   # pipelined: clusters of 4
    (dict(H=64, R=512, P=64, k=256), 160),   # pipelined: one CTA per row
    (dict(H=64, R=512, P=64, k=8192), 1),    # per-chunk: 64 splits through the merge kernel
    (dict(H=4, R=64, P=16, k=256), 7),       # per-chunk: a narrow row, 4 splits in a cluster
    (dict(H=16, R=192, P=32, k=300), 9),     # per-chunk: a ragged last column block and top-k
], ids=["chunk_b5", "chunk_c8_b12", "pipe_c4_b32", "pipe_b160", "chunk_b1_k8192", "chunk_tiny_b7",
        "chunk_r192_b9"])
def test_sparse_mla_decode_l8(shape, batch):
    rng = np.random.default_rng(batch + shape["k"])
    lengths = rng.integers(1, 3 * shape["k"], size=batch).tolist()
    wl = di.small_decode(lengths, H_I=4, D_I=32, topk=shape["k"], H=shape["H"], R=shape["R"],
                         P=shape["P"], seed=batch + 3, shuffle_pages=True)
    inp = _random_codes_and_scales(di.make_inputs(wl), seed=batch)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    sel = _selection(rng, lengths, shape["k"])
    if batch > 2:
        sel[batch // 2, :] = -1   # a row that keeps nothing
    idx = torch.from_numpy(sel).cuda()
    out = torch.full((batch, wl.H, wl.R), float("nan"), device="cuda")
    lse = torch.full((batch, wl.H), float("nan"), device="cuda")
    ws = dsa.workspace(dsa.OP_SPARSE_MLA_DECODE, dims, cache)
    l8, ls = _l8_tensors(inp)
    dsa.dsa_sparse_mla_decode_l8(t["q"], l8, ls, cache, idx, dims, out, lse, ws)
    assert dsa.workspace_check(ws)[0] == 0
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    _check_rows(inp, sel, out, lse, range(batch), lambda r: inp["block_table"][r], wl.R, wl.scale)


def test_sparse_mla_prefill_l8():
    T, k = 300, 128
    wl = di.small_prefill(T, q_pos0=0, H_I=4, D_I=32, topk=k, H=64, R=512, P=64, seed=4)
    inp = _random_codes_and_scales(di.make_inputs(wl), seed=11)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    sel = _selection(np.random.default_rng(1), [r + 1 for r in range(T)], k)
    idx = torch.from_numpy(sel).cuda()
    out = torch.full((T, wl.H, wl.R), float("nan"), device="cuda")
    lse = torch.full((T, wl.H), float("nan"), device="cuda")
    ws = dsa.workspace(dsa.OP_SPARSE_MLA_PREFILL, dims, cache)
    l8, ls = _l8_tensors(inp)
    dsa.dsa_sparse_mla_prefill_l8(t["q"], l8, ls, cache, idx, dims, out, lse, ws)
    assert dsa.workspace_check(ws)[0] == 0
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    _check_rows(inp, sel, out, lse, [0, 1, 63, 64, 127, 128, 200, 299],
                lambda r: inp["block_table"][0], wl.R, wl.scale)


def test_fp8_latent_matches_bf16_latent_of_the_same_values():
    # with_fp8_latent's codes stand for exactly the bf16 latent it returns:
    # both latent formats give the oracle's result for that latent
    lengths = [5000, 2100, 777, 3000]
    wl = di.small_decode(lengths, H_I=32, D_I=128, topk=2048, H=64, R=512, P=64, seed=21,
                         shuffle_pages=True)
    inp = di.with_fp8_latent(di.make_inputs(wl), seed=8)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    sel = _selection(np.random.default_rng(2), lengths, wl.topk)
    idx = torch.from_numpy(sel).cuda()
    ws = dsa.workspace(dsa.OP_SPARSE_MLA_DECODE, dims, cache)
    res = {}
    for kind in ("bf16", "l8"):
        out = torch.empty((wl.n_q, wl.H, wl.R), device="cuda")
        lse = torch.empty((wl.n_q, wl.H), device="cuda")
        if kind == "bf16":
            dsa.dsa_sparse_mla_decode(t["q"], t["latent_pages"], cache, idx, dims, out, lse, ws)
        else:
            l8, ls = _l8_tensors(inp)
            dsa.dsa_sparse_mla_decode_l8(t["q"], l8, ls, cache, idx, dims, out, lse, ws)
        assert dsa.workspace_check(ws)[0] == 0
        res[kind] = (out.cpu().numpy(), lse.cpu().numpy())
    q = orc.bf16_to_f64(inp["q"])
    for b in range(wl.n_q):
        s = sel[b][sel[b] >= 0]
        rows = orc.bf16_to_f64(orc.gather_paged_rows(inp["latent_pages"], inp["block_table"][b], s))
        ref_out, ref_lse, _ = orc.mla_attention(q[b], rows, wl.R, wl.scale)
        for kind in res:
            assert norm_err(res[kind][0][b], ref_out) <= OUT_TOL, (kind, b)
            assert np.max(np.abs(res[kind][1][b] - ref_lse)) <= LSE_TOL, (kind, b)


@pytest.mark.parametrize("lengths", [[9000, 2048, 70000, 4097], [8192]], ids=["b4", "b1"])
def test_attention_forward_fp8(lengths):
    # both caches in FP8: indices exact and outputs within tolerance of the
    # oracle's step over the dequantized caches
    wl = di.small_decode(lengths, H_I=32, D_I=128, topk=2048, H=64, R=512, P=64, seed=12,
                         shuffle_pages=True)
    inp = di.with_fp8_latent(di.with_fp8_keys(di.make_inputs(wl), seed=6), seed=7)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    k8p = torch.from_numpy(inp["k8_pages"]).cuda()
    ks = torch.from_numpy(inp["k_scale"]).cuda()
    l8, ls = _l8_tensors(inp)
    idx = torch.full((wl.n_q, wl.topk), -7, dtype=torch.int32, device="cuda")
    out = torch.full((wl.n_q, wl.H, wl.R), float("nan"), device="cuda")
    lse = torch.full((wl.n_q, wl.H), float("nan"), device="cuda")
    ws = dsa.workspace(dsa.OP_ATTENTION_FORWARD_FP8, dims, cache)
    dsa.dsa_attention_forward_fp8(t["q_idx"], t["w"], k8p, ks, t["q"], l8, ls, cache, dims, idx,
                                  out, lse, ws)
    assert dsa.workspace_check(ws)[0] == 0
    idx, out, lse = idx.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy()
    for r, res in orc.dsa_decode(inp).items():
        assert_row_matches(r, res, idx, out, lse)
