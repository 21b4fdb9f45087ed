"""The absorption GEMMs on the GPU: the absorbed query and the value
projection against the oracle, and the whole non-absorbed attention block
(absorb -> step -> project) against the oracle's non-absorbed attention."""

import math

import numpy as np
import pytest
import torch

import dsa_inputs as di
import sparse_attention_scores_b200 as dsa
from oracle import dsa_oracle as orc
from dsa_testutil import bf16_tensor, upload, cache_of, dims_of, norm_err

pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _bf16_rne(x: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bits, round to nearest even (through an exact float32)."""
    return di.f32_to_bf16_bits(x.astype(np.float32))


def _ints(rng, shape, lo=-3, hi=4):
    return di.f32_to_bf16_bits(rng.integers(lo, hi, shape).astype(np.float32))


def _normal(rng, shape, scale=1.0):
    return di.f32_to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


@pytest.mark.parametrize("n,H,d_nope,R,P", [(1, 64, 128, 512, 64), (5, 64, 128, 512, 64),
                                            (300, 8, 128, 512, 64), (3, 4, 64, 128, 16),
                                            (17, 2, 256, 256, 0), (2, 4, 64, 64, 16),
                                            (9, 3, 128, 192, 32)])
def test_absorb_integer_inputs_bit_exact(n, H, d_nope, R, P):
    # integer inputs: fp32 accumulation is exact, so the only rounding is the
    # final bf16 one, which the oracle's exact result takes the same way
    rng = np.random.default_rng(n * 7 + R)
    qn, wk = _ints(rng, (n, H, d_nope)), _ints(rng, (H, d_nope, R))
    qr = _normal(rng, (n, H, P)) if P else None
    q_abs = torch.empty((n, H, R + P), dtype=torch.bfloat16, device="cuda")
    ws = dsa.status_workspace()
    dsa.dsa_absorb_query(bf16_tensor(qn), bf16_tensor(qr) if P else None, bf16_tensor(wk), q_abs,
                         ws)
    st, info = dsa.workspace_check(ws)
    assert st == 0, (st, hex(info))
    got = _bits(q_abs)
    for b in range(n):
        qp = orc.bf16_to_f64(qr[b]) if P else np.zeros((H, 0))
        ref = orc.absorb_query(orc.bf16_to_f64(qn[b]), qp, orc.bf16_to_f64(wk))
        assert np.array_equal(got[b, :, :R], _bf16_rne(ref[:, :R])), f"row {b}"
        if P:
            assert np.array_equal(got[b, :, R:], qr[b])


def test_absorb_normal_inputs_within_bf16_rounding():
    rng = np.random.default_rng(3)
    n, H, d_nope, R, P = 40, 64, 128, 512, 64
    qn, qr = _normal(rng, (n, H, d_nope)), _normal(rng, (n, H, P))
    wk = _normal(rng, (H, d_nope, R), 1 / math.sqrt(d_nope))
    q_abs = torch.empty((n, H, R + P), dtype=torch.bfloat16, device="cuda")
    ws = dsa.status_workspace()
    dsa.dsa_absorb_query(bf16_tensor(qn), bf16_tensor(qr), bf16_tensor(wk), q_abs, ws)
    assert dsa.workspace_check(ws)[0] == 0
    got = q_abs.float().cpu().numpy().astype(np.float64)
    for b in range(0, n, 7):
        ref = orc.absorb_query(orc.bf16_to_f64(qn[b]), orc.bf16_to_f64(qr[b]), orc.bf16_to_f64(wk))
        # each element within a bf16 rounding (half an ulp, 2^-9 relative) of
        # the exact value, plus the fp32 accumulation error near cancellations
        assert np.all(np.abs(got[b] - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-5)


@pytest.mark.parametrize("n,H,R,d_v", [(1, 64, 512, 128), (33, 64, 512, 128), (70, 3, 64, 256),
                                       (5, 16, 512, 512), (4, 2, 128, 64), (3, 5, 192, 192)])
def test_project_values_near_fp32(n, H, R, d_v):
    rng = np.random.default_rng(n + d_v)
    o = rng.standard_normal((n, H, R)).astype(np.float32)
    wv = _normal(rng, (H, R, d_v), 1 / math.sqrt(R))
    v = torch.full((n, H, d_v), float("nan"), device="cuda")
    ws = dsa.status_workspace()
    dsa.dsa_project_values(torch.from_numpy(o).cuda(), bf16_tensor(wv), v, ws)
    assert dsa.workspace_check(ws)[0] == 0
    got = v.cpu().numpy()
    W = orc.bf16_to_f64(wv)
    for b in range(n):
        ref = orc.project_values(o[b].astype(np.float64), W)
        assert norm_err(got[b], ref) <= 1e-4, b


def test_absorb_many_items_per_cta():
    # 1,000 rows of 64 heads: 512 (head, 128-row tile) items over the SMs, so
    # a CTA walks several items (weight tile kept, stage and accumulator rings
    # wrapping) and the last tile is ragged (104 rows)
    rng = np.random.default_rng(41)
    n, H, d_nope, R, P = 1000, 64, 128, 512, 64
    qn, qr = _ints(rng, (n, H, d_nope)), _normal(rng, (n, H, P))
    wk = _ints(rng, (H, d_nope, R))
    q_abs = torch.empty((n, H, R + P), dtype=torch.bfloat16, device="cuda")
    ws = dsa.status_workspace()
    dsa.dsa_absorb_query(bf16_tensor(qn), bf16_tensor(qr), bf16_tensor(wk), q_abs, ws)
    assert dsa.workspace_check(ws)[0] == 0
    got = _bits(q_abs)
    WK = orc.bf16_to_f64(wk)
    for b in list(range(0, n, 37)) + [127, 128, 895, 896, 999]:
        ref = orc.absorb_query(orc.bf16_to_f64(qn[b]), orc.bf16_to_f64(qr[b]), WK)
        assert np.array_equal(got[b, :, :R], _bf16_rne(ref[:, :R])), b
        assert np.array_equal(got[b, :, R:], qr[b]), b


def test_project_many_items_per_cta():
    # the projection's rings over several items per CTA and a ragged last tile
    rng = np.random.default_rng(42)
    n, H, R, d_v = 1000, 64, 512, 128
    o = rng.standard_normal((n, H, R)).astype(np.float32)
    wv = _normal(rng, (H, R, d_v), 1 / math.sqrt(R))
    v = torch.full((n, H, d_v), float("nan"), device="cuda")
    ws = dsa.status_workspace()
    dsa.dsa_project_values(torch.from_numpy(o).cuda(), bf16_tensor(wv), v, ws)
    assert dsa.workspace_check(ws)[0] == 0
    got = v.cpu().numpy()
    W = orc.bf16_to_f64(wv)
    for b in list(range(0, n, 37)) + [127, 128, 895, 896, 999]:
        ref = orc.project_values(o[b].astype(np.float64), W)
        assert norm_err(got[b], ref) <= 1e-4, b


def test_project_values_unaligned_output():
    # an output that is 4- but not 16-byte aligned takes scalar stores
    rng = np.random.default_rng(43)
    n, H, R, d_v = 130, 4, 128, 64
    o = rng.standard_normal((n, H, R)).astype(np.float32)
    wv = _normal(rng, (H, R, d_v), 1 / math.sqrt(R))
    buf = torch.full((n * H * d_v + 1,), float("nan"), device="cuda")
    v = buf[1:].view(n, H, d_v)
    ws = dsa.status_workspace()
    dsa.dsa_project_values(torch.from_numpy(o).cuda(), bf16_tensor(wv), v, ws)
    assert dsa.workspace_check(ws)[0] == 0
    assert np.isnan(buf[0].item())
    got = v.cpu().numpy()
    W = orc.bf16_to_f64(wv)
    for b in range(n):
        assert norm_err(got[b], orc.project_values(o[b].astype(np.float64), W)) <= 1e-4, b


def test_nonabsorbed_block_end_to_end():
    # q_nope, q_rope, W_UK, W_UV, caches -> absorb -> step -> project, against
    # the oracle's non-absorbed attention over the same selected tokens
    wl = di.small_decode([700, 2100, 3000], H_I=32, D_I=128, topk=512, H=64, R=512, P=64,
                         seed=21, scale=1 / math.sqrt(192))
    inp = di.make_inputs(wl)
    t = upload(inp)
    rng = np.random.default_rng(22)
    d_nope, d_v, n, H, R, P = 128, 128, wl.n_q, wl.H, wl.R, wl.P
    qn, qr = _normal(rng, (n, H, d_nope)), _normal(rng, (n, H, P))
    wk = _normal(rng, (H, d_nope, R), 1 / math.sqrt(d_nope))
    wv = _normal(rng, (H, R, d_v), 1 / math.sqrt(R))
    ws = dsa.status_workspace()
    q_abs = torch.empty((n, H, R + P), dtype=torch.bfloat16, device="cuda")
    dsa.dsa_absorb_query(bf16_tensor(qn), bf16_tensor(qr), bf16_tensor(wk), q_abs, ws)
    cache, dims = cache_of(inp, t), dims_of(inp)
    idx = torch.empty((n, wl.topk), dtype=torch.int32, device="cuda")
    o_lat = torch.empty((n, H, R), device="cuda")
    lse = torch.empty((n, H), device="cuda")
    fws = dsa.workspace(dsa.OP_ATTENTION_FORWARD, dims, cache)
    dsa.dsa_attention_forward(t["q_idx"], t["w"], t["k_pages"], q_abs, t["latent_pages"], cache,
                              dims, idx, o_lat, lse, fws)
    v = torch.empty((n, H, d_v), device="cuda")
    dsa.dsa_project_values(o_lat, bf16_tensor(wv), v, ws)
    assert dsa.workspace_check(ws)[0] == 0 and dsa.workspace_check(fws)[0] == 0
    idx, v, qa = idx.cpu().numpy(), v.cpu().numpy(), _bits(q_abs)
    WK, WV = orc.bf16_to_f64(wk), orc.bf16_to_f64(wv)
    for b in range(n):
        ref_idx = orc.dsa_decode(inp, rows=[b])[b]["idx"]
        assert np.array_equal(idx[b].astype(np.int64), ref_idx)
        sel = ref_idx[ref_idx >= 0]
        rows = orc.bf16_to_f64(orc.gather_paged_rows(inp["latent_pages"], inp["block_table"][b],
                                                     sel))
        # the step and the projection, from the bf16 absorbed query the step got
        lat, _, _ = orc.mla_attention(orc.bf16_to_f64(qa[b]), rows, R, wl.scale)
        assert norm_err(v[b], orc.project_values(lat, WV)) <= 2e-3, b
        # the whole block against the non-absorbed definition; the bf16
        # rounding of the absorbed query (2^-9 relative) is the difference
        ref_v, _ = orc.mla_attention_nonabsorbed(orc.bf16_to_f64(qn[b]), orc.bf16_to_f64(qr[b]),
                                                 rows[:, :R], rows[:, R:], WK, WV, wl.scale)
        assert norm_err(v[b], ref_v) <= 1e-2, b
