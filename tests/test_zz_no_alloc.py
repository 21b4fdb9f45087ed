"""The sparse MLA decode entry point that allocates nothing.

Some callers cannot allocate device memory where they run the step (a
memory pool that must not grow, a host that only hands over its input and
output buffers).  dsa_sparse_mla_decode_noalloc serves them: its scratch is a
fixed array inside the library.  This test calls it through the C ABI and
checks it against dsa_sparse_mla_decode (the entry point with a caller
workspace) on two calls in a row, within the tolerances of the other tests,
on every way a row's work is laid out over CTAs: one CTA per row, a row split
over the CTAs of one cluster, and a row split further (partials through the
built-in array).  One case is also checked against the float64 oracle, and
the built-in status block is read back after every call.
This file is named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

import dsa_inputs as di
import sparse_attention_scores_b200 as dsa
from oracle import dsa_oracle as orc
from tests.dsa_testutil import LSE_TOL, OUT_TOL, cache_of, dims_of, norm_err, upload

pytestmark = pytest.mark.gpu


def _selection(rng, lengths, k):
    idx = np.full((len(lengths), k), -1, np.int32)
    for r, n in enumerate(lengths):
        m = min(n, k)
        idx[r, :m] = np.sort(rng.choice(n, size=m, replace=False))
    return idx


def _noalloc(L, t, cache, idx, dims, out, lse):
    stream = torch.cuda.current_stream().cuda_stream or None
    return L.dsa_sparse_mla_decode_noalloc(
        ctypes.c_void_p(t["q"].data_ptr()), ctypes.c_void_p(t["latent_pages"].data_ptr()),
        ctypes.byref(cache.struct()), ctypes.c_void_p(idx.data_ptr()),
        ctypes.byref(dims.struct()), ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(lse.data_ptr()), stream)


CASES = {
    # a few rows: each row split over several CTAs
    "batch4_top2048": ([9000, 2500, 4100, 700], 2048),
    # one long selection: a row split as far as it goes
    "batch1_top8192": ([30000], 8192),
    # 32 rows of top-2,048: a row split over the CTAs of one cluster
    "batch32_top2048": ([2048 + 997 * i for i in range(32)], 2048),
    # more rows than SMs: one CTA per row, no partials at all
    "batch160_top256": ([300 + 7 * i for i in range(160)], 256),
}


@pytest.mark.parametrize("case", list(CASES))
def test_noalloc_matches_workspace_entry_point(case):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lengths, topk = CASES[case]
    L = dsa.lib()
    rng = np.random.default_rng(77)
    wl = di.small_decode(lengths, H_I=4, D_I=32, topk=topk, H=64, R=512, P=64, seed=5)
    inp = di.make_inputs(wl)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    B = wl.n_q
    ws = dsa.workspace(dsa.OP_SPARSE_MLA_DECODE, dims, cache)
    for call in range(2):
        sel = _selection(rng, lengths, wl.topk)
        idx = torch.from_numpy(sel).cuda()
        ref_out = torch.empty((B, wl.H, wl.R), device="cuda")
        ref_lse = torch.empty((B, wl.H), device="cuda")
        dsa.dsa_sparse_mla_decode(t["q"], t["latent_pages"], cache, idx, dims, ref_out, ref_lse, ws)
        out = torch.full((B, wl.H, wl.R), float("nan"), device="cuda")
        lse = torch.full((B, wl.H), float("nan"), device="cuda")
        st = _noalloc(L, t, cache, idx, dims, out, lse)
        assert st == 0, dsa.STATUS_NAMES.get(st, st)
        st, info = dsa.noalloc_status()
        assert st == 0, (dsa.STATUS_NAMES.get(st, st), hex(info))
        torch.cuda.synchronize()
        assert dsa.workspace_check(ws)[0] == 0
        o, l = out.cpu().numpy(), lse.cpu().numpy()
        ro, rl = ref_out.cpu().numpy().astype(np.float64), ref_lse.cpu().numpy().astype(np.float64)
        for b in range(B):
            assert norm_err(o[b], ro[b]) <= OUT_TOL, (call, b)
            assert np.max(np.abs(l[b] - rl[b])) <= LSE_TOL, (call, b)
        if case == "batch4_top2048":
            # the float64 definition on the same selection, row by row
            q = orc.bf16_to_f64(inp["q"])
            lat = orc.bf16_to_f64(inp["latent_pages"])
            for b in range(B):
                pos = sel[b][sel[b] >= 0]
                rows = orc.gather_paged_rows(lat, inp["block_table"][b], pos)
                ref_o, ref_l, _ = orc.mla_attention(q[b], rows, wl.R, wl.scale)
                assert norm_err(o[b], ref_o) <= OUT_TOL, (call, b)
                assert np.max(np.abs(l[b] - ref_l)) <= LSE_TOL, (call, b)


def test_noalloc_reports_bad_index():
    # a selected position beyond the row's context is skipped on the device
    # and reported through the built-in status block, not silently dropped
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = dsa.lib()
    lengths = [3000, 1200]
    wl = di.small_decode(lengths, H_I=4, D_I=32, topk=256, H=64, R=512, P=64, seed=9)
    inp = di.make_inputs(wl)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    sel = _selection(np.random.default_rng(3), lengths, wl.topk)
    sel[1, 5] = lengths[1] + 10   # outside row 1's context
    idx = torch.from_numpy(sel).cuda()
    out = torch.empty((wl.n_q, wl.H, wl.R), device="cuda")
    lse = torch.empty((wl.n_q, wl.H), device="cuda")
    assert _noalloc(L, t, cache, idx, dims, out, lse) == 0
    st, info = dsa.noalloc_status()
    assert st == 6, dsa.STATUS_NAMES.get(st, st)    # DSA_ERR_DEVICE_CHECK
    assert info >> 24 == 3                            # the sparse MLA kernel
    # the next call starts from a clear status block
    sel[1, 5] = 0
    sel[1] = np.sort(sel[1])
    idx.copy_(torch.from_numpy(sel))
    assert _noalloc(L, t, cache, idx, dims, out, lse) == 0
    assert dsa.noalloc_status()[0] == 0


def test_noalloc_rejects_oversize_request():
    # two rows of top-65,536 split 64 ways need 16.8 MB of partials: more than
    # the 16 MiB array, so the call must return DSA_ERR_WORKSPACE before
    # launching.  Real, correctly sized buffers (every slot unused) keep the
    # call memory-safe regardless.
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = dsa.lib()
    B, k, H, R, P = 2, 65536, 64, 512, 64
    q = torch.zeros((B, H, R + P), dtype=torch.bfloat16, device="cuda")
    latent = torch.zeros((1, 64, R + P), dtype=torch.bfloat16, device="cuda")
    idx = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    out = torch.empty((B, H, R), device="cuda")
    lse = torch.empty((B, H), device="cuda")
    seq_lens = torch.ones(B, dtype=torch.int32, device="cuda")
    table = torch.zeros((B, 1), dtype=torch.int32, device="cuda")
    cache = dsa.PagedCache(seq_lens, table, num_pages=1, max_seq_len=1)
    dims = dsa.Dims(n_q=B, H_I=4, D_I=32, topk=k, H=H, R=R, P=P, scale=0.1)
    t = {"q": q, "latent_pages": latent}
    st = _noalloc(L, t, cache, idx, dims, out, lse)
    torch.cuda.synchronize()
    assert st == 4, dsa.STATUS_NAMES.get(st, st)   # DSA_ERR_WORKSPACE
