"""The whole step with host buffers (dsa_attention_forward_host) on the GPU:
its results equal dsa_attention_forward's on the same inputs bit for bit (the
same kernels run on copies of the same bytes), on two calls in a row through
one workspace, and match the oracle (indices exactly, outputs within 2e-3)."""

import numpy as np
import pytest
import torch

import dsa_inputs as di
import sparse_attention_scores_b200 as dsa
from oracle import dsa_oracle as orc
from dsa_testutil import assert_row_matches, cache_of, dims_of, upload

pytestmark = pytest.mark.gpu

CASES = [
    di.small_decode([2100, 2048, 5000], H_I=32, D_I=128, topk=2048, H=64, R=512, P=64, seed=11),
    di.small_decode([50, 64, 300, 1000], H_I=4, D_I=32, topk=128, H=8, R=64, P=16, seed=12),
    di.small_prefill(150, q_pos0=40, H_I=4, D_I=32, topk=100, H=4, R=64, P=16, seed=13),
]


def _pinned(x: torch.Tensor) -> torch.Tensor:
    return x.cpu().pin_memory()


@pytest.mark.parametrize("wl", CASES, ids=lambda w: f"{w.mode}_{w.n_q}_{w.topk}")
def test_host_buffers_equal_device_call(wl):
    inp = di.make_inputs(wl)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    n, k, H, R = wl.n_q, wl.topk, wl.H, wl.R
    # the device-buffer call
    idx = torch.empty((n, k), dtype=torch.int32, device="cuda")
    out = torch.empty((n, H, R), device="cuda")
    lse = torch.empty((n, H), device="cuda")
    ws = dsa.workspace(dsa.OP_ATTENTION_FORWARD, dims, cache)
    dsa.dsa_attention_forward(t["q_idx"], t["w"], t["k_pages"], t["q"], t["latent_pages"], cache,
                              dims, idx, out, lse, ws)
    # the host-buffer call, twice through one workspace (second time on other inputs' memory)
    hin = {name: _pinned(t[name]) for name in ("q_idx", "w", "q", "seq_lens", "block_table")}
    cache_h = dsa.PagedCache(hin["seq_lens"], hin["block_table"], num_pages=cache.num_pages,
                             max_seq_len=cache.max_seq_len)
    hws = dsa.workspace(dsa.OP_ATTENTION_FORWARD_HOST, dims, cache_h)
    for _ in range(2):
        idx_h = torch.full((n, k), -9, dtype=torch.int32).pin_memory()
        out_h = torch.full((n, H, R), float("nan")).pin_memory()
        lse_h = torch.full((n, H), float("nan")).pin_memory()
        dsa.dsa_attention_forward_host(hin["q_idx"], hin["w"], t["k_pages"], hin["q"],
                                       t["latent_pages"], cache_h, dims, idx_h, out_h, lse_h, hws)
        torch.cuda.synchronize()
        assert dsa.workspace_check(hws)[0] == 0
        assert torch.equal(idx_h, idx.cpu())
        assert torch.equal(out_h, out.cpu())
        assert torch.equal(lse_h, lse.cpu())
    # and the host results are the oracle's (rows at both ends): indices exact,
    # outputs and lse within the tolerances
    rows = [0, n - 1]
    ref = orc.dsa_decode(inp, rows=rows) if wl.mode == "decode" else orc.dsa_prefill(inp, rows=rows)
    for r in rows:
        assert_row_matches(r, ref[r], idx_h.numpy(), out_h.numpy(), lse_h.numpy())
    assert dsa.workspace_check(ws)[0] == 0


def test_host_buffers_without_index_output():
    wl = CASES[1]
    inp = di.make_inputs(wl)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    hin = {name: _pinned(t[name]) for name in ("q_idx", "w", "q", "seq_lens", "block_table")}
    cache_h = dsa.PagedCache(hin["seq_lens"], hin["block_table"], num_pages=cache.num_pages,
                             max_seq_len=cache.max_seq_len)
    hws = dsa.workspace(dsa.OP_ATTENTION_FORWARD_HOST, dims, cache_h)
    out_h = torch.full((wl.n_q, wl.H, wl.R), float("nan")).pin_memory()
    lse_h = torch.full((wl.n_q, wl.H), float("nan")).pin_memory()
    dsa.dsa_attention_forward_host(hin["q_idx"], hin["w"], t["k_pages"], hin["q"],
                                   t["latent_pages"], cache_h, dims, None, out_h, lse_h, hws)
    torch.cuda.synchronize()
    assert dsa.workspace_check(hws)[0] == 0
    assert torch.isfinite(out_h).all() and torch.isfinite(lse_h).all()


def test_pageable_host_buffers_take_the_copy_engine():
    # pageable host memory is not device-addressable: the call copies it with
    # cudaMemcpyAsync instead, with the same results
    wl = CASES[0]
    inp = di.make_inputs(wl)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    n, k, H, R = wl.n_q, wl.topk, wl.H, wl.R
    idx = torch.empty((n, k), dtype=torch.int32, device="cuda")
    out = torch.empty((n, H, R), device="cuda")
    lse = torch.empty((n, H), device="cuda")
    ws = dsa.workspace(dsa.OP_ATTENTION_FORWARD, dims, cache)
    dsa.dsa_attention_forward(t["q_idx"], t["w"], t["k_pages"], t["q"], t["latent_pages"], cache,
                              dims, idx, out, lse, ws)
    hin = {name: t[name].cpu() for name in ("q_idx", "w", "q", "seq_lens", "block_table")}
    assert not hin["q"].is_pinned()
    cache_h = dsa.PagedCache(hin["seq_lens"], hin["block_table"], num_pages=cache.num_pages,
                             max_seq_len=cache.max_seq_len)
    hws = dsa.workspace(dsa.OP_ATTENTION_FORWARD_HOST, dims, cache_h)
    idx_h = torch.full((n, k), -9, dtype=torch.int32)
    out_h = torch.full((n, H, R), float("nan"))
    lse_h = torch.full((n, H), float("nan"))
    dsa.dsa_attention_forward_host(hin["q_idx"], hin["w"], t["k_pages"], hin["q"],
                                   t["latent_pages"], cache_h, dims, idx_h, out_h, lse_h, hws)
    torch.cuda.synchronize()
    assert dsa.workspace_check(hws)[0] == 0
    assert torch.equal(idx_h, idx.cpu()) and torch.equal(out_h, out.cpu())
    assert torch.equal(lse_h, lse.cpu())


def test_back_to_back_calls_keep_their_own_queries():
    # calls queued without a sync between them, through one workspace, on
    # different queries: each must attend with its own (the next call's input
    # copy overwrites the staging only after the previous step's MLA has read it)
    wl = CASES[0]
    inp = di.make_inputs(wl)
    t = upload(inp)
    cache, dims = cache_of(inp, t), dims_of(inp)
    n, k, H, R = wl.n_q, wl.topk, wl.H, wl.R
    q_b = -t["q"]   # every sign flipped (exact in bf16)
    ws = dsa.workspace(dsa.OP_ATTENTION_FORWARD, dims, cache)
    want = []
    for q in (t["q"], q_b):
        out = torch.empty((n, H, R), device="cuda")
        lse = torch.empty((n, H), device="cuda")
        dsa.dsa_attention_forward(t["q_idx"], t["w"], t["k_pages"], q, t["latent_pages"], cache,
                                  dims, None, out, lse, ws)
        want.append((out.cpu(), lse.cpu()))
    assert not torch.equal(want[0][0], want[1][0])
    hin = {name: _pinned(t[name]) for name in ("q_idx", "w", "seq_lens", "block_table")}
    q_h = [_pinned(t["q"]), _pinned(q_b)]
    cache_h = dsa.PagedCache(hin["seq_lens"], hin["block_table"], num_pages=cache.num_pages,
                             max_seq_len=cache.max_seq_len)
    hws = dsa.workspace(dsa.OP_ATTENTION_FORWARD_HOST, dims, cache_h)
    got = []
    for rep in range(3):
        for q in q_h:
            out_h = torch.full((n, H, R), float("nan")).pin_memory()
            lse_h = torch.full((n, H), float("nan")).pin_memory()
            dsa.dsa_attention_forward_host(hin["q_idx"], hin["w"], t["k_pages"], q,
                                           t["latent_pages"], cache_h, dims, None, out_h, lse_h,
                                           hws)
            got.append((out_h, lse_h))
    torch.cuda.synchronize()
    assert dsa.workspace_check(hws)[0] == 0
    for i, (out_h, lse_h) in enumerate(got):
        assert torch.equal(out_h, want[i % 2][0]), f"call {i}"
        assert torch.equal(lse_h, want[i % 2][1]), f"call {i}"
