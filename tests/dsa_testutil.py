"""Helpers shared by the GPU tests: upload seeded inputs, call the library
through its binding, compare with the oracle."""

from __future__ import annotations

import numpy as np
import torch

import sparse_attention_scores_b200 as dsa

OUT_TOL = 2e-3   # max |gpu - ref| / max |ref| on fp32 attention outputs
LSE_TOL = 2e-3   # absolute, natural-log units


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def upload(inp: dict, device="cuda") -> dict:
    return {
        "q_idx": bf16_tensor(inp["q_idx"], device),
        "k_pages": bf16_tensor(inp["k_pages"], device),
        "q": bf16_tensor(inp["q"], device),
        "latent_pages": bf16_tensor(inp["latent_pages"], device),
        "w": torch.from_numpy(inp["w"]).to(device),
        "block_table": torch.from_numpy(inp["block_table"]).to(device),
        "seq_lens": torch.from_numpy(inp["seq_lens"]).to(device),
    }


def cache_of(inp: dict, t: dict) -> dsa.PagedCache:
    return dsa.PagedCache(t["seq_lens"], t["block_table"], num_pages=int(inp["k_pages"].shape[0]),
                          max_seq_len=int(inp["seq_lens"].max()))


def dims_of(inp: dict) -> dsa.Dims:
    return dsa.Dims(n_q=int(inp["n_q"]), H_I=int(inp["H_I"]), D_I=int(inp["D_I"]),
                    topk=int(inp["topk"]), H=int(inp["H"]), R=int(inp["R"]), P=int(inp["P"]),
                    causal=int(inp["mode"] == "prefill"), q_pos0=int(inp["q_pos0"]),
                    scale=float(inp["scale"]))


def row_lengths(inp: dict) -> np.ndarray:
    if inp["mode"] == "prefill":
        return inp["q_pos0"] + np.arange(inp["n_q"]) + 1
    return inp["seq_lens"].astype(np.int64)


def run_forward(inp: dict, t: dict | None = None):
    t = upload(inp) if t is None else t
    cache, dims = cache_of(inp, t), dims_of(inp)
    n_q, k, H, R = dims.n_q, dims.topk, dims.H, dims.R
    idx = torch.full((n_q, k), -7, dtype=torch.int32, device="cuda")
    out = torch.full((n_q, H, R), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((n_q, H), float("nan"), dtype=torch.float32, device="cuda")
    ws = dsa.workspace(dsa.OP_ATTENTION_FORWARD, dims, cache)
    dsa.dsa_attention_forward(t["q_idx"], t["w"], t["k_pages"], t["q"], t["latent_pages"], cache,
                              dims, idx, out, lse, ws)
    st, info = dsa.workspace_check(ws)
    assert st == 0, (st, hex(info))
    return idx.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy()


def norm_err(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.max(np.abs(got.astype(np.float64) - ref)) / max(np.max(np.abs(ref)), 1e-30))


def assert_row_matches(r: int, ref: dict, idx, out, lse):
    assert np.array_equal(idx[r].astype(np.int64), ref["idx"]), f"row {r}: indices differ"
    e = norm_err(out[r], ref["out"])
    assert e <= OUT_TOL, f"row {r}: normalised out error {e:.3e}"
    le = float(np.max(np.abs(lse[r].astype(np.float64) - ref["lse"])))
    assert le <= LSE_TOL, f"row {r}: lse error {le:.3e}"
    return e, le
