"""Python binding of libdsa, the B200 (sm_100a) DSA sparse-attention step.

Argument marshalling only: every function below forwards torch tensors'
device pointers to the C ABI of include/dsa.h, on the current CUDA stream,
and raises DsaError on a non-OK status.  There is no fallback: when the
compiled library is missing, loading it raises.

    import sparse_attention_scores_b200 as dsa
    cache = dsa.PagedCache(seq_lens, block_table, num_pages, max_seq_len)
    dims = dsa.Dims(n_q, H_I, D_I, topk, H, R, P, causal, q_pos0, scale)
    ws = dsa.workspace(dsa.OP_ATTENTION_FORWARD, dims, cache)
    dsa.dsa_attention_forward(q_idx, w, k_pages, q, latent_pages, cache, dims,
                              idx_out, out, lse, ws)
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")

OP_INDEXER_SCORES = 0
OP_TOPK = 1
OP_SPARSE_MLA_DECODE = 2
OP_SPARSE_MLA_PREFILL = 3
OP_ATTENTION_FORWARD = 4
OP_CACHE_APPEND = 5
OP_INDEXER_SCORES_K8 = 6
OP_ATTENTION_FORWARD_K8 = 7
OP_ATTENTION_FORWARD_HOST = 8
OP_ATTENTION_FORWARD_FP8 = 9

STATUS_NAMES = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED",
                3: "DSA_ERR_CUDA", 4: "DSA_ERR_WORKSPACE", 5: "DSA_ERR_TIMEOUT",
                6: "DSA_ERR_DEVICE_CHECK"}

EXPORTED = ["dsa_version", "dsa_status_string", "dsa_workspace_bytes", "dsa_workspace_init",
            "dsa_workspace_check", "dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla_decode",
            "dsa_sparse_mla_prefill", "dsa_attention_forward", "dsa_sparse_mla_decode_noalloc",
            "dsa_cache_append", "dsa_absorb_query", "dsa_project_values",
            "dsa_indexer_scores_k8", "dsa_attention_forward_k8", "dsa_cp_workspace_bytes",
            "dsa_cp_candidates", "dsa_cp_select", "dsa_cp_merge",
            "dsa_attention_forward_host", "dsa_noalloc_status", "dsa_forward_launches",
            "dsa_sparse_mla_decode_l8", "dsa_sparse_mla_prefill_l8", "dsa_attention_forward_fp8",
            "dsa_last_cuda_error"]


class DsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {STATUS_NAMES.get(status, status)}"
        if status == 3 and _lib is not None:   # DSA_ERR_CUDA: the CUDA error behind it
            msg += f" ({_lib.dsa_last_cuda_error().decode()})"
        super().__init__(msg)


class CacheStruct(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("seq_lens", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("max_pages", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("max_seq_len", ctypes.c_int32)]


class DimsStruct(ctypes.Structure):
    _fields_ = [("n_q", ctypes.c_int32), ("H_I", ctypes.c_int32), ("D_I", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("H", ctypes.c_int32), ("R", ctypes.c_int32),
                ("P", ctypes.c_int32), ("causal", ctypes.c_int32), ("q_pos0", ctypes.c_int32),
                ("scale", ctypes.c_float)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libdsa.so (built in place by __graft_entry__.build or
    `python -m sparse_attention_scores_b200.build`).  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libdsa.so not built ({LIB_PATH}); run "
                               "`python -m sparse_attention_scores_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32, i64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64
        pc, pd = ctypes.POINTER(CacheStruct), ctypes.POINTER(DimsStruct)
        sigs = {
            "dsa_version": ([], ctypes.c_int),
            "dsa_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "dsa_last_cuda_error": ([], ctypes.c_char_p),
            "dsa_workspace_bytes": ([ctypes.c_int, pd, pc], sz),
            "dsa_workspace_init": ([vp, sz, vp], ctypes.c_int),
            "dsa_workspace_check": ([vp, vp, ctypes.POINTER(ctypes.c_uint32)], ctypes.c_int),
            "dsa_indexer_scores": ([vp, vp, vp, pc, pd, vp, i64, vp, sz, vp], ctypes.c_int),
            "dsa_topk": ([vp, i64, i32, vp, i32, i32, vp, vp, sz, vp], ctypes.c_int),
            "dsa_sparse_mla_decode": ([vp, vp, pc, vp, pd, vp, vp, vp, sz, vp], ctypes.c_int),
            "dsa_sparse_mla_prefill": ([vp, vp, pc, vp, pd, vp, vp, vp, sz, vp], ctypes.c_int),
            "dsa_attention_forward": ([vp, vp, vp, vp, vp, pc, pd, vp, vp, vp, vp, sz, vp],
                                      ctypes.c_int),
            "dsa_sparse_mla_decode_noalloc": ([vp, vp, pc, vp, pd, vp, vp, vp], ctypes.c_int),
            "dsa_noalloc_status": ([vp, ctypes.POINTER(ctypes.c_uint32)], ctypes.c_int),
            "dsa_forward_launches": ([ctypes.c_int, pd, pc], i32),
            "dsa_sparse_mla_decode_l8": ([vp, vp, vp, pc, vp, pd, vp, vp, vp, sz, vp], ctypes.c_int),
            "dsa_sparse_mla_prefill_l8": ([vp, vp, vp, pc, vp, pd, vp, vp, vp, sz, vp], ctypes.c_int),
            "dsa_attention_forward_fp8": ([vp, vp, vp, vp, vp, vp, vp, pc, pd, vp, vp, vp, vp, sz,
                                           vp], ctypes.c_int),
            "dsa_cache_append": ([vp, vp, vp, vp, pc, pd, vp, sz, vp], ctypes.c_int),
            "dsa_absorb_query": ([vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, sz, vp],
                                 ctypes.c_int),
            "dsa_project_values": ([vp, vp, vp, i32, i32, i32, i32, vp, sz, vp], ctypes.c_int),
            "dsa_indexer_scores_k8": ([vp, vp, vp, vp, pc, pd, vp, i64, vp, sz, vp], ctypes.c_int),
            "dsa_attention_forward_k8": ([vp, vp, vp, vp, vp, vp, pc, pd, vp, vp, vp, vp, sz, vp],
                                         ctypes.c_int),
            "dsa_cp_workspace_bytes": ([i32, i32, i32], sz),
            "dsa_cp_candidates": ([vp, i64, i32, vp, i32, vp, vp, vp, vp, sz, vp], ctypes.c_int),
            "dsa_cp_select": ([vp, vp, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
            "dsa_cp_merge": ([vp, vp, i32, i32, i32, i32, vp, vp, vp, sz, vp], ctypes.c_int),
            "dsa_attention_forward_host": ([vp, vp, vp, vp, vp, pc, pd, vp, vp, vp, vp, sz, vp],
                                           ctypes.c_int),
        }
        for name, (args, res) in sigs.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


@dataclass
class Dims:
    n_q: int
    H_I: int
    D_I: int
    topk: int
    H: int
    R: int
    P: int
    causal: int = 0
    q_pos0: int = 0
    scale: float = 1.0

    def struct(self) -> DimsStruct:
        return DimsStruct(self.n_q, self.H_I, self.D_I, self.topk, self.H, self.R, self.P,
                          self.causal, self.q_pos0, self.scale)


@dataclass
class PagedCache:
    """Device-side view of the paged caches: seq_lens [B] int32 and
    block_table [B, max_pages] int32 CUDA tensors, plus host-side sizes."""
    seq_lens: object
    block_table: object
    num_pages: int
    max_seq_len: int
    page_size: int = 64

    def struct(self) -> CacheStruct:
        return CacheStruct(int(self.seq_lens.shape[0]), _ptr(self.seq_lens),
                           _ptr(self.block_table), int(self.block_table.shape[1]),
                           self.page_size, int(self.num_pages), int(self.max_seq_len))


def _ptr(t) -> int | None:
    return None if t is None else int(t.data_ptr())


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream) or None
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _check(status: int, where: str) -> None:
    if status != 0:
        raise DsaError(status, where)


def workspace_bytes(op: int, dims: Dims, cache: PagedCache | None) -> int:
    c = ctypes.byref(cache.struct()) if cache is not None else None
    return int(lib().dsa_workspace_bytes(op, ctypes.byref(dims.struct()), c))


def workspace(op: int, dims: Dims, cache: PagedCache | None, device="cuda", stream=None):
    """Allocate (with torch) and initialise a workspace for `op`."""
    import torch
    n = workspace_bytes(op, dims, cache)
    if n == 0:
        raise DsaError(1, "dsa_workspace_bytes")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _check(lib().dsa_workspace_init(_ptr(ws), n, _stream(stream)), "dsa_workspace_init")
    return ws


STATUS_WORKSPACE_BYTES = 256  # DSA_STATUS_WORKSPACE_BYTES


def status_workspace(device="cuda", stream=None):
    """Workspace of the entry points that need only the status block."""
    import torch
    ws = torch.empty(STATUS_WORKSPACE_BYTES, dtype=torch.uint8, device=device)
    _check(lib().dsa_workspace_init(_ptr(ws), STATUS_WORKSPACE_BYTES, _stream(stream)),
           "dsa_workspace_init")
    return ws


def workspace_check(ws, stream=None) -> tuple[int, int]:
    info = ctypes.c_uint32(0)
    st = lib().dsa_workspace_check(_ptr(ws), _stream(stream), ctypes.byref(info))
    return int(st), int(info.value)


def dsa_indexer_scores(q_idx, w, k_idx_pages, cache: PagedCache, dims: Dims, scores, ws,
                       stream=None) -> None:
    _check(lib().dsa_indexer_scores(_ptr(q_idx), _ptr(w), _ptr(k_idx_pages),
                                    ctypes.byref(cache.struct()), ctypes.byref(dims.struct()),
                                    _ptr(scores), int(scores.stride(0)), _ptr(ws), ws.numel(),
                                    _stream(stream)), "dsa_indexer_scores")


def dsa_topk(scores, valid_len, causal_base: int, k: int, idx, ws, stream=None) -> None:
    _check(lib().dsa_topk(_ptr(scores), int(scores.stride(0)), int(scores.shape[0]),
                          _ptr(valid_len), int(causal_base), int(k), _ptr(idx), _ptr(ws),
                          ws.numel(), _stream(stream)), "dsa_topk")


def dsa_sparse_mla_decode(q, latent_pages, cache: PagedCache, idx, dims: Dims, out, lse, ws,
                          stream=None) -> None:
    _check(lib().dsa_sparse_mla_decode(_ptr(q), _ptr(latent_pages), ctypes.byref(cache.struct()),
                                       _ptr(idx), ctypes.byref(dims.struct()), _ptr(out),
                                       _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_sparse_mla_decode")


def dsa_sparse_mla_prefill(q, latent_pages, cache: PagedCache, idx, dims: Dims, out, lse, ws,
                           stream=None) -> None:
    _check(lib().dsa_sparse_mla_prefill(_ptr(q), _ptr(latent_pages),
                                        ctypes.byref(cache.struct()), _ptr(idx),
                                        ctypes.byref(dims.struct()), _ptr(out), _ptr(lse),
                                        _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_sparse_mla_prefill")


def dsa_sparse_mla_decode_l8(q, latent8_pages, latent_scale, cache: PagedCache, idx, dims: Dims,
                             out, lse, ws, stream=None) -> None:
    """Sparse MLA decode over an FP8 latent cache (E4M3 rows, one fp32 scale per token)."""
    _check(lib().dsa_sparse_mla_decode_l8(_ptr(q), _ptr(latent8_pages), _ptr(latent_scale),
                                          ctypes.byref(cache.struct()), _ptr(idx),
                                          ctypes.byref(dims.struct()), _ptr(out), _ptr(lse),
                                          _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_sparse_mla_decode_l8")


def dsa_sparse_mla_prefill_l8(q, latent8_pages, latent_scale, cache: PagedCache, idx, dims: Dims,
                              out, lse, ws, stream=None) -> None:
    _check(lib().dsa_sparse_mla_prefill_l8(_ptr(q), _ptr(latent8_pages), _ptr(latent_scale),
                                           ctypes.byref(cache.struct()), _ptr(idx),
                                           ctypes.byref(dims.struct()), _ptr(out), _ptr(lse),
                                           _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_sparse_mla_prefill_l8")


def dsa_attention_forward_fp8(q_idx, w, k8_pages, k_scale, q, latent8_pages, latent_scale,
                              cache: PagedCache, dims: Dims, idx_out, out, lse, ws,
                              stream=None) -> None:
    """The whole step with both caches in FP8 (E4M3 + one scale per token)."""
    _check(lib().dsa_attention_forward_fp8(_ptr(q_idx), _ptr(w), _ptr(k8_pages), _ptr(k_scale),
                                           _ptr(q), _ptr(latent8_pages), _ptr(latent_scale),
                                           ctypes.byref(cache.struct()),
                                           ctypes.byref(dims.struct()), _ptr(idx_out), _ptr(out),
                                           _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_attention_forward_fp8")


def dsa_sparse_mla_decode_noalloc(q, latent_pages, cache: PagedCache, idx, dims: Dims, out, lse,
                                  stream=None) -> None:
    """Sparse MLA decode without a workspace, for callers that cannot allocate
    device memory: the scratch is a fixed array inside the library (see
    include/dsa.h for its limits and sharing rules)."""
    _check(lib().dsa_sparse_mla_decode_noalloc(_ptr(q), _ptr(latent_pages),
                                               ctypes.byref(cache.struct()), _ptr(idx),
                                               ctypes.byref(dims.struct()), _ptr(out), _ptr(lse),
                                               _stream(stream)), "dsa_sparse_mla_decode_noalloc")


def forward_launches(op: int, dims: Dims, cache: PagedCache) -> int:
    """Kernels one fused forward call launches for these shapes on the current device."""
    return int(lib().dsa_forward_launches(op, ctypes.byref(dims.struct()),
                                          ctypes.byref(cache.struct())))


def noalloc_status(stream=None):
    """(status, info) of the last no-alloc decode on the current device: its
    device-side range checks and bounded waits (synchronises the stream)."""
    info = ctypes.c_uint32(0)
    st = lib().dsa_noalloc_status(_stream(stream), ctypes.byref(info))
    return st, info.value


def dsa_attention_forward(q_idx, w, k_idx_pages, q, latent_pages, cache: PagedCache, dims: Dims,
                          idx_out, out, lse, ws, stream=None) -> None:
    _check(lib().dsa_attention_forward(_ptr(q_idx), _ptr(w), _ptr(k_idx_pages), _ptr(q),
                                       _ptr(latent_pages), ctypes.byref(cache.struct()),
                                       ctypes.byref(dims.struct()), _ptr(idx_out), _ptr(out),
                                       _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_attention_forward")


def dsa_attention_forward_host(q_idx_h, w_h, k_idx_pages, q_h, latent_pages,
                               cache_h: PagedCache, dims: Dims, idx_h, out_h, lse_h, ws,
                               stream=None) -> None:
    """The whole step with host buffers: q_idx_h, w_h, q_h, cache_h.seq_lens,
    cache_h.block_table, idx_h (may be None), out_h and lse_h are CPU tensors
    (pinned for an asynchronous call); the page pools and ws are CUDA tensors.
    The host results are valid once the stream has reached the call."""
    _check(lib().dsa_attention_forward_host(_ptr(q_idx_h), _ptr(w_h), _ptr(k_idx_pages),
                                            _ptr(q_h), _ptr(latent_pages),
                                            ctypes.byref(cache_h.struct()),
                                            ctypes.byref(dims.struct()), _ptr(idx_h), _ptr(out_h),
                                            _ptr(lse_h), _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_attention_forward_host")


def dsa_cache_append(k_idx_new, latent_new, k_idx_pages, latent_pages, cache: PagedCache,
                     dims: Dims, ws, stream=None) -> None:
    """Write the new tokens' index keys [n_q, D_I] and latent rows [n_q, R + P]
    into the page pools at the positions of the step's query rows (decode row b:
    seq_lens[b] - 1 of sequence b; prefill row t: q_pos0 + t of sequence 0)."""
    _check(lib().dsa_cache_append(_ptr(k_idx_new), _ptr(latent_new), _ptr(k_idx_pages),
                                  _ptr(latent_pages), ctypes.byref(cache.struct()),
                                  ctypes.byref(dims.struct()), _ptr(ws), ws.numel(),
                                  _stream(stream)), "dsa_cache_append")


def dsa_absorb_query(q_nope, q_rope, w_uk, q_abs, ws, stream=None) -> None:
    """q_abs [n, H, R + P] = [q_nope [n, H, d_nope] . w_uk [H, d_nope, R] | q_rope [n, H, P]]."""
    n, H, d_nope = (int(x) for x in q_nope.shape)
    R = int(w_uk.shape[2])
    P = int(q_rope.shape[2]) if q_rope is not None else 0
    _check(lib().dsa_absorb_query(_ptr(q_nope), _ptr(q_rope), _ptr(w_uk), _ptr(q_abs), n, H,
                                  d_nope, R, P, _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_absorb_query")


def dsa_project_values(o_lat, w_uv, v_out, ws, stream=None) -> None:
    """v_out [n, H, d_v] = o_lat [n, H, R] (fp32) . w_uv [H, R, d_v]."""
    n, H, R = (int(x) for x in o_lat.shape)
    d_v = int(w_uv.shape[2])
    _check(lib().dsa_project_values(_ptr(o_lat), _ptr(w_uv), _ptr(v_out), n, H, R, d_v,
                                    _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_project_values")


def dsa_indexer_scores_k8(q_idx, w, k8_pages, k_scale, cache: PagedCache, dims: Dims, scores, ws,
                          stream=None) -> None:
    """dsa_indexer_scores over E4M3 index keys [pages, 64, D_I] (uint8) with one
    fp32 scale per key row [pages * 64]."""
    _check(lib().dsa_indexer_scores_k8(_ptr(q_idx), _ptr(w), _ptr(k8_pages), _ptr(k_scale),
                                       ctypes.byref(cache.struct()), ctypes.byref(dims.struct()),
                                       _ptr(scores), int(scores.stride(0)), _ptr(ws), ws.numel(),
                                       _stream(stream)), "dsa_indexer_scores_k8")


def dsa_attention_forward_k8(q_idx, w, k8_pages, k_scale, q, latent_pages, cache: PagedCache,
                             dims: Dims, idx_out, out, lse, ws, stream=None) -> None:
    """dsa_attention_forward with the index-key cache as E4M3 bytes plus scales."""
    _check(lib().dsa_attention_forward_k8(_ptr(q_idx), _ptr(w), _ptr(k8_pages), _ptr(k_scale),
                                          _ptr(q), _ptr(latent_pages), ctypes.byref(cache.struct()),
                                          ctypes.byref(dims.struct()), _ptr(idx_out), _ptr(out),
                                          _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_attention_forward_k8")


def cp_workspace(ranks: int, n_q: int, k: int, device="cuda", stream=None):
    """Workspace of dsa_cp_select."""
    import torch
    n = int(lib().dsa_cp_workspace_bytes(ranks, n_q, k))
    if n == 0:
        raise DsaError(1, "dsa_cp_workspace_bytes")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _check(lib().dsa_workspace_init(_ptr(ws), n, _stream(stream)), "dsa_workspace_init")
    return ws


def dsa_cp_candidates(scores, idx_local, offsets, cand_scores, cand_idx, ws, stream=None) -> None:
    n_q, k = (int(x) for x in idx_local.shape)
    _check(lib().dsa_cp_candidates(_ptr(scores), int(scores.stride(0)), n_q, _ptr(idx_local), k,
                                   _ptr(offsets), _ptr(cand_scores), _ptr(cand_idx), _ptr(ws),
                                   ws.numel(), _stream(stream)), "dsa_cp_candidates")


def dsa_cp_select(all_scores, all_idx, my_offsets, my_lens, gidx, own_idx, ws, stream=None) -> None:
    ranks, n_q, k = (int(x) for x in all_scores.shape)
    _check(lib().dsa_cp_select(_ptr(all_scores), _ptr(all_idx), ranks, n_q, k, _ptr(my_offsets),
                               _ptr(my_lens), _ptr(gidx), _ptr(own_idx), _ptr(ws), ws.numel(),
                               _stream(stream)), "dsa_cp_select")


def dsa_cp_merge(outs, lses, out, lse, ws, stream=None) -> None:
    ranks, n_q, H, dv = (int(x) for x in outs.shape)
    _check(lib().dsa_cp_merge(_ptr(outs), _ptr(lses), ranks, n_q, H, dv, _ptr(out), _ptr(lse),
                              _ptr(ws), ws.numel(), _stream(stream)), "dsa_cp_merge")
