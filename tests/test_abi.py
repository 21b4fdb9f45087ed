"""The C-ABI library without a GPU: it loads, exports every declared symbol,
and rejects bad arguments on the host before touching the device."""

import ctypes
import os
import re
import subprocess

import pytest

import sparse_attention_scores_b200 as dsa
from sparse_attention_scores_b200 import build as dsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    dsa_build.build()
    return dsa.lib()


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "dsa.h")).read()
    return sorted(set(re.findall(r"^DSA_API[^(]*?\b(dsa_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported(L):
    declared = _declared_symbols()
    assert len(declared) == 27
    assert sorted(declared) == sorted(dsa.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", dsa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (dsa_\w+)$", out, flags=re.M))
    assert set(declared) <= exported
    for name in declared:
        assert getattr(L, name) is not None


def test_version_and_status_strings(L):
    assert L.dsa_version() >= 100
    for code in range(7):
        assert L.dsa_status_string(code).decode()
    assert L.dsa_status_string(99).decode() == "unknown status"
    assert L.dsa_last_cuda_error().decode() == ""


def _dims(**kw):
    base = dict(n_q=1, H_I=32, D_I=128, topk=2048, H=64, R=512, P=64, causal=0, q_pos0=0,
                scale=1.0)
    base.update(kw)
    return dsa.Dims(**base).struct()


def _cache(num_seqs=1, max_pages=128, num_pages=128, max_seq_len=8192, page_size=64):
    # fake (never dereferenced) device addresses: validation runs on the host first
    return dsa.CacheStruct(num_seqs, 0x100000, 0x200000, max_pages, page_size, num_pages,
                           max_seq_len)


def test_workspace_bytes_host_only(L):
    d, c = _dims(), _cache()
    n_idx = L.dsa_workspace_bytes(dsa.OP_INDEXER_SCORES, ctypes.byref(d), ctypes.byref(c))
    n_fwd = L.dsa_workspace_bytes(dsa.OP_ATTENTION_FORWARD, ctypes.byref(d), ctypes.byref(c))
    assert n_idx == 256
    # status + scores (8192 fp32) + idx (2048 int32) at least
    assert n_fwd >= 256 + 8192 * 4 + 2048 * 4
    bad = _dims(R=100)
    assert L.dsa_workspace_bytes(dsa.OP_ATTENTION_FORWARD, ctypes.byref(bad), ctypes.byref(c)) == 0
    # host-buffer step: the step's workspace, then the staged inputs and results
    # (q_idx 8 KiB, w 128 B, q 72 KiB, seq_lens, block_table 512 B, idx 8 KiB,
    # out 128 KiB, lse 256 B, each rounded up to 256 bytes)
    n_host = L.dsa_workspace_bytes(dsa.OP_ATTENTION_FORWARD_HOST, ctypes.byref(d), ctypes.byref(c))
    assert n_host == n_fwd + 8192 + 256 + 73728 + 256 + 512 + 8192 + 131072 + 256
    assert L.dsa_workspace_bytes(dsa.OP_ATTENTION_FORWARD_HOST, ctypes.byref(d), None) == 0


def _no_device():
    # the fake addresses below must never reach a kernel: these host-only
    # checks run where there is no CUDA device
    try:
        import torch
        if torch.cuda.is_available():
            pytest.skip("host-only validation test; a CUDA device is present")
    except ImportError:
        pass


def test_noalloc_size_check_host_only(L):
    _no_device()
    # 2 rows x 64 splits x 64 heads x 512 x 4 B = 16.8 MB > the 16 MiB array
    d = _dims(n_q=2, topk=65536)
    c = _cache(num_seqs=2, max_pages=1024, num_pages=1024, max_seq_len=65536)
    fake = ctypes.c_void_p(0x300000)
    st = L.dsa_sparse_mla_decode_noalloc(fake, fake, ctypes.byref(c), fake, ctypes.byref(d),
                                         fake, fake, None)
    assert st == 4


def test_noalloc_shares_the_workspace_entry_checks(L):
    _no_device()
    fake = ctypes.c_void_p(0x300000)
    # a page pool whose token rows overflow a 32-bit row index: rejected as
    # unsupported, exactly like the workspace entry point, before any launch
    big = _cache(num_pages=1 << 25)
    d = _dims()
    st_ws = L.dsa_sparse_mla_decode(fake, fake, ctypes.byref(big), fake, ctypes.byref(d), fake,
                                    fake, ctypes.c_void_p(0x400000), 1 << 30, None)
    st = L.dsa_sparse_mla_decode_noalloc(fake, fake, ctypes.byref(big), fake, ctypes.byref(d),
                                         fake, fake, None)
    assert st_ws == 2 and st == 2
    # prefill rows, a batch whose sequence count differs from n_q, a bad page size
    assert L.dsa_sparse_mla_decode_noalloc(fake, fake, ctypes.byref(_cache()), fake,
                                           ctypes.byref(_dims(causal=1)), fake, fake, None) == 1
    assert L.dsa_sparse_mla_decode_noalloc(fake, fake, ctypes.byref(_cache(num_seqs=2)), fake,
                                           ctypes.byref(d), fake, fake, None) == 1
    assert L.dsa_sparse_mla_decode_noalloc(fake, fake, ctypes.byref(_cache(page_size=32)), fake,
                                           ctypes.byref(d), fake, fake, None) == 2


def test_host_validation_rejects_without_launch(L):
    _no_device()
    d, c = _dims(), _cache()
    fake = ctypes.c_void_p(0x300000)
    ws = ctypes.c_void_p(0x400000)
    # null pointers
    st = L.dsa_attention_forward(None, None, None, None, None, ctypes.byref(c), ctypes.byref(d),
                                 None, None, None, ws, 1 << 30, None)
    assert st == 1
    # misaligned q (not 16-byte aligned)
    st = L.dsa_sparse_mla_decode(ctypes.c_void_p(0x300002), fake, ctypes.byref(c), fake,
                                 ctypes.byref(d), fake, fake, ws, 1 << 30, None)
    assert st == 1
    # unsupported shapes
    for kw in (dict(R=100), dict(H=65), dict(P=8), dict(R=512, P=128)):
        st = L.dsa_sparse_mla_decode(fake, fake, ctypes.byref(c), fake, ctypes.byref(_dims(**kw)),
                                     fake, fake, ws, 1 << 30, None)
        assert st == 2, kw
    st = L.dsa_indexer_scores(fake, fake, fake, ctypes.byref(c), ctypes.byref(_dims(D_I=48)),
                              fake, 8192, ws, 1 << 30, None)
    assert st == 2
    # page size other than 64
    st = L.dsa_indexer_scores(fake, fake, fake, ctypes.byref(_cache(page_size=32)),
                              ctypes.byref(d), fake, 8192, ws, 1 << 30, None)
    assert st == 2
    # decode with num_seqs != n_q
    st = L.dsa_indexer_scores(fake, fake, fake, ctypes.byref(_cache(num_seqs=2)),
                              ctypes.byref(d), fake, 8192, ws, 1 << 30, None)
    assert st == 1
    # ld too small for the longest row
    st = L.dsa_indexer_scores(fake, fake, fake, ctypes.byref(c), ctypes.byref(d), fake, 4096,
                              ws, 1 << 30, None)
    assert st == 1
    # workspace too small / misaligned
    st = L.dsa_attention_forward(fake, fake, fake, fake, fake, ctypes.byref(c), ctypes.byref(d),
                                 None, fake, fake, ws, 16, None)
    assert st == 4
    st = L.dsa_topk(fake, 8192, 1, None, 0, 16, fake, ctypes.c_void_p(0x400010), 1 << 20, None)
    assert st == 4
    # top-k with k < 1
    st = L.dsa_topk(fake, 8192, 1, None, 0, 0, fake, ws, 1 << 20, None)
    assert st == 1
    # max_seq_len beyond what the block table can address
    st = L.dsa_indexer_scores(fake, fake, fake, ctypes.byref(_cache(max_seq_len=128 * 64 + 1)),
                              ctypes.byref(d), fake, 8196, ws, 1 << 30, None)
    assert st == 1
    # FP8 keys: missing scales, D_I = 32
    st = L.dsa_indexer_scores_k8(fake, fake, fake, None, ctypes.byref(c), ctypes.byref(d), fake,
                                 8192, ws, 1 << 30, None)
    assert st == 1
    st = L.dsa_indexer_scores_k8(fake, fake, fake, fake, ctypes.byref(c),
                                 ctypes.byref(_dims(D_I=64)), fake, 8192, ws, 1 << 30, None)
    assert st == 2
    # the FP8-key indexer needs room for its query terms
    st = L.dsa_indexer_scores_k8(fake, fake, fake, fake, ctypes.byref(c), ctypes.byref(d), fake,
                                 8192, ws, 256, None)
    assert st == 4
    st = L.dsa_attention_forward_k8(fake, fake, None, fake, fake, fake, ctypes.byref(c),
                                    ctypes.byref(d), None, fake, fake, ws, 1 << 30, None)
    assert st == 1
    # absorption GEMMs: shapes outside the tiles, misaligned pointers, no workspace
    st = L.dsa_absorb_query(fake, fake, fake, fake, 4, 64, 128, 160, 64, ws, 256, None)
    assert st == 2
    st = L.dsa_absorb_query(fake, fake, fake, fake, 4, 64, 100, 512, 64, ws, 256, None)
    assert st == 2
    st = L.dsa_absorb_query(fake, ctypes.c_void_p(0x300008), fake, fake, 4, 64, 128, 512, 64, ws,
                            256, None)
    assert st == 1
    st = L.dsa_absorb_query(fake, fake, fake, fake, 4, 64, 128, 512, 64, ws, 16, None)
    assert st == 4
    st = L.dsa_project_values(fake, fake, fake, 4, 64, 512, 96, ws, 256, None)
    assert st == 2
    st = L.dsa_project_values(fake, fake, None, 4, 64, 512, 128, ws, 256, None)
    assert st == 1
    # cache append: null / misaligned pointers, unsupported widths, no workspace
    st = L.dsa_cache_append(None, fake, fake, fake, ctypes.byref(c), ctypes.byref(d), ws,
                            1 << 20, None)
    assert st == 1
    st = L.dsa_cache_append(ctypes.c_void_p(0x300008), fake, fake, fake, ctypes.byref(c),
                            ctypes.byref(d), ws, 1 << 20, None)
    assert st == 1
    st = L.dsa_cache_append(fake, fake, fake, fake, ctypes.byref(c), ctypes.byref(_dims(D_I=48)),
                            ws, 1 << 20, None)
    assert st == 2
    st = L.dsa_cache_append(fake, fake, fake, fake, ctypes.byref(c), ctypes.byref(_dims(P=8)),
                            ws, 1 << 20, None)
    assert st == 2
    st = L.dsa_cache_append(fake, fake, fake, fake, ctypes.byref(c), ctypes.byref(d), ws, 16,
                            None)
    assert st == 4
    # host-buffer step: missing host buffers, misaligned device pools, shapes,
    # a workspace without room for the staging
    hb = ctypes.c_void_p(0x500004)  # host buffers need no alignment
    n_host = L.dsa_workspace_bytes(dsa.OP_ATTENTION_FORWARD_HOST, ctypes.byref(d), ctypes.byref(c))
    n_fwd = L.dsa_workspace_bytes(dsa.OP_ATTENTION_FORWARD, ctypes.byref(d), ctypes.byref(c))
    args = lambda **kw: dict(dict(qi=hb, w=hb, kp=fake, q=hb, lp=fake, c=ctypes.byref(c),
                                  d=ctypes.byref(d), idx=hb, out=hb, lse=hb, ws=ws, n=n_host), **kw)
    call = lambda a: L.dsa_attention_forward_host(a["qi"], a["w"], a["kp"], a["q"], a["lp"], a["c"],
                                                  a["d"], a["idx"], a["out"], a["lse"], a["ws"],
                                                  a["n"], None)
    assert call(args(q=None)) == 1
    assert call(args(out=None)) == 1
    assert call(args(kp=ctypes.c_void_p(0x300008))) == 1
    assert call(args(d=ctypes.byref(_dims(R=100)))) == 2
    assert call(args(n=n_fwd)) == 4
