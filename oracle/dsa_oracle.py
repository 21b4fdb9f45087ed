"""Float64 CPU oracle for the DSA sparse-attention step (TEST INFRASTRUCTURE ONLY).

This module is the plain, slow definition that the CUDA library is checked
against.  Only the test suite, the smoke check and the CPU-baseline leg of the
benchmark may import it; the product path never does, and this module imports
nothing from the product.  It shares no code, tables or constants with the CUDA
kernels: inputs arrive as NumPy arrays (bf16 values as raw uint16 bits) and
every step is written out in float64.

What it computes (one query row), after the new tokens' rows have been
appended to the paged caches (cache_append):

1. Indexer scores.  "GLM on an A100, in Vx", section "The model": a separate
   indexer scores every earlier token; section "How do we know it is right?":
   the indexer applies a ReLU per indexer head before the heads are combined.
   Reading used here: score[s] = sum_h w[h] * max(0, q_idx[h] . k_idx[s]),
   one index key per token shared by all indexer heads, no extra scale.
2. Exact top-k.  Same page, "The model": each query keeps the 2,048 highest
   scores, everything when fewer tokens exist; "How do we know it is right?":
   ties resolve like a stable argsort of -scores (lower token index first).
   "Self-contained GLM-5 serving stack ..." names exact heap selection among
   its implemented optimizations; the oracle selects with a heap.
   The kept indices are emitted in ascending token order, padded with -1.
3. Absorbed MLA attention over the compressed latent rows of the kept tokens
   only.  "Self-contained GLM-5 serving stack ...", file list (glm_vx/model.py):
   absorbed MLA decode over compressed request-local KV; "GLM on an A100, in
   Vx", "The model": keys and values are compressed into one small latent
   vector per token.  Each latent row is [c_kv (R) | k_rope (P)]; the absorbed
   query has the same layout; V is the c_kv part.
   z[h, j] = scale * q[h, :] . L[sel_j, :];  p = softmax_j(z);
   out[h, :] = sum_j p[h, j] * L[sel_j, :R];  lse[h] = log sum_j exp(z[h, j]).

Every function here is pinned by tests that do not re-type its formula:
hand-computed golden values, closed forms, brute force over all subsets on
tiny inputs, the stable-argsort library rule, dense-vs-sparse and
absorbed-vs-non-absorbed identities, and special cases.
"""

from __future__ import annotations

import heapq
import math

import numpy as np

PAGE_SIZE = 64


# --------------------------------------------------------------------------
# bf16 decoding of the input bits (exact widening)
# --------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bit patterns (uint16) to float64 exactly.

    A bf16 value is the upper half of an IEEE binary32; placing the 16 bits
    in the high half of a 32-bit word and reading it as float32 is exact, and
    float32 -> float64 is exact.
    """
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """Widen E4M3 bytes to float64 exactly ("GLM on an A100, in Vx", section
    "INT4, FP8 and BF16": E4M3 bytes).  Bit 7 is the sign, bits 6..3 the
    exponent with bias 7, bits 2..0 the mantissa; exponent 0 holds subnormals
    (m / 8 * 2^-6); exponent 15 with mantissa 7 is NaN (there is no infinity).
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e - 7.0)
    sub = (m / 8.0) * 2.0 ** -6
    v = sign * np.where(e == 0, sub, normal)
    return np.where((e == 15) & ((c & 0x7) == 7), np.nan, v)


def dequantize_keys(k8_rows: np.ndarray, scale_rows: np.ndarray) -> np.ndarray:
    """Index keys from E4M3 codes [n, D_I] and one fp32 scale per token [n]:
    the FP8 format the pages describe, with a block of one token's key."""
    return np.asarray(scale_rows, np.float64).reshape(-1, 1) * e4m3_to_f64(k8_rows)


def dequantize_latent(l8_rows: np.ndarray, scale_rows: np.ndarray) -> np.ndarray:
    """Latent rows from E4M3 codes [n, W] and one fp32 scale per token [n]
    ("GLM on an A100, in Vx", section "INT4, FP8 and BF16": E4M3 bytes with a
    float32 scale per block; here the block is one token's whole latent row
    [c_kv | k_rope]).  The dequantized row serves as key and value exactly as a
    bf16 row does: z uses all W columns, V the first R."""
    return np.asarray(scale_rows, np.float64).reshape(-1, 1) * e4m3_to_f64(l8_rows)


# --------------------------------------------------------------------------
# paged cache lookup
# --------------------------------------------------------------------------

def gather_paged_rows(pages: np.ndarray, block_table_row: np.ndarray,
                      positions) -> np.ndarray:
    """Rows of a paged cache at the given token positions of one sequence.

    pages: [num_pages, PAGE_SIZE, width]; block_table_row: physical page id of
    each logical page of the sequence.  Token position s lives in logical page
    s // PAGE_SIZE, slot s % PAGE_SIZE.
    """
    pos = np.asarray(positions, dtype=np.int64).reshape(-1)
    phys = np.asarray(block_table_row, dtype=np.int64)[pos // PAGE_SIZE]
    return pages[phys, pos % PAGE_SIZE]


# --------------------------------------------------------------------------
# the step in front of the indexer: appending the new tokens to the caches
# --------------------------------------------------------------------------

def append_positions(inp: dict) -> list:
    """(sequence, position) that each new row of the step is written to.

    Decode row b is the query at position seq_lens[b] - 1 of sequence b (its
    own token is part of the context it scores); prefill row t sits at
    position q_pos0 + t of sequence 0.
    """
    if inp.get("mode") == "prefill":
        return [(0, int(inp["q_pos0"]) + t) for t in range(inp["q_idx"].shape[0])]
    return [(b, int(n) - 1) for b, n in enumerate(inp["seq_lens"])]


def cache_append(k_pages, latent_pages, block_table, positions, k_new, latent_new):
    """The page pools after writing row i of k_new / latent_new at (seq, pos) =
    positions[i].  "Self-contained GLM-5 serving stack ...", file list: the
    decode runs over compressed request-local KV, one compressed row per token,
    plus the indexer's key for that token.  Returns new arrays (the inputs are
    not modified); raises on a position outside the block table or an invalid
    page id.
    """
    k_out = np.array(k_pages, copy=True)
    l_out = np.array(latent_pages, copy=True)
    for i, (seq, pos) in enumerate(positions):
        if pos < 0 or pos // PAGE_SIZE >= block_table.shape[1]:
            raise ValueError(f"row {i}: position {pos} outside the block table")
        page = int(block_table[seq, pos // PAGE_SIZE])
        if page < 0 or page >= k_out.shape[0]:
            raise ValueError(f"row {i}: page id {page} outside the pool")
        k_out[page, pos % PAGE_SIZE] = k_new[i]
        l_out[page, pos % PAGE_SIZE] = latent_new[i]
    return k_out, l_out


# --------------------------------------------------------------------------
# step 1: indexer scores
# --------------------------------------------------------------------------

def indexer_scores(q_idx: np.ndarray, w: np.ndarray, k_idx: np.ndarray) -> np.ndarray:
    """score[s] = sum_h w[h] * relu(q_idx[h] . k_idx[s]) in float64.

    q_idx: [H_I, D_I] float64; w: [H_I] float64; k_idx: [n, D_I] float64.
    Returns [n] float64.
    """
    q_idx = np.asarray(q_idx, dtype=np.float64)
    k_idx = np.asarray(k_idx, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    dots = k_idx @ q_idx.T                 # [n, H_I]: one dot per key and head
    relu = np.where(dots > 0.0, dots, 0.0)  # ReLU per indexer head
    return relu @ w                         # head-weighted sum


# --------------------------------------------------------------------------
# step 2: exact top-k with the stable tie rule
# --------------------------------------------------------------------------

def topk_select(scores, k: int) -> np.ndarray:
    """Indices of the k best tokens, ascending, padded with -1 to length k.

    "Best" follows a stable argsort of -scores: a higher score first, and at
    equal scores the lower token index first.  With n <= k every token is kept.
    Scores are compared as float64 values, so -0.0 and +0.0 are equal.
    """
    scores = [float(x) for x in scores]
    n = len(scores)
    out = np.full(k, -1, dtype=np.int64)
    if n <= k:
        out[:n] = np.arange(n)
        return out
    # a heap selection of the k smallest keys (-score, index)
    chosen = heapq.nsmallest(k, range(n), key=lambda s: (-scores[s], s))
    out[:] = sorted(chosen)
    return out


# --------------------------------------------------------------------------
# step 3: absorbed MLA over the selected latent rows
# --------------------------------------------------------------------------

def mla_attention(q: np.ndarray, rows: np.ndarray, R: int, scale: float):
    """Absorbed MLA attention of one query row over the given latent rows.

    q: [H, W] float64 absorbed query ([latent part R | rope part P]);
    rows: [n, W] float64 latent rows, n >= 1.
    Returns (out [H, R], lse [H], p [H, n]) in float64, lse in natural log.
    """
    q = np.asarray(q, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.float64)
    z = scale * (q @ rows.T)                       # [H, n] logits
    m = z.max(axis=1, keepdims=True)               # stable softmax: subtract the max
    e = np.exp(z - m)
    l = e.sum(axis=1, keepdims=True)
    p = e / l
    out = p @ rows[:, :R]                          # V is the c_kv part of the latent
    lse = m[:, 0] + np.log(l[:, 0])
    return out, lse, p


def dense_mla_attention(q: np.ndarray, latent: np.ndarray, R: int, scale: float):
    """MLA attention of one query over ALL given latent rows, no selection.

    Written separately from mla_attention (explicit per-head loops over the
    keys) so that the sparse == dense identity below the top-k size compares
    two independent routines.
    """
    q = np.asarray(q, dtype=np.float64)
    latent = np.asarray(latent, dtype=np.float64)
    H = q.shape[0]
    n = latent.shape[0]
    out = np.zeros((H, R))
    lse = np.zeros(H)
    for h in range(H):
        logits = [scale * float(np.dot(q[h], latent[j])) for j in range(n)]
        top = max(logits)
        weights = [math.exp(x - top) for x in logits]
        total = math.fsum(weights)
        acc = np.zeros(R)
        for j in range(n):
            acc += (weights[j] / total) * latent[j, :R]
        out[h] = acc
        lse[h] = top + math.log(total)
    return out, lse


def mla_attention_nonabsorbed(q_nope, q_rope, c_kv, k_rope, W_UK, W_UV, scale):
    """Standard (non-absorbed) multi-head attention that MLA absorption rewrites.

    Per head h: k_h[s] = [W_UK[h] @ c_kv[s] | k_rope[s]], v_h[s] = c_kv[s] @ W_UV[h],
    q_h = [q_nope[h] | q_rope[h]]; out_h = softmax(scale * q_h . k_h) @ v_h.
    q_nope [H, d_nope], q_rope [H, P], c_kv [n, R], k_rope [n, P],
    W_UK [H, d_nope, R], W_UV [H, R, d_v].  Returns (out [H, d_v], lse [H]).
    """
    H = q_nope.shape[0]
    n = c_kv.shape[0]
    d_v = W_UV.shape[2]
    out = np.zeros((H, d_v))
    lse = np.zeros(H)
    for h in range(H):
        k_nope = c_kv @ W_UK[h].T                   # [n, d_nope]
        keys = np.concatenate([k_nope, k_rope], axis=1)
        query = np.concatenate([q_nope[h], q_rope[h]])
        values = c_kv @ W_UV[h]                     # [n, d_v]
        z = scale * (keys @ query)
        m = z.max()
        e = np.exp(z - m)
        out[h] = (e / e.sum()) @ values
        lse[h] = m + np.log(e.sum())
    return out, lse


def absorb_query(q_nope, q_rope, W_UK):
    """Absorbed query [H, R + P]: q_lat[h] = W_UK[h]^T q_nope[h], rope part unchanged."""
    H = q_nope.shape[0]
    q_lat = np.stack([W_UK[h].T @ q_nope[h] for h in range(H)])
    return np.concatenate([q_lat, q_rope], axis=1)


def project_values(o_lat, W_UV):
    """Per-head value up-projection of the latent-space output:
    v[h] = W_UV[h]^T o_lat[h].  o_lat [H, R], W_UV [H, R, d_v] -> [H, d_v]."""
    H = o_lat.shape[0]
    return np.stack([W_UV[h].T @ o_lat[h] for h in range(H)])


# --------------------------------------------------------------------------
# the whole step
# --------------------------------------------------------------------------

def dsa_query(q_idx, w, k_rows, q, latent_of, k: int, R: int, scale: float):
    """One query row of the DSA step over its own context (float64 inputs).

    q_idx [H_I, D_I], w [H_I], k_rows [n, D_I] (index keys of tokens 0..n-1),
    q [H, W]; latent_of(positions) returns the float64 latent rows [len, W] of
    those token positions.  Returns dict(scores, idx, out, lse).
    """
    scores = indexer_scores(q_idx, w, k_rows)
    idx = topk_select(scores, k)
    sel = idx[idx >= 0]
    out, lse, _ = mla_attention(q, latent_of(sel), R, scale)
    return {"scores": scores, "idx": idx, "out": out, "lse": lse}


def _query_row(inp, r, table_row, n):
    if "k8_pages" in inp:   # FP8 index keys with one scale per token
        codes = gather_paged_rows(inp["k8_pages"], table_row, np.arange(n))
        scales = gather_paged_rows(np.asarray(inp["k_scale"]).reshape(-1, PAGE_SIZE, 1), table_row,
                                   np.arange(n))
        k_rows = dequantize_keys(codes, scales)
    else:
        k_rows = bf16_to_f64(gather_paged_rows(inp["k_pages"], table_row, np.arange(n)))

    def latent_of(sel):
        if "latent8_pages" in inp:   # FP8 latent rows with one scale per token
            codes = gather_paged_rows(inp["latent8_pages"], table_row, sel)
            scales = gather_paged_rows(np.asarray(inp["latent_scale"]).reshape(-1, PAGE_SIZE, 1),
                                       table_row, sel)
            return dequantize_latent(codes, scales)
        return bf16_to_f64(gather_paged_rows(inp["latent_pages"], table_row, sel))

    return dsa_query(bf16_to_f64(inp["q_idx"][r]), np.asarray(inp["w"][r], np.float64),
                     k_rows, bf16_to_f64(inp["q"][r]), latent_of,
                     int(inp["topk"]), int(inp["R"]), float(inp["scale"]))


def dsa_decode(inp: dict, rows=None) -> dict:
    """Decode step over a paged cache, from the raw input arrays.

    inp keys: q_idx [B, H_I, D_I] u16, w [B, H_I] f32, k_pages [pages, 64, D_I] u16,
    q [B, H, W] u16, latent_pages [pages, 64, W] u16, block_table [B, maxp] i32,
    seq_lens [B] i32, topk, R, scale.  The query of sequence b sits at position
    seq_lens[b] - 1 and sees tokens 0..seq_lens[b]-1.  `rows` restricts the
    computation to those sequences.
    """
    B = inp["q_idx"].shape[0]
    rows = range(B) if rows is None else rows
    return {int(b): _query_row(inp, b, inp["block_table"][b], int(inp["seq_lens"][b]))
            for b in rows}


def dsa_prefill(inp: dict, rows=None) -> dict:
    """Causal prefill of one sequence: query row t sits at position q_pos0 + t
    and sees tokens 0..q_pos0+t (diagonal included).

    inp keys as in dsa_decode, with q_idx [T, H_I, D_I], w [T, H_I], q [T, H, W],
    a single block-table row block_table [1, maxp] and q_pos0.
    """
    T = inp["q_idx"].shape[0]
    rows = range(T) if rows is None else rows
    q_pos0 = int(inp.get("q_pos0", 0))
    return {int(t): _query_row(inp, t, inp["block_table"][0], q_pos0 + int(t) + 1)
            for t in rows}


# --------------------------------------------------------------------------
# context-parallel decode of one long sequence (key range split over ranks)
# --------------------------------------------------------------------------

def cp_local_candidates(scores_local: np.ndarray, k: int, offset: int):
    """One rank's candidates: its exact top-k over its own key range, as
    (score, global index) pairs in ascending index order, padded with
    (-inf, -1).  "GLM on an A100, in Vx", "The model": a context of up to
    1,048,576 tokens; each query keeps the k best-scoring earlier tokens."""
    sel = topk_select(scores_local, k)
    cand_s = np.full(k, -np.inf)
    cand_i = np.full(k, -1, dtype=np.int64)
    m = sel >= 0
    cand_s[m] = np.asarray(scores_local, np.float64)[sel[m]]
    cand_i[m] = offset + sel[m]
    return cand_s, cand_i


def cp_merge_candidates(cand_s: np.ndarray, cand_i: np.ndarray, k: int) -> np.ndarray:
    """The global top-k from every rank's candidates ([R, k] each, ranks in
    key-range order): the best k valid pairs by (-score, global index),
    ascending, padded with -1.  A token of the global top-k is in its own
    rank's local top-k, so nothing is lost."""
    s = np.asarray(cand_s, np.float64).reshape(-1)
    i = np.asarray(cand_i, np.int64).reshape(-1)
    valid = i >= 0
    pairs = sorted(zip(-s[valid], i[valid]))[:k]
    out = np.full(k, -1, dtype=np.int64)
    out[:len(pairs)] = sorted(int(g) for _, g in pairs)
    return out


def cp_merge_partials(outs, lses):
    """Attention over the union of disjoint key sets from each set's own
    normalised output and log-sum-exp: out = sum_r exp(lse_r - L) out_r with
    L = log sum_r exp(lse_r); a set with no key has lse = -inf."""
    lses = np.asarray(lses, np.float64)          # [R, H]
    outs = np.asarray(outs, np.float64)          # [R, H, dv]
    top = np.max(lses, axis=0)
    fin = np.isfinite(top)
    wts = np.where(np.isfinite(lses), np.exp(lses - np.where(fin, top, 0.0)), 0.0)
    tot = wts.sum(axis=0)
    out = np.einsum("rh,rhd->hd", wts, outs) / np.where(tot > 0, tot, 1.0)[:, None]
    lse = np.where(tot > 0, top + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    return out, lse
