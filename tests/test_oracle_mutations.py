"""The oracle's pins catch plausible mistakes (no GPU needed).

Each case below plants one mistake in the float64 oracle (on the CPU, through
monkeypatch, so the module on disk is untouched) and runs the pins of
test_oracle_pins.py against it; at least one pin must fail.  A mistake that
every pin tolerates would be a hole in the evidence that the oracle computes
what the pages define.
"""

import heapq
import inspect

import numpy as np
import pytest

from oracle import dsa_oracle as orc
import test_oracle_pins as pins


def _pin_calls(golden_dir):
    """Every pin of test_oracle_pins as a zero-argument callable (a few seeds
    of the parametrised ones)."""
    calls = []
    for name, fn in sorted(vars(pins).items()):
        if not (name.startswith("test_") and inspect.isfunction(fn)):
            continue
        params = inspect.signature(fn).parameters
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if marks:
            # the first eight parameter sets of the (single) parametrize mark
            argnames, argvalues = marks[0].args[0], marks[0].args[1]
            names = [a.strip() for a in argnames.split(",")] if isinstance(argnames, str) else list(argnames)
            for j, vals in enumerate(list(argvalues)[:8]):
                kw = dict(zip(names, vals if len(names) > 1 else (vals,)))
                calls.append((f"{name}[{j}]", lambda fn=fn, kw=kw: fn(**kw)))
        elif "golden_dir" in params:
            calls.append((name, lambda fn=fn: fn(golden_dir=golden_dir)))
        else:
            calls.append((name, fn))
    return calls


def _first_failing_pin(golden_dir):
    for name, call in _pin_calls(golden_dir):
        try:
            call()
        except Exception:          # an assertion, or a crash on the planted mistake
            return name
    return None


# ---------------------------------------------------------------- mutants

def _indexer_no_relu(q_idx, w, k_idx):
    return (np.asarray(k_idx, float) @ np.asarray(q_idx, float).T) @ np.asarray(w, float)


def _indexer_relu_after_sum(q_idx, w, k_idx):
    s = (np.asarray(k_idx, float) @ np.asarray(q_idx, float).T) @ np.asarray(w, float)
    return np.maximum(s, 0.0)


def _indexer_abs_instead_of_relu(q_idx, w, k_idx):
    return np.abs(np.asarray(k_idx, float) @ np.asarray(q_idx, float).T) @ np.asarray(w, float)


def _indexer_weights_reversed(q_idx, w, k_idx):
    d = np.asarray(k_idx, float) @ np.asarray(q_idx, float).T
    return np.maximum(d, 0.0) @ np.asarray(w, float)[::-1]


def _indexer_negated_dot(q_idx, w, k_idx):
    d = -(np.asarray(k_idx, float) @ np.asarray(q_idx, float).T)
    return np.maximum(d, 0.0) @ np.asarray(w, float)


def _best_first(sc, s):
    return (-sc[s], s)


def _topk_with(key_fn=_best_first, keep=lambda k: k, order=sorted, pad=-1):
    def topk(scores, k):
        scores = [float(x) for x in scores]
        n = len(scores)
        out = np.full(k, pad, dtype=np.int64)
        if n <= k:
            out[:n] = np.arange(n)
            return out
        chosen = heapq.nsmallest(keep(k), range(n), key=lambda s: key_fn(scores, s))
        chosen = order(chosen)
        out[:len(chosen)] = chosen
        return out
    return topk


def _mla_with(scale_fn=lambda scale: scale, v_slice="head", lse_no_max=False,
              softmax_axis=1):
    def mla(q, rows, R, scale):
        q = np.asarray(q, float)
        rows = np.asarray(rows, float)
        z = scale_fn(scale) * (q @ rows.T)
        m = z.max(axis=softmax_axis, keepdims=True)
        e = np.exp(z - m)
        l = e.sum(axis=softmax_axis, keepdims=True)
        p = e / l
        v = rows[:, :R] if v_slice == "head" else rows[:, rows.shape[1] - R:]
        out = p @ v
        if softmax_axis == 1:
            lse = (0.0 if lse_no_max else m[:, 0]) + np.log(l[:, 0])
        else:
            lse = m[0] + np.log(l[0])
            lse = np.resize(lse, q.shape[0])
        return out, lse, p
    return mla


def _gather_ignores_table(pages, block_table_row, positions):
    pos = np.asarray(positions, dtype=np.int64).reshape(-1)
    return pages[pos // orc.PAGE_SIZE, pos % orc.PAGE_SIZE]


def _gather_page_off_by_one(pages, block_table_row, positions):
    pos = np.asarray(positions, dtype=np.int64).reshape(-1)
    phys = np.asarray(block_table_row, dtype=np.int64)[pos // orc.PAGE_SIZE]
    return pages[phys, (pos + 1) % orc.PAGE_SIZE]


def _bf16_shift_15(bits):
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 15).view(np.float32).astype(np.float64)


def _bf16_truncated_mantissa(bits):
    bits = np.asarray(bits, dtype=np.uint16) & np.uint16(0xFFFE)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _prefill_excludes_diagonal(inp, rows=None):
    T = inp["q_idx"].shape[0]
    rows = range(T) if rows is None else rows
    q_pos0 = int(inp.get("q_pos0", 0))
    return {int(t): orc._query_row(inp, t, inp["block_table"][0], max(1, q_pos0 + int(t)))
            for t in rows}


def _decode_sees_one_less(inp, rows=None):
    B = inp["q_idx"].shape[0]
    rows = range(B) if rows is None else rows
    return {int(b): orc._query_row(inp, b, inp["block_table"][b],
                                   max(1, int(inp["seq_lens"][b]) - 1)) for b in rows}


def _query_skips_topk(q_idx, w, k_rows, q, latent_of, k, R, scale):
    scores = orc.indexer_scores(q_idx, w, k_rows)
    idx = np.arange(min(k, len(scores)))             # the first k tokens, not the best k
    out, lse, _ = orc.mla_attention(q, latent_of(idx), R, scale)
    full = np.full(k, -1, np.int64)
    full[:len(idx)] = idx
    return {"scores": scores, "idx": full, "out": out, "lse": lse}


def _absorb_without_transpose(q_nope, q_rope, W_UK):
    H = q_nope.shape[0]
    q_lat = np.stack([np.resize(W_UK[h] @ np.resize(q_nope[h], W_UK.shape[2]), W_UK.shape[2])
                      for h in range(H)])
    return np.concatenate([q_lat, q_rope], axis=1)


def _append_one_slot_late(k_pages, latent_pages, block_table, positions, k_new, latent_new):
    shifted = [(seq, pos + 1) for seq, pos in positions]
    return _ORIG_APPEND(k_pages, latent_pages, block_table, shifted, k_new, latent_new)


def _append_positions_of_the_next_token(inp):
    return [(seq, pos + 1) for seq, pos in _ORIG_POSITIONS(inp)]


def _project_without_transpose(o_lat, W_UV):
    H = o_lat.shape[0]
    return np.stack([np.resize(W_UV[h] @ np.resize(o_lat[h], W_UV.shape[2]), W_UV.shape[2])
                     for h in range(H)])


def _e4m3_bias_8(codes):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    e, m = (c >> 3) & 0xF, (c & 0x7).astype(np.float64)
    v = np.where(e == 0, m / 8 * 2.0 ** -7, (1 + m / 8) * np.exp2(e - 8.0))
    return np.where(c & 0x80, -v, v)


def _dequantize_scale_ignored(k8_rows, scale_rows):
    return orc.e4m3_to_f64(k8_rows)


def _dequantize_scale_squared(rows, scale_rows):
    s = np.asarray(scale_rows, np.float64).reshape(-1, 1)
    return s * s * orc.e4m3_to_f64(rows)


def _cp_merge_ties_to_higher_index(cand_s, cand_i, k):
    s = np.asarray(cand_s, np.float64).reshape(-1)
    i = np.asarray(cand_i, np.int64).reshape(-1)
    valid = i >= 0
    pairs = sorted(zip(-s[valid], -i[valid]))[:k]
    out = np.full(k, -1, dtype=np.int64)
    out[:len(pairs)] = sorted(-int(g) for _, g in pairs)
    return out


def _cp_merge_partials_unweighted(outs, lses):
    outs = np.asarray(outs, np.float64)
    return outs.mean(axis=0), np.max(np.asarray(lses, np.float64), axis=0)


_ORIG_APPEND = orc.cache_append
_ORIG_POSITIONS = orc.append_positions


MUTANTS = {
    "indexer: ReLU dropped": ("indexer_scores", _indexer_no_relu),
    "indexer: ReLU after the head sum": ("indexer_scores", _indexer_relu_after_sum),
    "indexer: |x| instead of ReLU": ("indexer_scores", _indexer_abs_instead_of_relu),
    "indexer: head weights misindexed": ("indexer_scores", _indexer_weights_reversed),
    "indexer: sign of the dot flipped": ("indexer_scores", _indexer_negated_dot),
    "top-k: ties to the higher index": (
        "topk_select", _topk_with(key_fn=lambda sc, s: (-sc[s], -s))),
    "top-k: smallest scores kept": (
        "topk_select", _topk_with(key_fn=lambda sc, s: (sc[s], s))),
    "top-k: keeps k - 1": ("topk_select", _topk_with(keep=lambda k: k - 1)),
    "top-k: score order instead of ascending": ("topk_select", _topk_with(order=list)),
    "top-k: padded with 0": ("topk_select", _topk_with(pad=0)),
    "MLA: scale dropped": ("mla_attention", _mla_with(scale_fn=lambda scale: 1.0)),
    "MLA: scale applied twice": ("mla_attention", _mla_with(scale_fn=lambda scale: scale ** 2)),
    "MLA: V taken from the tail of the row": ("mla_attention", _mla_with(v_slice="tail")),
    "MLA: lse without the max": ("mla_attention", _mla_with(lse_no_max=True)),
    "MLA: softmax over heads": ("mla_attention", _mla_with(softmax_axis=0)),
    "paging: block table ignored": ("gather_paged_rows", _gather_ignores_table),
    "paging: slot off by one": ("gather_paged_rows", _gather_page_off_by_one),
    "bf16: shifted by 15": ("bf16_to_f64", _bf16_shift_15),
    "bf16: last mantissa bit dropped": ("bf16_to_f64", _bf16_truncated_mantissa),
    "prefill: diagonal not visible": ("dsa_prefill", _prefill_excludes_diagonal),
    "decode: last token not visible": ("dsa_decode", _decode_sees_one_less),
    "step: selection skipped": ("dsa_query", _query_skips_topk),
    "absorption: W_UK not transposed": ("absorb_query", _absorb_without_transpose),
    "append: written one slot late": ("cache_append", _append_one_slot_late),
    "projection: W_UV not transposed": ("project_values", _project_without_transpose),
    "e4m3: exponent bias 8": ("e4m3_to_f64", _e4m3_bias_8),
    "cp: candidate ties to the higher index": ("cp_merge_candidates", _cp_merge_ties_to_higher_index),
    "cp: partials averaged without LSE weights": ("cp_merge_partials", _cp_merge_partials_unweighted),
    "fp8 keys: scale ignored": ("dequantize_keys", _dequantize_scale_ignored),
    "fp8 latent: scale ignored": ("dequantize_latent", _dequantize_scale_ignored),
    "fp8 latent: scale applied to the codes' exponent twice": ("dequantize_latent",
                                                               _dequantize_scale_squared),
    "append: the next token's position": ("append_positions", _append_positions_of_the_next_token),
}


def test_unmutated_oracle_passes_every_pin(golden_dir):
    assert _first_failing_pin(golden_dir) is None


@pytest.mark.parametrize("label", sorted(MUTANTS))
def test_planted_mistake_is_caught(label, golden_dir, monkeypatch):
    target, mutant = MUTANTS[label]
    monkeypatch.setattr(orc, target, mutant)
    caught = _first_failing_pin(golden_dir)
    assert caught is not None, f"no pin catches: {label}"
