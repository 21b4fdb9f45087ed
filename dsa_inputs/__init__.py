"""Seeded synthetic inputs for the DSA step, shared by the tests, the bench and
the smoke check.

This module only draws numbers and lays them out; it holds none of the
method's arithmetic.  Every array is NumPy: bf16 tensors are raw uint16 bit
patterns (round-to-nearest-even from float32), index tensors are int32,
weights float32.

Recipe (all configs): a NumPy Generator(PCG64(seed)) draws, in this order,
  q_idx   integers in [-3, 3]            -> bf16   [n_q, H_I, D_I]
  k_pages integers in [-3, 3]            -> bf16   [num_pages, 64, D_I]
  w       integers in [0, 3]             -> float32 [n_q, H_I]
  q       float32 standard normal        -> bf16   [n_q, H, R + P]
  latent  float32 standard normal        -> bf16   [num_pages, 64, R + P]
  then, when `shuffle_pages`, a permutation of the physical pages.
Normals are drawn in fixed chunks of 2**22 values.  Sequence lengths of the
ragged batched config are drawn first, from their own Generator(PCG64(1)),
uniformly in [2048, 65536].  Integer index queries/keys make every fp32
indexer score exact, as in the workloads the step is quoted on.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np

PAGE_SIZE = 64
_CHUNK = 1 << 22


@dataclass(frozen=True)
class Workload:
    name: str
    mode: str                 # "decode" or "prefill"
    seq_lens: tuple           # decode: per-sequence context (incl. current token)
    n_q: int                  # query rows (decode: B; prefill: T)
    H_I: int
    D_I: int
    topk: int
    H: int
    R: int
    P: int
    scale: float
    seed: int = 0
    shuffle_pages: bool = False
    q_pos0: int = 0           # prefill: absolute position of query row 0
    value_kind: str = "int"   # "int": index q/k integers; "normal": bf16 N(0,1)
    description: str = ""

    @property
    def W(self) -> int:
        return self.R + self.P

    @property
    def num_seqs(self) -> int:
        return len(self.seq_lens)


def ragged_lengths(batch: int, lo: int, hi: int, seed: int) -> tuple:
    rng = np.random.Generator(np.random.PCG64(seed))
    return tuple(int(x) for x in rng.integers(lo, hi + 1, size=batch))


CONFIGS = {
    "tiny_decode": Workload(
        name="tiny_decode", mode="decode", seq_lens=(4096,), n_q=1, H_I=4, D_I=32,
        topk=256, H=4, R=64, P=16, scale=1.0 / math.sqrt(80.0), seed=0,
        description="batch 1, context 4,096; indexer 4x32; top-k 256; MLA 4 heads, latent 64+16"),
    "glm5_decode_8k": Workload(
        name="glm5_decode_8k", mode="decode", seq_lens=(8192,), n_q=1, H_I=32, D_I=128,
        topk=2048, H=64, R=512, P=64, scale=1.0 / math.sqrt(192.0), seed=0,
        description="batch 1, context 8,192; indexer 32x128; top-k 2,048; MLA 64 heads, 512+64"),
    "glm5_decode_b32_ragged": Workload(
        name="glm5_decode_b32_ragged", mode="decode",
        seq_lens=ragged_lengths(32, 2048, 65536, 1), n_q=32, H_I=32, D_I=128,
        topk=2048, H=64, R=512, P=64, scale=1.0 / math.sqrt(192.0), seed=2,
        shuffle_pages=True,
        description="batch 32, contexts U[2,048, 65,536] (seed 1), shuffled 64-token pages"),
    "glm5_prefill_2300": Workload(
        name="glm5_prefill_2300", mode="prefill", seq_lens=(2300,), n_q=2300, H_I=32,
        D_I=128, topk=2048, H=64, R=512, P=64, scale=1.0 / math.sqrt(192.0), seed=0,
        description="causal prefill chunk of 2,300 tokens; top-k 2,048 per row"),
    "glm5_decode_4x128k": Workload(
        name="glm5_decode_4x128k", mode="decode", seq_lens=(131072,) * 4, n_q=4, H_I=32,
        D_I=128, topk=2048, H=64, R=512, P=64, scale=1.0 / math.sqrt(192.0), seed=0,
        description="batch 4, context 131,072 each; indexer key scan dominates"),
}
CONFIG_ORDER = ["tiny_decode", "glm5_decode_8k", "glm5_decode_b32_ragged",
                "glm5_prefill_2300", "glm5_decode_4x128k"]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + rounding) >> 16).astype(np.uint16)


def _ints_bf16(rng, lo, hi, shape):
    vals = rng.integers(lo, hi + 1, size=shape).astype(np.float32)
    return f32_to_bf16_bits(vals)


def _normal_bf16(rng, shape):
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for start in range(0, n, _CHUNK):
        m = min(_CHUNK, n - start)
        out[start:start + m] = f32_to_bf16_bits(rng.standard_normal(m, dtype=np.float32))
    return out.reshape(shape)


def pages_needed(n_tokens: int) -> int:
    return (n_tokens + PAGE_SIZE - 1) // PAGE_SIZE


def make_inputs(wl: Workload) -> dict:
    """Draw the arrays of one workload.  Returns a dict of NumPy arrays and scalars."""
    rng = np.random.Generator(np.random.PCG64(wl.seed))
    if wl.mode == "decode":
        lens = list(wl.seq_lens)
        assert len(lens) == wl.n_q
    else:
        lens = [wl.q_pos0 + wl.n_q]
    npages = [pages_needed(n) for n in lens]
    num_pages = int(sum(npages))
    max_pages = max(1, max(npages))

    if wl.value_kind == "int":
        q_idx = _ints_bf16(rng, -3, 3, (wl.n_q, wl.H_I, wl.D_I))
        k_pages = _ints_bf16(rng, -3, 3, (num_pages, PAGE_SIZE, wl.D_I))
    else:
        q_idx = _normal_bf16(rng, (wl.n_q, wl.H_I, wl.D_I))
        k_pages = _normal_bf16(rng, (num_pages, PAGE_SIZE, wl.D_I))
    w = rng.integers(0, 4, size=(wl.n_q, wl.H_I)).astype(np.float32)
    q = _normal_bf16(rng, (wl.n_q, wl.H, wl.W))
    latent_pages = _normal_bf16(rng, (num_pages, PAGE_SIZE, wl.W))

    phys = np.arange(num_pages, dtype=np.int64)
    if wl.shuffle_pages:
        phys = rng.permutation(num_pages)
    block_table = np.full((len(lens), max_pages), -1, dtype=np.int32)
    start = 0
    for b, npg in enumerate(npages):
        block_table[b, :npg] = phys[start:start + npg]
        start += npg

    return {
        "mode": wl.mode,
        "q_idx": q_idx, "w": w, "k_pages": k_pages,
        "q": q, "latent_pages": latent_pages,
        "block_table": block_table,
        "seq_lens": np.asarray(lens, dtype=np.int32),
        "topk": wl.topk, "R": wl.R, "P": wl.P, "H": wl.H,
        "H_I": wl.H_I, "D_I": wl.D_I, "scale": wl.scale,
        "q_pos0": wl.q_pos0, "n_q": wl.n_q,
    }


def small_decode(seq_lens, *, H_I=4, D_I=32, topk=64, H=8, R=64, P=16, seed=0,
                 shuffle_pages=True, value_kind="int", scale=None) -> Workload:
    """A small decode workload for parity tests (several tiles, ragged tails)."""
    W = R + P
    return Workload(name="small_decode", mode="decode", seq_lens=tuple(seq_lens),
                    n_q=len(seq_lens), H_I=H_I, D_I=D_I, topk=topk, H=H, R=R, P=P,
                    scale=(1.0 / math.sqrt(W)) if scale is None else scale, seed=seed,
                    shuffle_pages=shuffle_pages, value_kind=value_kind)


def small_prefill(T, *, q_pos0=0, H_I=4, D_I=32, topk=64, H=8, R=64, P=16, seed=0,
                  shuffle_pages=True, value_kind="int", scale=None) -> Workload:
    W = R + P
    return Workload(name="small_prefill", mode="prefill", seq_lens=(q_pos0 + T,), n_q=T,
                    H_I=H_I, D_I=D_I, topk=topk, H=H, R=R, P=P,
                    scale=(1.0 / math.sqrt(W)) if scale is None else scale, seed=seed,
                    shuffle_pages=shuffle_pages, q_pos0=q_pos0, value_kind=value_kind)


__all__ = ["Workload", "CONFIGS", "CONFIG_ORDER", "make_inputs", "f32_to_bf16_bits", "with_fp8_latent",
           "small_decode", "small_prefill", "ragged_lengths", "pages_needed", "PAGE_SIZE",
           "replace", "field"]


def with_fp8_keys(inp: dict, seed: int = 0, max_shift: int = 7) -> dict:
    """The same inputs with the index-key cache held as E4M3 bytes plus one
    fp32 scale per token: each token's integer key k is stored as the codes of
    k * 2^j and the scale 2^-j, j drawn per token in [0, max_shift] (seeded),
    so the keys the codes stand for are the original ones exactly.  The codes
    come from torch's float8_e4m3fn conversion (exact for these values)."""
    import torch
    k = (inp["k_pages"].astype(np.uint32) << 16).view(np.float32)   # bf16 -> f32, exact
    if not np.array_equal(k, np.round(k)) or np.abs(k).max() * 2 ** max_shift > 448:
        raise ValueError("FP8 key inputs need integer keys within E4M3 range")
    rng = np.random.default_rng(np.random.PCG64([seed, 0xF8]))
    j = rng.integers(0, max_shift + 1, k.shape[:2])                # one shift per token
    scaled = k * np.exp2(j)[..., None].astype(np.float32)
    codes = torch.from_numpy(np.ascontiguousarray(scaled)).to(torch.float8_e4m3fn).view(torch.uint8)
    out = dict(inp)
    out["k8_pages"] = codes.numpy()
    out["k_scale"] = np.exp2(-j).astype(np.float32).reshape(-1)
    return out


def with_fp8_latent(inp: dict, seed: int = 0, max_shift: int = 4) -> dict:
    """The same inputs with the latent cache held as E4M3 bytes plus one fp32
    scale per token.  Each token's latent row x (the bf16 values) is stored as
    the codes of x * 2^j and the scale 2^-j, j drawn per token in
    [0, max_shift] (seeded); the codes come from torch's float8_e4m3fn
    conversion (round to nearest even).  The returned "latent_pages" is
    replaced by the bf16 bits of the rows the codes stand for (exact: every
    E4M3 value times a power of two in this range is a bf16 value), so the
    bf16 and the FP8 inputs describe the same latent cache."""
    import torch
    pages = inp["latent_pages"]
    rng = np.random.default_rng(np.random.PCG64([seed, 0x1A7]))
    j = rng.integers(0, max_shift + 1, pages.shape[:2])                  # one shift per token
    codes_all = np.empty(pages.shape, np.uint8)
    bits_all = np.empty(pages.shape, np.uint16)
    for p0 in range(0, pages.shape[0], 2048):                           # bounded host memory
        p1 = min(p0 + 2048, pages.shape[0])
        lat = (pages[p0:p1].astype(np.uint32) << 16).view(np.float32)   # bf16 -> f32, exact
        if np.abs(lat).max() * 2 ** max_shift > 448:
            raise ValueError("latent values too large for E4M3 at this shift")
        scaled = lat * np.exp2(j[p0:p1])[..., None].astype(np.float32)
        codes = torch.from_numpy(np.ascontiguousarray(scaled)).to(torch.float8_e4m3fn)
        back = codes.to(torch.float32).numpy() * np.exp2(-j[p0:p1])[..., None].astype(np.float32)
        codes_all[p0:p1] = codes.view(torch.uint8).numpy()
        bits_all[p0:p1] = f32_to_bf16_bits(back)
    out = dict(inp)
    out["latent8_pages"] = codes_all
    out["latent_scale"] = np.exp2(-j).astype(np.float32).reshape(-1)
    out["latent_pages"] = bits_all
    return out


def shard_bounds(n: int, ranks: int) -> np.ndarray:
    """Key-range boundaries of n keys split over ranks: [bounds[i], bounds[i+1])."""
    return np.linspace(0, n, ranks + 1).astype(np.int64)


def shard_inputs(inp: dict, lo, hi) -> dict:
    """The keys [lo[b], hi[b]) of every sequence b (index keys and latent rows)
    as inputs of their own, re-paged from local position 0 with an identity
    block table; "offsets" holds lo.  Queries and weights are unchanged."""
    lo, hi = np.asarray(lo, np.int64), np.asarray(hi, np.int64)
    lens = (hi - lo).astype(np.int32)
    B = len(lens)
    maxp = max(1, max(pages_needed(int(n)) for n in lens))
    D, Wd = inp["k_pages"].shape[2], inp["latent_pages"].shape[2]
    kp, lp = [], []
    bt = np.full((B, maxp), -1, dtype=np.int32)
    for b in range(B):
        pos = np.arange(lo[b], hi[b])
        phys = inp["block_table"][b][pos // 64].astype(np.int64) * 64 + pos % 64
        k_rows = inp["k_pages"].reshape(-1, D)[phys]
        l_rows = inp["latent_pages"].reshape(-1, Wd)[phys]
        for j in range(pages_needed(int(lens[b]))):
            kpg = np.zeros((64, D), dtype=np.uint16)
            lpg = np.zeros((64, Wd), dtype=np.uint16)
            kpg[:len(k_rows[64 * j:64 * j + 64])] = k_rows[64 * j:64 * j + 64]
            lpg[:len(l_rows[64 * j:64 * j + 64])] = l_rows[64 * j:64 * j + 64]
            bt[b, j] = len(kp)
            kp.append(kpg)
            lp.append(lpg)
    if not kp:
        kp.append(np.zeros((64, D), np.uint16))
        lp.append(np.zeros((64, Wd), np.uint16))
    out = dict(inp)
    out.update(k_pages=np.stack(kp), latent_pages=np.stack(lp), block_table=bt, seq_lens=lens,
               offsets=lo.astype(np.int32))
    return out
