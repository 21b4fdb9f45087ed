#!/usr/bin/env python
"""Benchmark of the DSA sparse-attention step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config NAME] [--no-extra]

One step = one dsa_attention_forward call (indexer scores -> exact top-k ->
sparse MLA -> split combine) over one batch of synthetic GLM-5-shaped input
already resident in HBM.  The headline workload is the batched GLM-5-width
decode (32 sequences, contexts 2,048-65,536, ragged paged caches), the largest
workload that is a decode on one GPU; every other workload is measured too and
reported under "per_config".  L2 is flushed (a 512 MB read) before every timed
step; each step is timed with CUDA events on the launching stream; the same
step with L2 left warm is reported as "hot", and through the host-buffer entry
point (inputs and results in pinned host memory) as "e2e", for the headline
and every other bf16 workload.  Multi-GPU runs are independent
replicas (weak scaling) timed as the max over ranks.

`--impl reference` times the float64 CPU oracle on this host's cores on the
same workload (bounded samples), with the same JSON keys.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import dsa_inputs as di  # noqa: E402

HEADLINE = "glm5_decode_b32_ragged"
EXTRA = ["tiny_decode", "glm5_decode_8k", "glm5_prefill_2300", "glm5_decode_4x128k"]
# the same workloads with the index keys held as E4M3 bytes + one scale per token
EXTRA_K8 = ["glm5_decode_8k", "glm5_decode_b32_ragged", "glm5_decode_4x128k"]
# ... and with both caches (index keys and latent rows) in that format
EXTRA_FP8 = ["glm5_decode_b32_ragged", "glm5_decode_4x128k", "glm5_decode_8k"]
NOMINAL_HBM_GBS = 8000.0
FLUSH_BYTES = 512 << 20


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# ---------------------------------------------------------------------------
# workload arithmetic (algorithmic bytes / flops)
# ---------------------------------------------------------------------------

def row_lengths(wl):
    if wl.mode == "prefill":
        return [wl.q_pos0 + t + 1 for t in range(wl.n_q)]
    return list(wl.seq_lens)


def algorithmic(wl, k8=False, l8=False):
    """Must-move bytes and flops of one step (scores and page tables excluded).
    k8: the index keys as E4M3 bytes plus a 4-byte scale per token; l8: the
    latent rows likewise."""
    lens = row_lengths(wl)
    keys = sum(lens)
    sel = sum(min(wl.topk, n) for n in lens)
    key_bytes = (wl.D_I + 4) if k8 else wl.D_I * 2
    row_bytes = (wl.W + 4) if l8 else wl.W * 2
    b_keys = keys * key_bytes
    b_lat = sel * row_bytes
    b_small = wl.n_q * (wl.H * wl.W * 2 + wl.H_I * wl.D_I * 2 + wl.H_I * 4 + wl.H * wl.R * 4
                        + wl.H * 4)
    if wl.mode == "prefill":   # every row reads the same (L2-resident) cache
        b_keys = (wl.q_pos0 + wl.n_q) * key_bytes
        b_lat = (wl.q_pos0 + wl.n_q) * row_bytes
    flops_idx = 2 * wl.H_I * wl.D_I * keys
    flops_mla = sel * wl.H * 2 * (wl.W + wl.R)
    # indexer kernel alone: key rows read + fp32 score per key written
    b_indexer = keys * (key_bytes + 4) + wl.n_q * wl.H_I * (wl.D_I * 2 + 4)
    if wl.mode == "prefill":
        b_indexer = (wl.q_pos0 + wl.n_q) * key_bytes + keys * 4
    # top-k alone: every score read once, the index rows written
    b_topk = keys * 4 + wl.n_q * wl.topk * 4
    # sparse MLA + split merge: selected latent rows, q, idx in; out, lse out
    b_mla = b_lat + wl.n_q * (wl.H * wl.W * 2 + wl.topk * 4 + wl.H * wl.R * 4 + wl.H * 4)
    # cache append: each new row read once and written once (key + latent)
    b_append = 2 * wl.n_q * (wl.D_I * 2 + wl.W * 2)
    return {"bytes": b_keys + b_lat + b_small, "bytes_keys": b_keys, "bytes_latent": b_lat,
            "bytes_append": b_append,
            "flops": flops_idx + flops_mla, "flops_indexer": flops_idx, "flops_mla": flops_mla,
            "bytes_indexer": b_indexer, "bytes_topk": b_topk, "bytes_mla": b_mla,
            "keys": keys, "selected": sel}


# ---------------------------------------------------------------------------
# clocks (NVML, read only)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self._nv = None
        self._period = period_s
        self._thr = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._ok:
            self._thr.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._ok:
            self._thr.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# replicas across ranks (weak scaling, no data-path collective)
# ---------------------------------------------------------------------------

def replica_workload(wl, rank: int):
    """The workload rank `rank` runs: the same shapes, its own seeded batch."""
    return wl if rank == 0 else di.replace(wl, seed=wl.seed + 1000 * rank)


def max_over_ranks(x: float, dist, device) -> float:
    """The largest of every rank's `x` (every rank must call this, in the same order)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rows_per_s(rows_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: the rows all ranks processed over the slowest rank's step."""
    return rows_per_rank * world / (ms_per_step * 1e-3)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

class Case:
    """Device-resident inputs, outputs and workspace of one workload."""

    def __init__(self, wl, torch, dsa, k8=False, l8=False):
        self.wl = wl
        self.k8 = k8 or l8      # the FP8 latent cache goes with FP8 index keys
        self.l8 = l8
        self.inp = di.make_inputs(wl)
        if l8:   # the latent rows as E4M3 bytes with one scale per token
            self.inp = di.with_fp8_latent(self.inp, seed=wl.seed)
        inp = self.inp
        k8 = self.k8
        dev = "cuda"

        def bf(x):
            return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(dev)

        self.t = {"q_idx": bf(inp["q_idx"]), "k_pages": bf(inp["k_pages"]), "q": bf(inp["q"]),
                  "latent_pages": bf(inp["latent_pages"]), "w": torch.from_numpy(inp["w"]).to(dev),
                  "block_table": torch.from_numpy(inp["block_table"]).to(dev),
                  "seq_lens": torch.from_numpy(inp["seq_lens"]).to(dev)}
        if k8:   # the index keys as E4M3 bytes with one scale per token
            k8in = di.with_fp8_keys(inp, seed=wl.seed)
            self.t["k8_pages"] = torch.from_numpy(k8in["k8_pages"]).to(dev)
            self.t["k_scale"] = torch.from_numpy(k8in["k_scale"]).to(dev)
            del self.t["k_pages"]
        if l8:
            self.t["latent8_pages"] = torch.from_numpy(inp["latent8_pages"]).to(dev)
            self.t["latent_scale"] = torch.from_numpy(inp["latent_scale"]).to(dev)
            del self.t["latent_pages"]
        self.cache = dsa.PagedCache(self.t["seq_lens"], self.t["block_table"],
                                    num_pages=int(inp["k_pages"].shape[0]),
                                    max_seq_len=int(inp["seq_lens"].max()))
        self.dims = dsa.Dims(n_q=wl.n_q, H_I=wl.H_I, D_I=wl.D_I, topk=wl.topk, H=wl.H, R=wl.R,
                             P=wl.P, causal=int(wl.mode == "prefill"), q_pos0=wl.q_pos0,
                             scale=wl.scale)
        self.idx = torch.empty((wl.n_q, wl.topk), dtype=torch.int32, device=dev)
        self.out = torch.empty((wl.n_q, wl.H, wl.R), dtype=torch.float32, device=dev)
        self.lse = torch.empty((wl.n_q, wl.H), dtype=torch.float32, device=dev)
        self.ws = dsa.workspace(dsa.OP_ATTENTION_FORWARD_FP8 if l8 else
                                dsa.OP_ATTENTION_FORWARD_K8 if k8 else dsa.OP_ATTENTION_FORWARD,
                                self.dims, self.cache)
        ld = max(4, (max(row_lengths(wl)) + 3) // 4 * 4)
        self.scores = torch.empty((wl.n_q, ld), dtype=torch.float32, device=dev)
        # the current tokens' own rows, to time the cache append without
        # changing the caches (appending them again is idempotent)
        lens = np.asarray(row_lengths(wl), dtype=np.int64)
        seqs = np.zeros_like(lens) if wl.mode == "prefill" else np.arange(wl.n_q)
        pos = lens - 1
        phys = inp["block_table"][seqs, pos // 64].astype(np.int64) * 64 + pos % 64
        self.k_new = bf(inp["k_pages"].reshape(-1, wl.D_I)[phys])
        self.l_new = bf(inp["latent_pages"].reshape(-1, wl.W)[phys])
        # the absorption GEMMs around the step (GLM-5 head dims: q_nope 128, v 128)
        g = torch.Generator(device="cpu").manual_seed(wl.seed + 77)
        self.d_nope, self.d_v = 128, 128
        H, R, P = wl.H, wl.R, wl.P
        self.q_nope = torch.randn((wl.n_q, H, self.d_nope), generator=g).to(torch.bfloat16).to(dev)
        self.q_rope = torch.randn((wl.n_q, H, P), generator=g).to(torch.bfloat16).to(dev)
        self.w_uk = (torch.randn((H, self.d_nope, R), generator=g) / self.d_nope ** 0.5).to(
            torch.bfloat16).to(dev)
        self.w_uv = (torch.randn((H, R, self.d_v), generator=g) / R ** 0.5).to(torch.bfloat16).to(dev)
        self.q_abs = torch.empty((wl.n_q, H, R + P), dtype=torch.bfloat16, device=dev)
        self.v_out = torch.empty((wl.n_q, H, self.d_v), dtype=torch.float32, device=dev)
        self.sws = dsa.status_workspace()
        self.dsa = dsa
        self.torch = torch

    def step(self):
        t = self.t
        if self.l8:
            self.dsa.dsa_attention_forward_fp8(t["q_idx"], t["w"], t["k8_pages"], t["k_scale"],
                                               t["q"], t["latent8_pages"], t["latent_scale"],
                                               self.cache, self.dims, self.idx, self.out,
                                               self.lse, self.ws)
        elif self.k8:
            self.dsa.dsa_attention_forward_k8(t["q_idx"], t["w"], t["k8_pages"], t["k_scale"],
                                              t["q"], t["latent_pages"], self.cache, self.dims,
                                              self.idx, self.out, self.lse, self.ws)
        else:
            self.dsa.dsa_attention_forward(t["q_idx"], t["w"], t["k_pages"], t["q"],
                                           t["latent_pages"], self.cache, self.dims, self.idx,
                                           self.out, self.lse, self.ws)

    def indexer(self):
        t = self.t
        if self.k8:
            self.dsa.dsa_indexer_scores_k8(t["q_idx"], t["w"], t["k8_pages"], t["k_scale"],
                                           self.cache, self.dims, self.scores, self.ws)
        else:
            self.dsa.dsa_indexer_scores(t["q_idx"], t["w"], t["k_pages"], self.cache, self.dims,
                                        self.scores, self.ws)

    def append(self):
        t = self.t
        self.dsa.dsa_cache_append(self.k_new, self.l_new, t["k_pages"], t["latent_pages"],
                                  self.cache, self.dims, self.ws)

    def absorb(self):
        self.dsa.dsa_absorb_query(self.q_nope, self.q_rope, self.w_uk, self.q_abs, self.sws)

    def project(self):
        self.dsa.dsa_project_values(self.out, self.w_uv, self.v_out, self.sws)

    def absorb_bytes_flops(self):
        wl, n, H = self.wl, self.wl.n_q, self.wl.H
        a_bytes = H * self.d_nope * wl.R * 2 + n * H * (self.d_nope + wl.P + wl.R + wl.P) * 2
        p_bytes = H * wl.R * self.d_v * 2 + n * H * (wl.R + self.d_v) * 4
        return (a_bytes, 2 * n * H * self.d_nope * wl.R, p_bytes, 2 * n * H * wl.R * self.d_v)

    def topk(self):
        # the scores of the last indexer() call; decode rows end at their
        # sequence length, prefill rows at q_pos0 + t
        if self.wl.mode == "prefill":
            self.dsa.dsa_topk(self.scores, None, self.wl.q_pos0, self.wl.topk, self.idx, self.ws)
        else:
            self.dsa.dsa_topk(self.scores, self.t["seq_lens"], 0, self.wl.topk, self.idx,
                              self.ws)

    def mla(self):
        t = self.t
        if self.l8:
            fn = (self.dsa.dsa_sparse_mla_prefill_l8 if self.wl.mode == "prefill"
                  else self.dsa.dsa_sparse_mla_decode_l8)
            fn(t["q"], t["latent8_pages"], t["latent_scale"], self.cache, self.idx, self.dims,
               self.out, self.lse, self.ws)
            return
        fn = (self.dsa.dsa_sparse_mla_prefill if self.wl.mode == "prefill"
              else self.dsa.dsa_sparse_mla_decode)
        fn(t["q"], t["latent_pages"], self.cache, self.idx, self.dims, self.out, self.lse,
           self.ws)

    def launches_per_step(self):
        # the library's own launch plan for these shapes on this device
        op = (self.dsa.OP_ATTENTION_FORWARD_FP8 if self.l8 else
              self.dsa.OP_ATTENTION_FORWARD_K8 if self.k8 else self.dsa.OP_ATTENTION_FORWARD)
        n = self.dsa.forward_launches(op, self.dims, self.cache)
        if n <= 0:
            raise RuntimeError(f"no launch plan for {self.wl.name}")
        return n


def timed_events(torch, fn, steps, warmup, flush_buf):
    """Mean ms of fn over `steps` runs, each preceded (untimed) by an L2 flush:
    a read of a buffer four times the L2, which leaves no dirty lines behind."""
    for _ in range(warmup):
        flush_buf.sum()
        fn()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        flush_buf.sum()
        starts[i].record()
        fn()
        ends[i].record()
    torch.cuda.synchronize()
    times = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    return sum(times) / len(times), times


def timed_hot(torch, fn, steps, warmup):
    """Mean ms of fn over `steps` back-to-back runs (L2 left warm)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for _ in range(steps):
        fn()
    ev1.record()
    torch.cuda.synchronize()
    return ev0.elapsed_time(ev1) / steps


def measure(case, torch, steps, warmup, flush_buf, peaks, extras=True):
    wl = case.wl
    alg = algorithmic(wl, case.k8, case.l8)
    ms, _ = timed_events(torch, case.step, steps, warmup, flush_buf)
    ms_hot = timed_hot(torch, case.step, steps, warmup)
    st, info = case.dsa.workspace_check(case.ws)
    if st != 0:
        raise RuntimeError(f"device status {st} ({info:#x}) on {wl.name}")
    # each stage alone through its own entry point, L2 flushed before each
    ms_idx, _ = timed_events(torch, case.indexer, steps, warmup, flush_buf)
    ms_topk, _ = timed_events(torch, case.topk, steps, warmup, flush_buf)
    ms_mla, _ = timed_events(torch, case.mla, steps, warmup, flush_buf)
    st, info = case.dsa.workspace_check(case.ws)
    if st != 0:
        raise RuntimeError(f"device status {st} ({info:#x}) in the stage timings of {wl.name}")
    s = ms * 1e-3
    res = {
        "workload": wl.name, "mode": wl.mode, "index_keys": "e4m3+scale" if case.k8 else "bf16",
        "latent_rows": "e4m3+scale" if case.l8 else "bf16",
        "us_per_step": ms * 1e3,
        "tokens_per_s": wl.n_q / s,
        "alg_bytes": alg["bytes"], "alg_gbs": alg["bytes"] / s / 1e9,
        "frac_of_8tbs": alg["bytes"] / s / 1e9 / NOMINAL_HBM_GBS,
        "frac_of_measured_hbm": alg["bytes"] / s / 1e9 / peaks["hbm_gbs"],
        "hot_us_per_step": ms_hot * 1e3,
        "hot_tokens_per_s": wl.n_q / (ms_hot * 1e-3),
        "tflops": alg["flops"] / s / 1e12,
        "frac_of_bf16_peak": alg["flops"] / s / 1e12 / peaks["bf16_tflops"],
        "indexer_us": ms_idx * 1e3,
        "indexer_alg_bytes": alg["bytes_indexer"],
        "indexer_gbs": alg["bytes_indexer"] / (ms_idx * 1e-3) / 1e9,
        "indexer_frac_of_measured_hbm": alg["bytes_indexer"] / (ms_idx * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "launches_per_step": case.launches_per_step(),
        "stage_us": {"indexer": ms_idx * 1e3, "topk": ms_topk * 1e3, "mla": ms_mla * 1e3},
        "stage_alg_bytes": {"indexer": alg["bytes_indexer"], "topk": alg["bytes_topk"],
                            "mla": alg["bytes_mla"]},
    }
    if not extras:
        return res
    # the cache append in front of the step and the absorption GEMMs around it
    # (separate entry points, not in the step)
    ms_app, _ = timed_events(torch, case.append, steps, warmup, flush_buf)
    ms_abs, _ = timed_events(torch, case.absorb, steps, warmup, flush_buf)
    ms_prj, _ = timed_events(torch, case.project, steps, warmup, flush_buf)
    st, info = case.dsa.workspace_check(case.sws)
    if st != 0:
        raise RuntimeError(f"device status {st} ({info:#x}) in the absorption GEMMs of {wl.name}")
    ab, af, pb, pf = case.absorb_bytes_flops()
    res.update({
        "append_us": ms_app * 1e3,
        "append_alg_bytes": alg["bytes_append"],
        "append_gbs": alg["bytes_append"] / (ms_app * 1e-3) / 1e9,
        "absorb_query": {"us": ms_abs * 1e3, "alg_bytes": ab, "gbs": ab / (ms_abs * 1e-3) / 1e9,
                         "tflops": af / (ms_abs * 1e-3) / 1e12},
        "project_values": {"us": ms_prj * 1e3, "alg_bytes": pb, "gbs": pb / (ms_prj * 1e-3) / 1e9,
                           "tflops": pf / (ms_prj * 1e-3) / 1e12},
    })
    return res


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of
# each stage's kernels from one ncu capture of that kernel on that workload,
# with a digest of the sources the capture was taken on: the bench reports
# the figure only while those sources are unchanged.
TRAFFIC_SOURCES = {"indexer": ["indexer.cu"], "topk": ["topk.cu"], "mla": ["mla.cu"]}
TRAFFIC_COMMON = ["dsa_common.cuh", "dsa_internal.h"]
TRAFFIC = {
    # (stage, workload): (bytes per launch, digest of the stage's sources); the
    # median of 19 launches of one capture per workload
    ("indexer", "glm5_decode_b32_ragged"): (279734528, "fc474a6e2ffc96b0"),
    ("indexer", "glm5_decode_8k"): (2168576, "fc474a6e2ffc96b0"),
    ("indexer", "glm5_decode_4x128k"): (135001344, "fc474a6e2ffc96b0"),
    ("indexer", "glm5_prefill_2300"): (19788288, "fc474a6e2ffc96b0"),
    # topk_creg_kernel (32 rows, 4 x 131,072) and topk_small_kernel (8,192 keys, prefill rows)
    ("topk", "glm5_decode_b32_ragged"): (4351488, "86581b1144701485"),
    ("topk", "glm5_decode_8k"): (52224, "86581b1144701485"),
    ("topk", "glm5_decode_4x128k"): (2122240, "86581b1144701485"),
    ("topk", "glm5_prefill_2300"): (2234624, "86581b1144701485"),
    # mla_kernel + combine_kernel (the merge reads the split partials)
    ("mla", "glm5_decode_8k"): (2508800 + 4231936, "5514fc61eba92590"),
    ("mla", "glm5_decode_4x128k"): (9864704 + 16864256, "5514fc61eba92590"),
    # mla_pipe_kernel (rows merged inside clusters; prefill rows unsplit)
    ("mla", "glm5_decode_b32_ragged"): (78396672, "5514fc61eba92590"),
    ("mla", "glm5_prefill_2300"): (425517312, "5514fc61eba92590"),
}


def source_digest(stage):
    import hashlib
    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES[stage] + TRAFFIC_COMMON:
        with open(os.path.join(ROOT, "sparse_attention_scores_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_of(stage, workload):
    t = TRAFFIC.get((stage, workload))
    if t is None or t[1] != source_digest(stage):
        return None
    return t[0]


STAGE_KERNELS = {"indexer": "indexer_kernel (tcgen05 + TMA)",
                 "topk": "topk_small_kernel / topk_creg_kernel (radix select, keys in registers)",
                 "mla": "mla_kernel + combine_kernel (tcgen05, cp.async gather, split merge)",
                 "mla_pipe": "mla_pipe_kernel (gather warps, one tcgen05 issuer, softmax warps; "
                             "splits merged in clusters)"}


def mla_kernel_of(wl, sms=148, l8=False):
    """The sparse MLA kernel the library picks for either latent format: the
    pipelined one when the batch's 64-key blocks fill at least two waves of
    SMs, else the per-chunk one."""
    halves = wl.n_q * ((wl.topk + 63) // 64)
    return "mla_pipe" if halves >= 2 * sms else "mla"


def roofline_of(res, wl, peaks, k8=False, l8=False):
    """Roofline of the stage that takes the longest alone: algorithmic bytes
    (or flops, for the tensor-bound prefill MLA) over its event time.  FP8
    variants (k8) report no recorded traffic: it was captured on bf16 caches."""
    stage = max(res["stage_us"], key=res["stage_us"].get)
    us = res["stage_us"][stage]
    label = STAGE_KERNELS[mla_kernel_of(wl, l8=l8)] if stage == "mla" else STAGE_KERNELS[stage]
    if wl.mode == "prefill" and stage == "mla":
        alg = algorithmic(wl)
        achieved = alg["flops_mla"] / (us * 1e-6) / 1e12
        return {"kernel": label, "stage": stage, "bound": "tensor",
                "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"],
                "traffic": None if k8 else traffic_of(stage, wl.name),
                "peak_source": peaks["source"], "alg_flops_per_launch": alg["flops_mla"],
                "launch_us": us}
    b = res["stage_alg_bytes"][stage]
    achieved = b / (us * 1e-6) / 1e9
    return {"kernel": label, "stage": stage, "bound": "hbm",
            "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"],
            "traffic": None if k8 else traffic_of(stage, wl.name),
            "peak_source": peaks["source"], "alg_bytes_per_launch": b, "launch_us": us}


def measure_e2e(case, torch, steps, warmup, flush_buf):
    """Same metric through the C ABI's host-buffer entry point
    (dsa_attention_forward_host): every step copies its inputs in from pinned
    host memory and its results back, inside the timed region; the paged
    caches stay resident in HBM, and L2 is flushed before every step (outside
    the timed region) as for the device-timed step."""
    dsa, t = case.dsa, case.t
    names_in = ["q_idx", "w", "q", "seq_lens", "block_table"]
    host_in = {k: t[k].cpu().pin_memory() for k in names_in}
    host_out = {"idx": torch.empty_like(case.idx, device="cpu").pin_memory(),
                "out": torch.empty_like(case.out, device="cpu").pin_memory(),
                "lse": torch.empty_like(case.lse, device="cpu").pin_memory()}
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = sum(v.numel() * v.element_size() for v in host_out.values())
    cache_h = dsa.PagedCache(host_in["seq_lens"], host_in["block_table"],
                             num_pages=case.cache.num_pages, max_seq_len=case.cache.max_seq_len)
    hws = dsa.workspace(dsa.OP_ATTENTION_FORWARD_HOST, case.dims, cache_h)

    def one():
        dsa.dsa_attention_forward_host(host_in["q_idx"], host_in["w"], t["k_pages"], host_in["q"],
                                       t["latent_pages"], cache_h, case.dims, host_out["idx"],
                                       host_out["out"], host_out["lse"], hws)

    ms, _ = timed_events(torch, one, steps, warmup, flush_buf)
    st, info = dsa.workspace_check(hws)
    if st != 0:
        raise RuntimeError(f"device status {st} ({info:#x}) in the host-buffer step")
    return {"value": case.wl.n_q / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "api": "dsa_attention_forward_host", "workload": case.wl.name,
            "l2": "flushed (512 MB read) before every step, outside the timed region"}


def measure_cp(wl, ranks, torch, dsa, steps, warmup, flush_buf):
    """Context-parallel decode of `wl` split `ranks` ways, emulated on this GPU:
    each step of rank 0 (its local scores/top-k/candidates, the global select,
    its attention, the merge) timed with events; the two all-gathers between
    them cannot be timed on one GPU and are reported as bytes."""
    from sparse_attention_scores_b200.context_parallel import RankShard, cuda_ops
    inp = di.make_inputs(wl)
    dims = dsa.Dims(n_q=wl.n_q, H_I=wl.H_I, D_I=wl.D_I, topk=wl.topk, H=wl.H, R=wl.R, P=wl.P,
                    causal=0, q_pos0=0, scale=wl.scale)
    ops = cuda_ops(dims)

    def bf(x):
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()

    shards = []
    for r in range(ranks):
        lo = np.array([di.shard_bounds(n, ranks)[r] for n in wl.seq_lens])
        hi = np.array([di.shard_bounds(n, ranks)[r + 1] for n in wl.seq_lens])
        sh = di.shard_inputs(inp, lo, hi)
        t = {"q_idx": bf(sh["q_idx"]), "w": torch.from_numpy(sh["w"]).cuda(),
             "k_pages": bf(sh["k_pages"]), "q": bf(sh["q"]),
             "latent_pages": bf(sh["latent_pages"])}
        seq_lens = torch.from_numpy(sh["seq_lens"]).cuda()
        t["cache"] = dsa.PagedCache(seq_lens, torch.from_numpy(sh["block_table"]).cuda(),
                                    num_pages=int(sh["k_pages"].shape[0]),
                                    max_seq_len=int(sh["seq_lens"].max()))
        shards.append(RankShard(offsets=torch.from_numpy(sh["offsets"]).cuda(), lens=seq_lens,
                                local=t))
    cand = [ops.candidates(*ops.local_topk(s, wl.topk), s.offsets) for s in shards]
    all_s, all_i = torch.stack([c[0] for c in cand]), torch.stack([c[1] for c in cand])
    gidx, own = ops.select(all_s, all_i, shards[0].offsets, shards[0].lens)
    part = [ops.attend(s, ops.select(all_s, all_i, s.offsets, s.lens)[1]) for s in shards]
    outs, lses = torch.stack([p[0] for p in part]), torch.stack([p[1] for p in part])
    torch.cuda.synchronize()
    s0 = shards[0]
    t_local, _ = timed_events(torch, lambda: ops.candidates(*ops.local_topk(s0, wl.topk), s0.offsets),
                              steps, warmup, flush_buf)
    t_sel, _ = timed_events(torch, lambda: ops.select(all_s, all_i, s0.offsets, s0.lens), steps,
                            warmup, flush_buf)
    t_att, _ = timed_events(torch, lambda: ops.attend(s0, own), steps, warmup, flush_buf)
    t_mrg, _ = timed_events(torch, lambda: ops.merge(outs, lses), steps, warmup, flush_buf)
    cand_bytes = ranks * wl.n_q * wl.topk * 8
    part_bytes = ranks * wl.n_q * wl.H * (wl.R + 1) * 4
    return {"workload": wl.name, "ranks": ranks, "emulated_on_one_gpu": True,
            "keys_per_rank_per_row": int(max(wl.seq_lens)) // ranks,
            "rank_local_us": t_local * 1e3, "select_us": t_sel * 1e3,
            "attend_us": t_att * 1e3, "merge_us": t_mrg * 1e3,
            "per_rank_compute_us": (t_local + t_sel + t_att + t_mrg) * 1e3,
            "all_gather_bytes": {"candidates": cand_bytes, "partials": part_bytes},
            "all_gather_us_at_770_gbs_modelled": (cand_bytes + part_bytes) / 770e9 * 1e6}


def oracle_rows_per_s(wl, budget_s: float):
    """Time the float64 oracle on whole query rows of `wl` for ~budget_s."""
    from oracle import dsa_oracle as orc
    inp = di.make_inputs(wl)
    fn = orc.dsa_prefill if wl.mode == "prefill" else orc.dsa_decode
    rows = list(range(wl.n_q))
    if wl.mode == "prefill":   # rows past the top-k size exercise the selection
        rows = rows[::-1]
    done, t0 = 0, time.perf_counter()
    while True:
        fn(inp, [rows[done % len(rows)]])
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return done / el, done, el


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(wl, budget_s=10.0):
    """The oracle as it stands on this host: all BLAS threads, then one."""
    rate, n, el = oracle_rows_per_s(wl, budget_s)
    res = {"value": rate, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
           "sample": f"{n} query rows of {wl.name} through the float64 oracle in {el:.1f} s "
                     f"(host: {os.cpu_count()} logical cores)",
           "cpu_model": cpu_model(), "logical_cores": os.cpu_count()}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            r1, n1, el1 = oracle_rows_per_s(wl, budget_s / 2)
        res["one_thread"] = {"value": r1, "unit": "tokens/s", "cores": 1,
                             "sample": f"{n1} query rows in {el1:.1f} s with one BLAS thread"}
    except Exception as e:   # threadpoolctl missing: report why
        res["one_thread"] = {"unavailable": str(e)}
    return res


def run_ours(args):
    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    import sparse_attention_scores_b200 as dsa
    dsa.lib()
    peaks = load_peaks()
    flush_buf = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")

    wl = di.CONFIGS[args.config]
    # weak scaling: every rank runs its own replica of the workload (its own batch)
    case = Case(replica_workload(wl, rank), torch, dsa, k8=args.fp8_keys)
    case.step()
    torch.cuda.synchronize()
    pg = dist if world > 1 else None

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        # the append and absorption extras use the bf16 page pools
        head = measure(case, torch, args.steps, args.warmup, flush_buf, peaks,
                       extras=not args.fp8_keys)
        # keep the sampler on the same work long enough for NVML to see it
        t_end = time.perf_counter() + (0.0 if args.profile else 1.0)
        while time.perf_counter() < t_end:
            case.step()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(head["us_per_step"] / 1e3, pg, "cuda")
    # the host-buffer entry point serves bf16 index keys
    e2e = None if (args.profile or args.fp8_keys) else measure_e2e(case, torch, args.steps,
                                                                    args.warmup, flush_buf)
    if e2e is not None:
        e2e["ms_per_step"] = max_over_ranks(e2e["ms_per_step"], pg, "cuda")
        e2e["value"] = job_rows_per_s(wl.n_q, world, e2e["ms_per_step"])

    per_config = {}
    if not args.no_extra:
        for name in EXTRA:
            c = Case(replica_workload(di.CONFIGS[name], rank), torch, dsa)
            c.step()
            torch.cuda.synchronize()
            r = measure(c, torch, args.steps, args.warmup, flush_buf, peaks)
            r["us_per_step"] = max_over_ranks(r["us_per_step"], pg, "cuda")
            r["roofline"] = roofline_of(r, c.wl, peaks)
            # the same workload through the host-buffer entry point
            e = measure_e2e(c, torch, args.steps, args.warmup, flush_buf)
            e["ms_per_step"] = max_over_ranks(e["ms_per_step"], pg, "cuda")
            e["value"] = job_rows_per_s(c.wl.n_q, world, e["ms_per_step"])
            r["e2e"] = e
            per_config[name] = r
            del c
            torch.cuda.empty_cache()
        # context-parallel decode of the 4 x 131,072 rows over 8 ranks, emulated here
        per_config["glm5_decode_4x128k/context_parallel_8"] = measure_cp(
            di.CONFIGS["glm5_decode_4x128k"], 8, torch, dsa, args.steps, args.warmup, flush_buf)
        torch.cuda.empty_cache()
        for name in EXTRA_K8:
            c = Case(replica_workload(di.CONFIGS[name], rank), torch, dsa, k8=True)
            c.step()
            torch.cuda.synchronize()
            r = measure(c, torch, args.steps, args.warmup, flush_buf, peaks, extras=False)
            r["us_per_step"] = max_over_ranks(r["us_per_step"], pg, "cuda")
            r["roofline"] = roofline_of(r, c.wl, peaks, k8=True)
            per_config[name + "+fp8_keys"] = r
            del c
            torch.cuda.empty_cache()
        for name in EXTRA_FP8:
            c = Case(replica_workload(di.CONFIGS[name], rank), torch, dsa, l8=True)
            c.step()
            torch.cuda.synchronize()
            r = measure(c, torch, args.steps, args.warmup, flush_buf, peaks, extras=False)
            r["us_per_step"] = max_over_ranks(r["us_per_step"], pg, "cuda")
            r["roofline"] = roofline_of(r, c.wl, peaks, k8=True, l8=True)
            per_config[name + "+fp8_cache"] = r
            del c
            torch.cuda.empty_cache()

    if rank == 0:
        alg = algorithmic(wl)
        idx_s = head["indexer_us"] * 1e-6
        line = {
            "metric": "DSA attention decode tokens/s (one layer's DSA step: indexer, exact "
                      "top-2048, sparse absorbed MLA)",
            "value": job_rows_per_s(wl.n_q, world, ms),
            "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "us_per_step": ms * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 inputs, fp32 accumulate/outputs",
            "data": "synthetic (seeded GLM-5-shaped inputs; integer indexer q/k)",
            "config": {"workload": wl.name, "description": wl.description,
                       "global_batch": wl.n_q * world, "seq_len": max(wl.seq_lens),
                       "parallelism": f"replicas x{world}",
                       "l2": "flushed (512 MB read) before every timed step",
                       "alg_bytes_per_step": alg["bytes"],
                       "achieved_gbs": alg["bytes"] / (ms * 1e-3) / 1e9,
                       "frac_of_measured_hbm": alg["bytes"] / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                       "hbm_peak_gbs": peaks["hbm_gbs"], "hbm_peak_source": peaks["source"],
                       "frac_of_8tbs": alg["bytes"] / (ms * 1e-3) / 1e9 / NOMINAL_HBM_GBS},
            "hot": {"us_per_step": head["hot_us_per_step"],
                    "tokens_per_s": head["hot_tokens_per_s"],
                    "l2": "warm: steps back to back, no flush"},
            "roofline": roofline_of(head, wl, peaks, k8=args.fp8_keys),
            "stage_us": head["stage_us"],
            "e2e": e2e,
            "gpu_launches": head["launches_per_step"] * args.steps,
            "clocks": clk.summary(),
            "per_config": per_config,
        }
        if args.cpu_baseline_s > 0 and world == 1 and not args.profile:
            line["cpu_baseline"] = cpu_baseline(wl, args.cpu_baseline_s)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = di.CONFIGS[args.config]
    for _ in range(args.warmup):
        oracle_rows_per_s(wl, 0.0)
    times = []
    for _ in range(args.steps):
        rate, n, el = oracle_rows_per_s(wl, 0.0)   # one step = one whole query row
        times.append(el / n)
    s = sum(times) / len(times)
    value = 1.0 / s   # query rows (decode tokens) per second
    line = {
        "impl": "reference",
        "metric": "DSA attention decode tokens/s (one layer's DSA step: indexer, exact "
                  "top-2048, sparse absorbed MLA)",
        "value": value, "unit": "tokens/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded GLM-5-shaped inputs)",
        "config": {"workload": wl.name, "description": wl.description},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(),
                         "kind": "oracle",
                         "sample": f"{args.steps} steps, each one whole query row of {wl.name}"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=HEADLINE, choices=list(di.CONFIGS))
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--fp8-keys", action="store_true",
                    help="run the workload with FP8 (E4M3) index keys (for profiling; no e2e)")
    ap.add_argument("--cpu-baseline-s", type=float, default=10.0)
    ap.add_argument("--profile", action="store_true",
                    help="for profiler runs: no clock soak, no e2e leg, no CPU baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
