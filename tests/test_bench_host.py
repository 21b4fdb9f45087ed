"""Host logic of the benchmark on CPU: the must-move byte counts against their
closed forms, the gate on recorded DRAM traffic, the roofline's choice of
stage, and the JSON line of the reference (oracle) arm."""

import json
import subprocess
import sys

import pytest

import bench
import dsa_inputs as di


def test_algorithmic_bytes_of_the_8k_decode():
    # batch 1, 8,192 keys of 32 x 128 bf16 (256 B), 2,048 selected 576-wide
    # bf16 latent rows (1,152 B), plus q (64 x 576 bf16), q_idx (32 x 128
    # bf16), w (32 fp32), out (64 x 512 fp32) and lse (64 fp32)
    a = bench.algorithmic(di.CONFIGS["glm5_decode_8k"])
    assert a["bytes_keys"] == 8192 * 256
    assert a["bytes_latent"] == 2048 * 1152
    assert a["bytes"] == 8192 * 256 + 2048 * 1152 + 64 * 576 * 2 + 32 * 128 * 2 + 32 * 4 \
        + 64 * 512 * 4 + 64 * 4 == 4_669_824
    assert a["flops_mla"] == 2048 * 64 * 2 * (576 + 512)


def test_algorithmic_bytes_of_the_long_context_and_fp8_keys():
    wl = di.CONFIGS["glm5_decode_4x128k"]
    a, a8 = bench.algorithmic(wl), bench.algorithmic(wl, k8=True)
    assert a["bytes_keys"] == 4 * 131072 * 256
    # E4M3 keys: one byte per element plus a 4-byte scale per token
    assert a8["bytes_keys"] == 4 * 131072 * (128 + 4)
    assert a["bytes_latent"] == a8["bytes_latent"] == 4 * 2048 * 1152
    # the indexer kernel alone also writes one fp32 score per key
    assert a["bytes_indexer"] == 4 * 131072 * (256 + 4) + 4 * 32 * (128 * 2 + 4)


def test_prefill_reads_the_cache_once():
    wl = di.CONFIGS["glm5_prefill_2300"]
    a = bench.algorithmic(wl)
    assert a["bytes_keys"] == 2300 * 256 and a["bytes_latent"] == 2300 * 1152
    # every row t selects min(t + 1, 2048) keys
    assert a["selected"] == sum(min(t + 1, 2048) for t in range(2300))


def test_traffic_is_reported_only_for_the_captured_sources(monkeypatch):
    key = ("mla", "glm5_decode_8k")
    value, digest = bench.TRAFFIC[key]
    monkeypatch.setattr(bench, "source_digest", lambda stage: digest)
    assert bench.traffic_of(*key) == value
    monkeypatch.setattr(bench, "source_digest", lambda stage: "0" * 16)
    assert bench.traffic_of(*key) is None
    assert bench.traffic_of("mla", "tiny_decode") is None


def test_roofline_takes_the_longest_stage():
    wl = di.CONFIGS["glm5_decode_4x128k"]
    peaks = {"hbm_gbs": 6443.2, "bf16_tflops": 1671.8, "source": "measured"}
    alg = bench.algorithmic(wl)
    res = {"stage_us": {"indexer": 32.0, "topk": 18.0, "mla": 30.0},
           "stage_alg_bytes": {"indexer": alg["bytes_indexer"], "topk": alg["bytes_topk"],
                               "mla": alg["bytes_mla"]}}
    r = bench.roofline_of(res, wl, peaks)
    assert r["stage"] == "indexer" and r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(alg["bytes_indexer"] / 32e-6 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6443.2)
    # the prefill MLA stage is rated in flops against the bf16 peak
    wp = di.CONFIGS["glm5_prefill_2300"]
    rp = bench.roofline_of({"stage_us": {"indexer": 100.0, "topk": 30.0, "mla": 2000.0},
                            "stage_alg_bytes": {"indexer": 1, "topk": 1, "mla": 1}}, wp, peaks)
    assert rp["bound"] == "tensor" and rp["unit"] == "TFLOP/s"
    assert rp["achieved"] == pytest.approx(bench.algorithmic(wp)["flops_mla"] / 2000e-6 / 1e12)


def test_reference_arm_prints_one_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config",
                          "tiny_decode", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, check=True).stdout
    lines = [l for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["config"]["workload"] == "tiny_decode" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
