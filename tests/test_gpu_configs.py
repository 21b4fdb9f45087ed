"""The five GLM-5-shaped workloads at full size, in the launch configuration
bench.py times, against the float64 oracle.

Decode workloads are checked on every row.  The 2,300-token prefill checks the
kept indices of every row and the attention outputs of sampled rows (the
oracle's MLA over all rows would take minutes).
"""

import numpy as np
import pytest
import torch

import dsa_inputs as di
from oracle import dsa_oracle as orc
from tests.dsa_testutil import assert_row_matches, run_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("name", ["tiny_decode", "glm5_decode_8k", "glm5_decode_b32_ragged",
                                  "glm5_decode_4x128k"])
def test_decode_config(name):
    wl = di.CONFIGS[name]
    inp = di.make_inputs(wl)
    idx, out, lse = run_forward(inp)
    ref = orc.dsa_decode(inp)
    worst = 0.0
    for r, res in ref.items():
        e, _ = assert_row_matches(r, res, idx, out, lse)
        worst = max(worst, e)
    print(f"{name}: {len(ref)} rows, indices exact, worst normalised out error {worst:.2e}")


def test_prefill_config():
    wl = di.CONFIGS["glm5_prefill_2300"]
    inp = di.make_inputs(wl)
    idx, out, lse = run_forward(inp)
    T = wl.n_q
    # indices of every row (rows below 2,048 keep everything)
    k_all = orc.bf16_to_f64(orc.gather_paged_rows(inp["k_pages"], inp["block_table"][0], range(T)))
    for t in range(T):
        if t + 1 <= wl.topk:
            want = np.full(wl.topk, -1, np.int64)
            want[:t + 1] = np.arange(t + 1)
        else:
            s = orc.indexer_scores(orc.bf16_to_f64(inp["q_idx"][t]), inp["w"][t], k_all[:t + 1])
            want = orc.topk_select(s, wl.topk)
        assert np.array_equal(idx[t].astype(np.int64), want), t
    rows = [0, 1, 63, 127, 128, 1000, 2046, 2047, 2048, 2049, 2100, 2200, 2298, 2299]
    ref = orc.dsa_prefill(inp, rows)
    worst = 0.0
    for r, res in ref.items():
        e, _ = assert_row_matches(r, res, idx, out, lse)
        worst = max(worst, e)
    print(f"prefill: indices exact on {T} rows, worst out error {worst:.2e} on {len(rows)} rows")
