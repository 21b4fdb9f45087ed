"""The seeded input generator: determinism, shapes, value ranges, paging."""

import numpy as np
import torch

import dsa_inputs as di


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, -3.0, 1e-40, 3.4e38], np.float32)])
    mine = di.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(mine, ref)


def test_inputs_deterministic_and_shaped():
    wl = di.small_decode([100, 257, 64], H_I=4, D_I=32, topk=16, H=4, R=32, P=16, seed=3)
    a = di.make_inputs(wl)
    b = di.make_inputs(wl)
    for k in ("q_idx", "w", "k_pages", "q", "latent_pages", "block_table", "seq_lens"):
        np.testing.assert_array_equal(a[k], b[k])
    assert a["q_idx"].shape == (3, 4, 32) and a["q_idx"].dtype == np.uint16
    assert a["k_pages"].shape == (2 + 5 + 1, 64, 32)
    assert a["latent_pages"].shape == (8, 64, 48)
    assert a["block_table"].shape == (3, 5)
    assert sorted(a["block_table"][a["block_table"] >= 0].tolist()) == list(range(8))
    vals = (a["q_idx"].astype(np.uint32) << 16).view(np.float32)
    assert set(np.unique(vals).tolist()) <= {-3.0, -2.0, -1.0, 0.0, 1.0, 2.0, 3.0}
    assert set(np.unique(a["w"]).tolist()) <= {0.0, 1.0, 2.0, 3.0}


def test_ragged_config_lengths():
    wl = di.CONFIGS["glm5_decode_b32_ragged"]
    assert len(wl.seq_lens) == 32
    assert min(wl.seq_lens) >= 2048 and max(wl.seq_lens) <= 65536
    assert wl.seq_lens == di.ragged_lengths(32, 2048, 65536, 1)
