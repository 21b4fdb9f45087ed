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


def test_shards_hold_the_sequence_keys():
    wl = di.small_decode([300, 65], H_I=2, D_I=16, topk=8, H=2, R=16, P=8, seed=5,
                         shuffle_pages=True)
    inp = di.make_inputs(wl)
    for ranks in (2, 3):
        rows_k = [[] for _ in wl.seq_lens]
        for r in range(ranks):
            lo = np.array([di.shard_bounds(n, ranks)[r] for n in wl.seq_lens])
            hi = np.array([di.shard_bounds(n, ranks)[r + 1] for n in wl.seq_lens])
            sh = di.shard_inputs(inp, lo, hi)
            assert np.array_equal(sh["offsets"], lo) and np.array_equal(sh["seq_lens"], hi - lo)
            for b in range(len(wl.seq_lens)):
                for p in range(int(hi[b] - lo[b])):
                    pg = sh["block_table"][b][p // 64]
                    rows_k[b].append(sh["k_pages"][pg, p % 64])
        for b, n in enumerate(wl.seq_lens):
            want = [inp["k_pages"][inp["block_table"][b][p // 64], p % 64] for p in range(n)]
            assert np.array_equal(np.stack(rows_k[b]), np.stack(want))
