"""Shards of one decode workload for context-parallel tests (the input
module's shard construction)."""

from __future__ import annotations

import numpy as np

import dsa_inputs as di

shard_bounds = di.shard_bounds


def make_shard(inp: dict, wl, lo: np.ndarray, hi: np.ndarray) -> dict:
    return di.shard_inputs(inp, lo, hi)
