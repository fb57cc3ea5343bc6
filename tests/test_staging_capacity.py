"""The plan's staging rows always hold a call's tile-padded KV.

The gather kernel writes each request's KV positions into its own run of
256-row key tiles (padding rows zeroed), and the split kernel loads tiles by
global key-tile index. verify_attn_plan sizes the staging area as
256 * (ceil(max_total_kv / 256) + max_batch) rows; this checks, for random
batches within the plan's maxima, that the padded tiles never exceed it, and
that requests' tile runs are disjoint and in order.
"""
import numpy as np
import pytest

import mla_speculative_verify_absorb_b200 as va

KEYS = 256


def _plan(max_batch, max_kv_per_req, max_total_kv):
    p = va.VerifyAttnParams(max_batch=max_batch, num_heads=64, max_tree=64, d_latent=512, d_rope=64, num_sms=148,
                            max_kv_per_req=max_kv_per_req, max_total_kv=max_total_kv, pool_slots=1 << 20,
                            sm_scale=192 ** -0.5)
    return va.verify_attn_plan(p)[0]


@pytest.mark.parametrize("seed", range(20))
def test_padded_tiles_fit_staging(seed):
    rng = np.random.default_rng(seed)
    max_batch = int(rng.integers(1, 17))
    max_kv_per_req = int(rng.integers(64, 300_000))
    max_total_kv = int(rng.integers(max_kv_per_req, max_batch * max_kv_per_req + 1))
    plan = _plan(max_batch, max_kv_per_req, max_total_kv)
    assert plan.stage_rows % KEYS == 0
    capacity = plan.stage_rows // KEYS
    for _ in range(50):
        batch = int(rng.integers(1, max_batch + 1))
        # lengths within the per-request and total maxima, adversarially many padding tiles
        left = max_total_kv
        lens = []
        for b in range(batch):
            hi = min(max_kv_per_req, left - (batch - b - 1) * 64)
            n = int(rng.integers(64, max(65, hi + 1)))
            if rng.random() < 0.5:
                n = int(min(hi, (n // KEYS) * KEYS + 1))   # one key past a tile boundary
            n = max(64, min(n, hi))
            lens.append(n)
            left -= n
        tiles = [(n + KEYS - 1) // KEYS for n in lens]
        assert sum(tiles) <= capacity
        starts = np.cumsum([0] + tiles[:-1])
        for s0, t, n in zip(starts, tiles, lens):
            assert (s0 + t) * KEYS <= plan.stage_rows and n <= t * KEYS
