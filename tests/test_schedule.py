"""CPU check of the work schedule the split and reduce kernels share.

The split kernel walks each CTA pair's unit range segment by segment and
writes one partial state per (row tile g, pair c) to slot g + c; the reduce
kernel recomputes, from a closed form, which pairs touched row tile g. This
test replays both sides for the workload shapes and random batches and
checks that they agree, that every unit is processed exactly once, and that
slots are unique and inside the plan's workspace.
"""
import numpy as np
import pytest

import mla_speculative_verify_absorb_b200 as va
from workloads import WORKLOADS

ROWS, KEYS = 128, 256


def _requests(T_list, N_list, H):
    out = []
    for T, N in zip(T_list, N_list):
        out.append(((T * H + ROWS - 1) // ROWS, (N + KEYS - 1) // KEYS))
    return out


def _split_side(reqs, G):
    """(g, c) pairs the split kernel's segment walk produces, per cluster."""
    U = sum(rt * kt for rt, kt in reqs)
    touched = {}
    seen_units = []
    for c in range(G):
        u, u_end = c * U // G, (c + 1) * U // G
        while u < u_end:
            acc, g = 0, 0
            for rt_n, kt_n in reqs:
                ub = rt_n * kt_n
                if u < acc + ub:
                    local = u - acc
                    rt, kt0 = local // kt_n, local % kt_n
                    n = min(kt_n - kt0, u_end - u)
                    touched.setdefault(g + rt, []).append(c)
                    seen_units.extend(range(u, u + n))
                    u += n
                    break
                acc += ub
                g += rt_n
    return U, touched, seen_units


def _reduce_side(reqs, G, U):
    """Clusters the reduce kernel merges for every row tile."""
    out, g, acc = {}, 0, 0
    for rt_n, kt_n in reqs:
        for rt in range(rt_n):
            ustart = acc + rt * kt_n
            lo = ((ustart + 1) * G - 1) // U
            hi = ((ustart + kt_n) * G - 1) // U
            out[g + rt] = [c for c in range(lo, hi + 1) if c * U // G != (c + 1) * U // G]
        g += rt_n
        acc += rt_n * kt_n
    return out


def _check(T_list, N_list, H, max_batch, max_tree, G):
    reqs = _requests(T_list, N_list, H)
    U, touched, seen = _split_side(reqs, G)
    assert sorted(seen) == list(range(U))
    assert _reduce_side(reqs, G, U) == touched
    row_tiles_per_req = (max_tree * H + ROWS - 1) // ROWS
    slots = [g + c for g, cs in touched.items() for c in cs]
    assert len(slots) == len(set(slots))
    assert max(slots) < G + max_batch * row_tiles_per_req


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_schedule_workloads(name):
    wl = WORKLOADS[name]
    params = va.VerifyAttnParams(max_batch=wl.batch, num_heads=wl.num_heads, max_tree=max(wl.tree_sizes),
                                 d_latent=512, d_rope=64, num_sms=148, max_kv_per_req=max(wl.kv_lens),
                                 max_total_kv=wl.total_kv, pool_slots=wl.pool_slots, sm_scale=wl.sm_scale)
    plan, _ = va.verify_attn_plan(params)
    _check(list(wl.tree_sizes), wl.kv_lens, wl.num_heads, wl.batch, max(wl.tree_sizes), plan.num_clusters)


def test_schedule_random_batches():
    rng = np.random.default_rng(3)
    for _ in range(300):
        B = int(rng.integers(1, 7))
        H = int(rng.choice([1, 3, 8, 16, 64, 100, 128]))
        T = [int(rng.integers(1, 65)) for _ in range(B)]
        N = [t + int(rng.integers(0, 3000)) for t in T]
        G = int(rng.integers(1, 80))
        _check(T, N, H, B, 64, G)
