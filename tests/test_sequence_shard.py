"""Host side of KV-sequence sharding (CPU): the partition, the merge it
relies on (with the oracle), and the exchange of states with gloo ranks.

The partition must cover every KV position of the request exactly once, give
every dense chunk at least T keys (the library call's minimum), keep the tree
block on the last rank, and stay within the plan's bound. The merge of the
ranks' partial states, taken by the oracle, must equal the oracle's one-shot
rows: that pins the decomposition itself, independently of the CUDA path.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from mla_speculative_verify_absorb_b200.sequence_shard import gather_states, max_shard_keys, shard_ranges
from workloads import custom, generate

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("L,T,R", [(65536, 64, 8), (65536, 64, 1), (4096, 16, 3), (256, 4, 3), (100, 64, 4),
                                   (0, 5, 2), (63, 64, 2), (128, 64, 8), (1000, 7, 1000), (129, 64, 2)])
def test_shard_ranges_partition(L, T, R):
    ranges = shard_ranges(L, T, R)
    assert len(ranges) == R
    covered = np.zeros(L + T, dtype=np.int32)
    for r, (lo, hi) in enumerate(ranges):
        assert 0 <= lo <= hi <= L + T
        covered[lo:hi] += 1
        if r < R - 1 and hi > lo:
            assert hi <= L and hi - lo >= T                 # a dense chunk: prefix only, >= T keys
    assert np.all(covered == 1)                             # every position exactly once
    lo, hi = ranges[-1]
    assert hi == L + T and hi - lo >= T                     # the tree block sits on the last rank
    assert max(h - l for l, h in ranges) <= max_shard_keys(L, T, R)
    active = sum(1 for l, h in ranges if h > l)
    assert active == min(R, max(1, L // T))


def test_max_shard_keys_bounds_every_smaller_call():
    for R in (1, 2, 3, 8):
        bound = max_shard_keys(3000, 64, R)
        for L in range(0, 3001, 37):
            for T in (1, 2, 17, 63, 64):
                assert max(h - l for l, h in shard_ranges(L, T, R)) <= bound


@pytest.mark.parametrize("R", [1, 2, 3, 5])
def test_merge_of_shards_equals_one_shot_oracle(R):
    inp = generate(custom("shard_oracle", 81, 4, [700], [13], 2048))
    anc = oracle.ancestor_masks(inp.parents, inp.qo_indptr)
    T = 13
    rows = np.arange(T * 4, dtype=np.int64)
    ms, ls, os_ = [], [], []
    for lo, hi in shard_ranges(700, T, R):
        m, l, o = oracle.partial_rows(inp, anc, lo, hi, rows=rows)
        ms.append(m)
        ls.append(l)
        os_.append(o)
    out, lse = oracle.merge_states(np.stack(ms), np.stack(ls), np.stack(os_))
    ref, ref_lse, _ = oracle.verify_rows(inp, anc, rows=rows)
    assert np.abs(out - ref).max() <= 1e-12 and np.abs(lse - ref_lse).max() <= 1e-12


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        T, H, D = 3, 2, 8
        o_local = torch.full((T, H, D), float(rank + 1))
        lse_local = torch.full((T, H), -float(rank))
        o_all = torch.empty((world, T, H, D))
        lse_all = torch.empty((world, T, H))
        gather_states(o_local, lse_local, o_all, lse_all)
        q.put((rank, o_all[:, 0, 0, 0].tolist(), lse_all[:, -1, -1].tolist()))
    finally:
        dist.destroy_process_group()


def test_gather_states_gloo_two_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict((r, (o, l)) for r, o, l in (q.get(timeout=120) for _ in range(world)))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert got[r] == ([1.0, 2.0], [0.0, -1.0])          # rank-major on every rank
