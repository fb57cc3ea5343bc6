"""KV-sequence sharding on one GPU: the ranks' shards run one after another
(their kernels never wait on one another), their states are stacked as the
all-gather would stack them, and the library's stacked merge combines them.
The result must match the oracle within the fused path's tolerances."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import compare, product_anc
from mla_speculative_verify_absorb_b200.sequence_shard import ShardedVerify, shard_ranges
from workloads import WORKLOADS, custom, generate
from workloads import device as wdev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _emulate(inp, R):
    wl = inp.workload
    T = int(wl.tree_sizes[0])
    anc = product_anc(inp)
    d = wdev.to_device(inp, anc)
    sv = ShardedVerify(world=R, num_heads=wl.num_heads, max_tree=T, max_prefix=int(wl.prefixes[0]),
                       pool_slots=wl.pool_slots, sm_scale=wl.sm_scale)
    o_all, lse_all = sv.stacked(T)
    s = torch.cuda.current_stream().cuda_stream
    active = 0
    for r in range(R):
        if sv.local_state(r, d["q_latent"], d["q_rope"], d["kv_pool"], d["kv_indices"], d["tree_anc"],
                          o_all[r], lse_all[r], s):
            active += 1
        else:                                   # what an empty rank contributes to the exchange
            o_all[r].zero_()
            lse_all[r].fill_(float("-inf"))
    sv.merge(o_all, lse_all, d["out"], d["lse"], s)
    torch.cuda.synchronize()
    code, bits = sv.attn.status()
    assert code == 0, f"status {code} bits {bits:#x}"
    assert active == sum(1 for lo, hi in shard_ranges(int(wl.prefixes[0]), T, R) if hi > lo)
    return d


@pytest.mark.parametrize("name,R", [("tiny", 3), ("tp8", 2), ("tp8", 3), ("short_prefix", 4), ("tp8", 1)])
def test_sharded_matches_oracle(name, R):
    if name == "short_prefix":                  # L // T = 1: only the last rank has keys
        inp = generate(custom("shard_short", 82, 8, [100], [64], 1024))
    else:
        inp = generate(WORKLOADS[name])
    d = _emulate(inp, R)
    ref, ref_lse, _ = oracle.verify_rows(inp, oracle.ancestor_masks(inp.parents, inp.qo_indptr))
    out = d["out"].float().cpu().numpy().astype(np.float64).reshape(-1, 512)
    lse = d["lse"].cpu().numpy().astype(np.float64).reshape(-1)
    compare(out, ref, lse, ref_lse)


def test_sharded_long_eight_ranks_sampled():
    inp = generate(WORKLOADS["long"])
    d = _emulate(inp, 8)
    H = inp.q_latent.shape[1]
    rows = np.random.default_rng(83).choice(inp.q_latent.shape[0] * H, 96, replace=False).astype(np.int64)
    rows[:H] = np.arange(H)
    ref, ref_lse, _ = oracle.verify_rows(inp, oracle.ancestor_masks(inp.parents, inp.qo_indptr), rows=rows)
    out = d["out"].float().cpu().numpy().astype(np.float64).reshape(-1, 512)[rows]
    lse = d["lse"].cpu().numpy().astype(np.float64).reshape(-1)[rows]
    compare(out, ref, lse, ref_lse)
