"""The long-context call captured in a CUDA graph with static workspaces.

verify_attn_run / verify_attn_reduce are captured once (plan sized for the
65k-prefix workload) and replayed; between replays the per-request lengths
and the tree change through the device buffers only (kv_indptr, kv_indices,
tree_anc), as a serving loop would do. Every replay is checked against the
oracle on sampled rows and on all visible counts (page "The Execution
Phase", section "Making the Kernel CUDA Graph Capture-Safe": static buffers,
no host sync, no allocation; replay must match the eager result).
"""
import numpy as np
import pytest
import torch

import mla_speculative_verify_absorb_b200 as va
import oracle
from gpu_common import closed_form_counts, compare, make_attention, product_anc, sample_rows
from workloads import WORKLOADS, generate, random_parents
from workloads import device as wdev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _check(inp, d):
    ref_anc = oracle.ancestor_masks(inp.parents, inp.qo_indptr)
    vis = d["visible_count"].cpu().numpy()
    assert np.array_equal(vis, closed_form_counts(inp, ref_anc))
    rows = sample_rows(inp, 12, seed=7)
    ref_out, ref_lse, _ = oracle.verify_rows(inp, ref_anc, rows=rows)
    out = d["out"].float().cpu().numpy().astype(np.float64).reshape(-1, 512)[rows]
    lse = d["lse"].cpu().numpy().astype(np.float64).reshape(-1)[rows]
    compare(out, ref_out, lse, ref_lse)


def _shrink(inp, new_prefix: int, seed: int):
    """Same request with a shorter prefix and a new tree (device-side change only)."""
    T = int(inp.qo_indptr[1])
    L = int(inp.kv_indptr[1]) - T
    inp.kv_indices = np.concatenate([inp.kv_indices[:new_prefix], inp.kv_indices[L:L + T]]).astype(np.int32)
    inp.kv_indptr = np.array([0, new_prefix + T], dtype=np.int32)
    inp.parents = random_parents(np.random.default_rng(seed), T, 16)
    return inp


def test_long_context_graph_replay_with_changing_lengths():
    wl = WORKLOADS["long"]
    inp = generate(wl)
    attn = make_attention(wl)
    anc = product_anc(inp)
    d = wdev.to_device(inp, anc)
    stream = torch.cuda.Stream()
    args = attn.make_args(*wdev.positional(d), lse=d["lse"], visible_count=d["visible_count"])
    with torch.cuda.stream(stream):          # warm up before capture (first launch configures the kernel)
        attn.run(args, stream.cuda_stream)
        attn.reduce(args, stream.cuda_stream)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        attn.run(args, stream.cuda_stream)
        attn.reduce(args, stream.cuda_stream)

    # replay as captured
    d["out"].zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert attn.status()[0] == 0
    _check(inp, d)

    # shorter prefixes and new trees, written into the same device buffers
    for new_prefix, seed in ((40000, 1), (1000, 2), (65536, 3)):
        inp = _shrink(inp, new_prefix, seed) if new_prefix != 65536 else generate(wl)
        anc = product_anc(inp)
        d["kv_indices"][: inp.kv_indices.shape[0]].copy_(torch.from_numpy(inp.kv_indices))
        d["kv_indptr"].copy_(torch.from_numpy(inp.kv_indptr))
        d["tree_anc"].copy_(torch.from_numpy(anc.view(np.int64)))
        d["out"].zero_()
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        assert attn.status()[0] == 0
        _check(inp, d)
    del graph
