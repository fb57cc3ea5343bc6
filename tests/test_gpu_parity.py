"""GPU parity of the CUDA path (C ABI: verify_attn_run + verify_attn_reduce)
against the float64 oracle on the same seeded inputs.

Bar: bf16 output within max|err| <= 1e-2 and relative L2 <= 5e-3 of the
oracle; LSE within 2e-3; tree masks and visible-key counts bit-exact. Small
shapes are compared on every output; the full-size workloads (launched
exactly as the benchmark launches them) on sampled rows the oracle computes
one by one, plus every token's visible count.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import (closed_form_counts, compare, make_attention, oracle_all, run_gpu, sample_rows)
from workloads import WORKLOADS, custom, generate

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _full_check(inp):
    out, lse, vis, anc = run_gpu(inp)
    ref_anc, ref_out, ref_lse, ref_vis = oracle_all(inp)
    assert np.array_equal(anc, ref_anc)
    assert np.array_equal(vis, ref_vis[:, 0])
    return compare(out, ref_out, lse, ref_lse), out, ref_out


def test_tiny():
    _full_check(generate(WORKLOADS["tiny"]))


def test_tp8_slice():
    _full_check(generate(WORKLOADS["tp8"]))


EDGE = {
    # one request, one node, empty prefix: a single visible key
    "single_token": custom("single_token", 21, 8, [0], [1], 64),
    # chain tree: causal attention over the tree block
    "chain64": custom("chain64", 22, 2, [300], [64], 1024, fixed_parents=tuple(range(-1, 63))),
    # star tree, H not a power of two, rows spill into a second ragged row tile
    "star64_h3": custom("star64_h3", 23, 3, [129], [64], 1024, fixed_parents=(-1,) + (0,) * 63),
    # several requests: empty prefix, KV lengths on and off tile boundaries
    "batch5": custom("batch5", 24, 16, [0, 127, 128, 1000, 37], [5, 1, 64, 17, 33], 4096),
    "one_head": custom("one_head", 25, 1, [513], [64], 2048),
    "h100": custom("h100", 26, 100, [50], [64], 512),
    "h128_t1": custom("h128_t1", 27, 128, [255], [1], 512),
    "exact_tiles": custom("exact_tiles", 28, 8, [256 - 16], [16], 512, layout="contiguous"),
}


@pytest.mark.parametrize("name", sorted(EDGE))
def test_edge_cases(name):
    _full_check(generate(EDGE[name]))


def test_single_visible_token_is_exact():
    inp = generate(EDGE["single_token"])
    out, _, vis, _ = run_gpu(inp)
    slot = int(inp.kv_indices[0])
    row = (inp.kv_pool[slot, :512].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert (vis == 1).all()
    for h in range(8):
        assert np.array_equal(out[0, h], row)


def test_equal_scores_give_mean_row():
    inp = generate(custom("equal", 29, 8, [300], [9], 1024, fixed_parents=(-1, 0, 1, 2, 0, 4, 4, 6, 7)))
    inp.q_latent[:] = 0
    inp.q_rope[:] = 0
    out, _, _, _ = run_gpu(inp)
    _, ref_out, _, _ = oracle_all(inp)
    compare(out, ref_out)


def test_strided_query_and_output_views():
    """q / out given as views with padded token and head strides."""
    import mla_speculative_verify_absorb_b200 as va
    from workloads import device as wdev
    from gpu_common import product_anc

    inp = generate(custom("strided", 30, 8, [700], [12], 2048))
    anc = product_anc(inp)
    d = wdev.to_device(inp, anc)
    H = 8
    big_ql = torch.zeros((12, H + 2, 512 + 64), dtype=torch.bfloat16, device="cuda")
    big_ql[:, :H, :512] = d["q_latent"]
    big_qr = torch.zeros((12, H, 64 + 8), dtype=torch.bfloat16, device="cuda")
    big_qr[:, :, :64] = d["q_rope"]
    big_out = torch.zeros((12, H + 1, 512 + 8), dtype=torch.bfloat16, device="cuda")
    attn = make_attention(inp.workload)
    attn(big_ql[:, :H, :512], big_qr[:, :, :64], d["kv_pool"], d["kv_indices"], d["kv_indptr"], d["qo_indptr"],
         d["tree_anc"], big_out[:, :H, :512])
    torch.cuda.synchronize()
    assert attn.status()[0] == 0
    _, ref_out, _, _ = oracle_all(inp)
    compare(big_out[:, :H, :512].float().cpu().numpy().astype(np.float64), ref_out)
    assert (big_out[:, H:, :] == 0).all() and (big_out[:, :, 512:] == 0).all()


@pytest.mark.parametrize("name", ["full_contiguous", "full_scattered", "long", "ragged"])
def test_full_size_sampled(name):
    inp = generate(WORKLOADS[name])
    out, lse, vis, anc = run_gpu(inp)
    ref_anc = oracle.ancestor_masks(inp.parents, inp.qo_indptr)
    assert np.array_equal(anc, ref_anc)
    assert np.array_equal(vis, closed_form_counts(inp, ref_anc))
    H = inp.q_latent.shape[1]
    rows = sample_rows(inp, 24)
    ref_out, ref_lse, ref_vis = oracle.verify_rows(inp, ref_anc, rows=rows)
    got = out.reshape(-1, 512)[rows]
    compare(got, ref_out, lse.reshape(-1)[rows], ref_lse)
    assert np.array_equal(vis[rows // H], ref_vis)
    assert np.isfinite(out).all()
