"""Device-side input errors are reported in the status word, never fault,
and leave the other requests' results exact.

Each case is one the kernels check before acting on it:
* a kv_indices slot outside the pool: the gather writes a zero row instead
  of reading the pool and sets the bad-slot bit;
* a tree mask with a bit at or beyond T: the bit would name a key past the
  request's KV and is masked out; the reduce sets the bad-tree bit;
* a request longer than the plan's max_tree: the request is skipped (its
  output rows are not written) and the bad-length bit is set.
"""
import numpy as np
import pytest
import torch

import mla_speculative_verify_absorb_b200 as va
import oracle
from gpu_common import MAX_ABS, REL_L2, make_attention, product_anc
from workloads import custom, generate
from workloads import device as wdev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

BAD_LENGTHS, BAD_SLOT, BAD_TREE = 1 << 1, 1 << 2, 1 << 3


def _run(attn, d):
    attn(*wdev.positional(d), lse=d["lse"], visible_count=d["visible_count"])
    torch.cuda.synchronize()
    return attn.status()


def _rows_of(inp, b):
    H = inp.q_latent.shape[1]
    q0, q1 = int(inp.qo_indptr[b]), int(inp.qo_indptr[b + 1])
    return np.arange(q0 * H, q1 * H, dtype=np.int64)


def _check_rows(inp, d, rows):
    ref_anc = oracle.ancestor_masks(inp.parents, inp.qo_indptr)
    ref, ref_lse, _ = oracle.verify_rows(inp, ref_anc, rows=rows)
    out = d["out"].float().cpu().numpy().astype(np.float64).reshape(-1, 512)[rows]
    assert np.isfinite(out).all()
    assert np.abs(out - ref).max() <= MAX_ABS
    assert np.linalg.norm(out - ref) / np.linalg.norm(ref) <= REL_L2


def test_slot_outside_pool():
    inp = generate(custom("badslot", 51, 8, [700, 300], [9, 5], 4096))
    anc = product_anc(inp)
    attn = make_attention(inp.workload)
    d = wdev.to_device(inp, anc)
    d["kv_indices"][17] = inp.workload.pool_slots        # request 0, prefix position 17
    code, bits = _run(attn, d)
    assert code == -6 and bits & BAD_SLOT and not bits & 1
    assert torch.isfinite(d["out"].float()).all()
    _check_rows(inp, d, _rows_of(inp, 1))                 # the other request is untouched


def test_tree_bit_beyond_request():
    inp = generate(custom("badtree", 52, 8, [500], [12], 2048))
    anc = product_anc(inp)
    attn = make_attention(inp.workload)
    d = wdev.to_device(inp, anc)
    bad = anc.copy()
    bad[3] |= np.uint64(1) << np.uint64(12)               # node 12 does not exist (T = 12)
    d["tree_anc"].copy_(torch.from_numpy(bad.view(np.int64)))
    code, bits = _run(attn, d)
    assert code == -6 and bits & BAD_TREE and not bits & 1
    _check_rows(inp, d, _rows_of(inp, 0))                 # the stray bit names no key: results exact


def test_request_longer_than_plan():
    inp = generate(custom("badlen", 53, 8, [400, 600], [9, 4], 4096))
    anc = product_anc(inp)
    attn = make_attention(inp.workload, max_tree=8)        # request 0 has 9 nodes
    d = wdev.to_device(inp, anc)
    d["out"].fill_(7.0)
    code, bits = _run(attn, d)
    assert code == -6 and bits & BAD_LENGTHS and not bits & 1
    rows0 = torch.from_numpy(_rows_of(inp, 0)).cuda()
    assert (d["out"].reshape(-1, 512)[rows0] == 7.0).all()   # skipped, not written
    _check_rows(inp, d, _rows_of(inp, 1))
