"""KV relocation on the GPU against the oracle's relocation.

Page "The Execution Phase", section "Tier 0 KV Defragmentation" defers live
relocation of a request's fragmented slots (Tier 1); the library's kernel
places each request's leading min(N_b, budget) positions in one contiguous
run. Pool and indices must match the oracle bit for bit, attention over the
relocated pool must be bit-identical to attention over the original one, a
second call with the same runs must change nothing, and bad slots or runs
must be reported and skipped.
"""
import numpy as np
import pytest
import torch

import mla_speculative_verify_absorb_b200 as va
import oracle.defrag as odf
from gpu_common import make_attention, product_anc
from workloads import custom, generate
from workloads import device as wdev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

BAD_LENGTHS, BAD_SLOT = 1 << 1, 1 << 2
BF16_NAN = 0x7FC0


def _extended(inp, budget, stride=576, pad_value=0x1234):
    """The pool with free rows appended for every request's run, and the runs' first slots."""
    P = inp.workload.pool_slots
    lens = np.diff(inp.kv_indptr)
    n = np.minimum(lens, budget)
    dst_begin = (P + np.concatenate([[0], np.cumsum(n)[:-1]])).astype(np.int32)
    pool = np.full((P + int(n.sum()), stride), pad_value, dtype=np.uint16)
    pool[:, :576] = BF16_NAN
    pool[:P, :576] = inp.kv_pool
    return pool, dst_begin


def _run(pool, idx, indptr, dst_begin, budget):
    d_pool = torch.from_numpy(pool.view(np.int16)).cuda().view(torch.bfloat16)
    d_idx = torch.from_numpy(idx.astype(np.int32)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    va.defrag(d_pool, d_idx, torch.from_numpy(indptr.astype(np.int32)).cuda(),
              torch.from_numpy(dst_begin).cuda(), budget, status=status)
    torch.cuda.synchronize()
    return d_pool.view(torch.int16).cpu().numpy().view(np.uint16), d_idx.cpu().numpy(), int(status.item())


@pytest.mark.parametrize("budget", [0, 1, 37, 300, 10 ** 6])
@pytest.mark.parametrize("stride", [576, 640])
def test_defrag_matches_oracle(budget, stride):
    inp = generate(custom("defrag", 61, 8, [700, 1, 300, 0, 1500], [9, 1, 5, 3, 17], 8192))
    pool, dst_begin = _extended(inp, budget, stride)
    ref_pool, ref_idx = odf.defrag(pool, inp.kv_indices, inp.kv_indptr, dst_begin, budget)
    got_pool, got_idx, st = _run(pool, inp.kv_indices, inp.kv_indptr, dst_begin, budget)
    assert st == 0
    assert np.array_equal(got_idx, ref_idx)
    assert np.array_equal(got_pool, ref_pool)          # includes the untouched row padding


def test_defrag_is_idempotent_and_keeps_in_place_rows():
    inp = generate(custom("defrag2", 62, 8, [513, 0, 64], [4, 1, 6], 4096))
    pool, dst_begin = _extended(inp, 10 ** 6)
    assert inp.kv_indptr[2] - inp.kv_indptr[1] == 1
    dst_begin[1] = inp.kv_indices[inp.kv_indptr[1]]       # a one-row request already in its run
    once_pool, once_idx, st = _run(pool, inp.kv_indices, inp.kv_indptr, dst_begin, 10 ** 6)
    assert st == 0
    ref_pool, ref_idx = odf.defrag(pool, inp.kv_indices, inp.kv_indptr, dst_begin, 10 ** 6)
    assert np.array_equal(once_idx, ref_idx) and np.array_equal(once_pool, ref_pool)
    twice_pool, twice_idx, st = _run(once_pool, once_idx, inp.kv_indptr, dst_begin, 10 ** 6)
    assert st == 0
    assert np.array_equal(twice_idx, once_idx) and np.array_equal(twice_pool, once_pool)
    for b in range(3):                                    # each run is now contiguous
        k0, k1 = inp.kv_indptr[b], inp.kv_indptr[b + 1]
        assert np.array_equal(once_idx[k0:k1], dst_begin[b] + np.arange(k1 - k0))


def test_attention_unchanged_by_relocation():
    inp = generate(custom("defrag3", 63, 16, [900, 2100], [11, 7], 8192))
    anc = product_anc(inp)
    pool, dst_begin = _extended(inp, 1000)               # request 1 keeps a fragmented tail
    new_pool, new_idx, st = _run(pool, inp.kv_indices, inp.kv_indptr, dst_begin, 1000)
    assert st == 0
    outs = []
    for p, idx in ((pool, inp.kv_indices), (new_pool, new_idx)):
        attn = make_attention(inp.workload, pool_slots=p.shape[0])
        d = wdev.to_device(inp, anc)
        d["kv_pool"] = torch.from_numpy(np.ascontiguousarray(p).view(np.int16)).cuda().view(torch.bfloat16)
        d["kv_indices"] = torch.from_numpy(idx.astype(np.int32)).cuda()
        attn(*wdev.positional(d), lse=d["lse"], visible_count=d["visible_count"])
        torch.cuda.synchronize()
        assert attn.status()[0] == 0
        outs.append((d["out"].view(torch.int16).cpu().numpy(), d["lse"].cpu().numpy()))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])


def test_bad_slot_and_bad_run_are_reported_and_skipped():
    inp = generate(custom("defrag4", 64, 8, [200, 300], [3, 3], 2048))
    pool, dst_begin = _extended(inp, 10 ** 6)
    idx = inp.kv_indices.copy()
    idx[5] = pool.shape[0]                                # request 0, position 5: outside the pool
    got_pool, got_idx, st = _run(pool, idx, inp.kv_indptr, dst_begin, 10 ** 6)
    assert st & BAD_SLOT and not st & BAD_LENGTHS
    assert got_idx[5] == idx[5]
    keep = np.ones(len(idx), bool)
    keep[5] = False
    ref_pool, ref_idx = odf.defrag(pool, np.where(keep, idx, 0), inp.kv_indptr, dst_begin, 10 ** 6)
    assert np.array_equal(got_idx[keep], ref_idx[keep])
    rows = np.ones(pool.shape[0], bool)
    rows[dst_begin[0] + 5] = False                        # the skipped destination row stays free
    assert np.array_equal(got_pool[rows], ref_pool[rows])
    assert np.all(got_pool[dst_begin[0] + 5] == pool[dst_begin[0] + 5])

    bad_runs = dst_begin.copy()
    bad_runs[1] = pool.shape[0] - 10                      # 300 rows cannot fit
    got_pool, got_idx, st = _run(pool, inp.kv_indices, inp.kv_indptr, bad_runs, 10 ** 6)
    assert st & BAD_LENGTHS and not st & BAD_SLOT
    k1 = inp.kv_indptr[1]
    assert np.array_equal(got_idx[k1:], inp.kv_indices[k1:])   # request 1 untouched
    ref_pool, ref_idx = odf.defrag(pool, inp.kv_indices, inp.kv_indptr[:2], dst_begin[:1], 10 ** 6)
    assert np.array_equal(got_idx[:k1], ref_idx[:k1]) and np.array_equal(got_pool, ref_pool)
