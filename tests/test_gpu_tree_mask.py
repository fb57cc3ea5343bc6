"""GPU test of verify_attn_build_tree_mask_device against the oracle's masks
(bit-exact), including a malformed tree that must be flagged while the other
requests of the batch stay correct."""
import numpy as np
import pytest
import torch

import mla_speculative_verify_absorb_b200 as va
import oracle
from workloads import random_parents

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _batch(seed, sizes, depth=None):
    rng = np.random.default_rng(seed)
    parents = np.concatenate([random_parents(rng, T, depth) for T in sizes]).astype(np.int32)
    qo = np.zeros(len(sizes) + 1, np.int32)
    qo[1:] = np.cumsum(sizes)
    return parents, qo


def _run(parents, qo):
    p = torch.from_numpy(parents).cuda()
    q = torch.from_numpy(qo).cuda()
    anc = torch.zeros(parents.shape[0], dtype=torch.int64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    va.verify_attn_build_tree_mask_device(p.data_ptr(), q.data_ptr(), len(qo) - 1, anc.data_ptr(), status.data_ptr(),
                                          torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return anc.cpu().numpy().view(np.uint64), int(status.item())


@pytest.mark.parametrize("sizes,depth", [([4], None), ([64], 16), ([1, 2, 3, 33, 64, 17], None), ([32] * 4, None),
                                         ([64] * 8, 8)])
def test_device_masks_match_oracle(sizes, depth):
    parents, qo = _batch(sum(sizes) + len(sizes), sizes, depth)
    anc, status = _run(parents, qo)
    assert status == 0
    assert np.array_equal(anc, oracle.ancestor_masks(parents, qo))


def test_malformed_tree_is_flagged_and_isolated():
    parents, qo = _batch(5, [9, 12, 7])
    parents[9 + 4] = 6            # request 1, node 4 points forward: malformed
    anc, status = _run(parents, qo)
    assert status & (1 << 3)
    good = oracle.ancestor_masks(parents[:9], qo[:2])
    assert np.array_equal(anc[:9], good)
    assert np.array_equal(anc[9:21], (np.uint64(1) << np.arange(12, dtype=np.uint64)))
    third = oracle.ancestor_masks(parents[21:], np.array([0, 7], np.int32))
    assert np.array_equal(anc[21:], third)
