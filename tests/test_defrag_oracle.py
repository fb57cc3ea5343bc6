"""Pins of the relocation oracle against what the operation must preserve.

The point of relocation is that attention sees the same KV afterwards: the
row sequence pool[kv_indices] of every request is unchanged, while the first
min(N_b, budget) positions become one contiguous run at dst_begin[b]. These
checks use only that property, the untouched remainder, idempotence and a
hand-worked example; a dropped copy, a wrong destination offset or a rewrite
of the wrong position each fail one of them.
"""
import numpy as np

from oracle.defrag import defrag


def _case(seed, lens=(37, 5, 120), pool_slots=600, stride=580):
    rng = np.random.default_rng(seed)
    total = sum(lens)
    slots = rng.permutation(pool_slots - total)[:total].astype(np.int32)   # sources in the low part
    pool = rng.integers(0, 1 << 16, size=(pool_slots, stride), dtype=np.uint16)
    kv_indptr = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    dst = (pool_slots - total + np.concatenate([[0], np.cumsum(lens)[:-1]])).astype(np.int32)  # free high part
    return pool, slots, kv_indptr, dst


def _rows(pool, idx, kv_indptr, b):
    return pool[idx[kv_indptr[b]:kv_indptr[b + 1]], :576]


def test_attention_inputs_unchanged_and_runs_contiguous():
    for budget in (0, 3, 37, 1000):
        pool, idx, ptr, dst = _case(1)
        new_pool, new_idx = defrag(pool, idx, ptr, dst, budget)
        for b in range(3):
            assert np.array_equal(_rows(new_pool, new_idx, ptr, b), _rows(pool, idx, ptr, b))
            n = min(int(ptr[b + 1] - ptr[b]), budget)
            assert np.array_equal(new_idx[ptr[b]:ptr[b] + n], dst[b] + np.arange(n))
            assert np.array_equal(new_idx[ptr[b] + n:ptr[b + 1]], idx[ptr[b] + n:ptr[b + 1]])


def test_other_slots_and_padding_untouched():
    pool, idx, ptr, dst = _case(2)
    new_pool, new_idx = defrag(pool, idx, ptr, dst, 1000)
    written = set(int(s) for s in new_idx) - set(int(s) for s in idx)
    untouched = [s for s in range(pool.shape[0]) if s not in written]
    assert np.array_equal(new_pool[untouched], pool[untouched])
    assert np.array_equal(new_pool[:, 576:], pool[:, 576:])          # row padding is never written


def test_idempotent():
    pool, idx, ptr, dst = _case(3)
    p1, i1 = defrag(pool, idx, ptr, dst, 50)
    p2, i2 = defrag(p1, i1, ptr, dst, 50)
    assert np.array_equal(p1, p2) and np.array_equal(i1, i2)


def test_worked_example():
    # two requests; request 0 keeps its second row where it is (already in place)
    pool = np.arange(8 * 576, dtype=np.uint16).reshape(8, 576)
    idx = np.array([5, 7, 2], dtype=np.int32)
    ptr = np.array([0, 2, 3], dtype=np.int32)
    dst = np.array([6, 0], dtype=np.int32)                            # run [6, 7] and run [0]
    new_pool, new_idx = defrag(pool, idx, ptr, dst, 2)
    assert list(new_idx) == [6, 7, 0]
    assert np.array_equal(new_pool[6], pool[5]) and np.array_equal(new_pool[7], pool[7])
    assert np.array_equal(new_pool[0], pool[2])
    assert np.array_equal(new_pool[[1, 2, 3, 4, 5]], pool[[1, 2, 3, 4, 5]])
