"""Why the split-verify composition keeps the tree-block state in fp32 (CPU).

The pages merge two bf16 states (page "The Architecture Detective", section
"The Split Verify Design"). For a request with an empty prefix, the output
is a mix of a few latent rows of magnitude up to ~4, where one bf16 step is
2^-6. Rounding both states and then the merged output stacks two such
errors. These checks take the exact float64 states from the oracle, apply
each rounding scheme, and compare with the oracle's one-shot rows against
the path's tolerance: two bf16 states exceed it, an fp32 tree-block state
stays inside.
"""
import numpy as np

import oracle
from workloads import _to_bf16_bits, bf16_bits_to_f64, custom, generate

MAX_ABS = 1e-2


def _bf(x):
    return bf16_bits_to_f64(_to_bf16_bits(np.asarray(x, dtype=np.float32)))


def _states():
    # request 0: empty prefix, a 3-node tree; 32 heads
    inp = generate(custom("sv_ragged", 73, 32, [0, 777, 4000, 12], [3, 64, 9, 1], 16384))
    anc = oracle.ancestor_masks(inp.parents, inp.qo_indptr)
    T, H = 3, 32
    rows = np.arange(T * H, dtype=np.int64)
    t = rows // H
    self_only = anc.copy()
    strict = anc.copy()
    for i in range(T):
        self_only[i] = np.uint64(1) << np.uint64(i)
        strict[i] = anc[i] & ~(np.uint64(1) << np.uint64(i))
    mp, lp, op = oracle.partial_rows(inp, self_only, 0, T, rows=rows)     # dense pass: own key (L = 0)
    mt, lt, ot = oracle.partial_rows(inp, strict, 0, T, rows=rows)        # tree block: strict ancestors
    ref, ref_lse, _ = oracle.verify_rows(inp, anc, rows=rows)
    return (mp, lp, op), (mt, lt, ot), ref, t


def _compose(dense, tree, round_tree):
    mp, lp, op = dense
    mt, lt, ot = tree
    o_p = _bf(op / lp[:, None])
    lse_p = mp + np.log(lp)
    has_t = lt > 0
    o_t = np.zeros_like(ot)
    o_t[has_t] = ot[has_t] / lt[has_t, None]
    if round_tree:
        o_t = _bf(o_t)
    lse_t = np.where(has_t, mt + np.log(np.where(has_t, lt, 1.0)), -np.inf)
    m = np.maximum(lse_p, lse_t)
    wp, wt = np.exp(lse_p - m), np.exp(lse_t - m)
    return _bf((wp[:, None] * o_p + wt[:, None] * o_t) / (wp + wt)[:, None])


def test_fp32_tree_state_stays_within_tolerance():
    dense, tree, ref, t = _states()
    assert (tree[1][t > 0] > 0).all() and (tree[1][t == 0] == 0).all()    # only the root has no strict ancestor
    err = np.abs(_compose(dense, tree, round_tree=False) - ref).max()
    assert err <= MAX_ABS


def test_two_bf16_states_exceed_tolerance_here():
    dense, tree, ref, _ = _states()
    err = np.abs(_compose(dense, tree, round_tree=True) - ref).max()
    assert err > MAX_ABS
