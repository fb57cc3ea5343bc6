"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test fixes part of the definition (MLA-absorb attention with an
ancestor-or-self tree mask: page "The Execution Phase", section "The
Transition: From Planning to Execution"; the tree block mask and the dense
prefix: page "The Architecture Detective", section "The Split Verify
Design"; the partial-state merge: same page and section, plus page "The
Verify Kernel Breakthrough", section "The Message in Context") with an
independent check:

* library routine: a chain tree is plain causal attention, and any tree is
  attention with the walked-parents mask -- both against torch's float64
  ``scaled_dot_product_attention``;
* exact special cases: one visible token returns its latent row bit for bit;
  equal scores return the mean visible row with lse = ln |V|;
* invariance: permuting pool rows together with kv_indices changes nothing;
* brute force: a separately written dense numpy version on tiny inputs;
* closed forms for the masks (chain, star, transitive closure) and the
  printed tiny-workload visible counts under ``tests/golden``;
* the merge identity: merged partial states equal the one-shot result.

A dropped rope term, a value that includes k_rope, a wrong scale, a mask
shifted by one position or a transposed operand each break at least one of
these.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from workloads import custom, generate, bf16_bits_to_f64, WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows_f64(inp):
    return bf16_bits_to_f64(inp.kv_pool)


def _sdpa(inp, b, mask):
    """torch float64 SDPA for request b with a [T, N] boolean mask."""
    q0, q1 = int(inp.qo_indptr[b]), int(inp.qo_indptr[b + 1])
    k0, k1 = int(inp.kv_indptr[b]), int(inp.kv_indptr[b + 1])
    q = np.concatenate([bf16_bits_to_f64(inp.q_latent[q0:q1]), bf16_bits_to_f64(inp.q_rope[q0:q1])], -1)
    rows = bf16_bits_to_f64(inp.kv_pool[inp.kv_indices[k0:k1]])
    H = q.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]                          # [1, H, T, 576]
    kt = torch.from_numpy(rows)[None, None].expand(1, H, -1, -1)              # [1, H, N, 576]
    vt = torch.from_numpy(rows[:, :512].copy())[None, None].expand(1, H, -1, -1)
    m = torch.from_numpy(mask)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=inp.sm_scale)
    return o[0].permute(1, 0, 2).numpy()                                      # [T, H, 512]


def _oracle_all(inp):
    anc = oracle.ancestor_masks(inp.parents, inp.qo_indptr)
    out, lse, vis = oracle.verify_rows(inp, anc)
    H = inp.q_latent.shape[1]
    return anc, out.reshape(-1, H, 512), lse.reshape(-1, H), vis.reshape(-1, H)


# ----------------------------------------------------------------------------- masks

def test_ancestor_masks_chain_closed_form():
    T = 64
    parents = np.arange(-1, T - 1, dtype=np.int32)
    anc = oracle.ancestor_masks(parents, np.array([0, T], np.int32))
    for i in range(T):
        assert int(anc[i]) == (1 << (i + 1)) - 1


def test_ancestor_masks_star_closed_form():
    T = 17
    parents = np.array([-1] + [0] * (T - 1), dtype=np.int32)
    anc = oracle.ancestor_masks(parents, np.array([0, T], np.int32))
    assert int(anc[0]) == 1
    for i in range(1, T):
        assert int(anc[i]) == 1 | (1 << i)
        assert bin(int(anc[i])).count("1") == 2


def test_ancestor_masks_match_transitive_closure():
    rng = np.random.default_rng(123)
    for T in (1, 2, 5, 31, 64):
        parents = np.full(T, -1, np.int32)
        for i in range(1, T):
            parents[i] = rng.integers(0, i)
        # reachability by repeated boolean products of the parent adjacency
        adj = np.zeros((T, T), dtype=bool)
        for i in range(1, T):
            adj[i, parents[i]] = True
        reach = np.eye(T, dtype=bool)
        step = np.eye(T, dtype=bool)
        for _ in range(T):
            step = (step.astype(np.int64) @ adj.astype(np.int64)) > 0
            reach |= step
        anc = oracle.ancestor_masks(parents, np.array([0, T], np.int32))
        for i in range(T):
            expect = sum(1 << j for j in range(T) if reach[i, j])
            assert int(anc[i]) == expect


@pytest.mark.parametrize("parents", [[0, 0], [-1, 1], [-1, 0, 3, 0], [-1, -1], []])
def test_ancestor_masks_reject_malformed(parents):
    p = np.asarray(parents, dtype=np.int32)
    with pytest.raises(ValueError):
        oracle.ancestor_masks(p, np.array([0, len(parents)], np.int32))


def test_ancestor_masks_reject_oversized_tree():
    T = 65
    parents = np.arange(-1, T - 1, dtype=np.int32)
    with pytest.raises(ValueError):
        oracle.ancestor_masks(parents, np.array([0, T], np.int32))


def test_tiny_visible_counts_golden():
    expect = [int(x) for x in open(os.path.join(GOLDEN, "tiny_visible_counts.txt"))
              if x.strip() and not x.startswith("#")]
    inp = generate(WORKLOADS["tiny"])
    _, _, _, vis = _oracle_all(inp)
    assert vis[:, 0].tolist() == expect
    assert (vis == vis[:, :1]).all()      # same for every head


def test_visible_counts_chain_and_star():
    L = 11
    chain = custom("chain", 7, 2, [L], [9], 64, fixed_parents=tuple(range(-1, 8)))
    star = custom("star", 7, 2, [L], [9], 64, fixed_parents=(-1,) + (0,) * 8)
    _, _, _, vc = _oracle_all(generate(chain))
    _, _, _, vs = _oracle_all(generate(star))
    assert vc[:, 0].tolist() == [L + t + 1 for t in range(9)]
    assert vs[:, 0].tolist() == [L + 1] + [L + 2] * 8


# ----------------------------------------------------------------------------- library routine

def test_chain_tree_equals_causal_attention():
    T, L = 12, 53
    wl = custom("chain", 11, 4, [L], [T], 128, fixed_parents=tuple(range(-1, T - 1)))
    inp = generate(wl)
    _, out, _, _ = _oracle_all(inp)
    N = L + T
    causal = np.zeros((T, N), dtype=bool)
    for t in range(T):
        causal[t, : L + t + 1] = True           # bottom-right aligned causal mask
    ref = _sdpa(inp, 0, causal)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-11)


def test_random_trees_equal_masked_attention():
    wl = custom("trees", 12, 3, [40, 0, 7], [9, 5, 16], 512)
    inp = generate(wl)
    _, out, _, _ = _oracle_all(inp)
    for b in range(3):
        q0, q1 = int(inp.qo_indptr[b]), int(inp.qo_indptr[b + 1])
        L = wl.prefixes[b]
        mask = brute.visibility(inp.parents[q0:q1], L)
        ref = _sdpa(inp, b, mask)
        np.testing.assert_allclose(out[q0:q1], ref, rtol=0, atol=1e-11)


# ----------------------------------------------------------------------------- exact special cases

def test_single_visible_token_returns_its_latent_row():
    # Empty prefixes, one tree node per request: the root sees only itself.
    wl = custom("single", 13, 5, [0, 0, 0], [1, 1, 1], 64)
    inp = generate(wl)
    _, out, lse, vis = _oracle_all(inp)
    assert (vis == 1).all()
    for b in range(3):
        slot = int(inp.kv_indices[inp.kv_indptr[b]])
        row = bf16_bits_to_f64(inp.kv_pool[slot])
        for h in range(5):
            assert np.array_equal(out[b, h], row[:512])     # p = 1 exactly, v = c_kv only
            q = np.concatenate([bf16_bits_to_f64(inp.q_latent[b, h]), bf16_bits_to_f64(inp.q_rope[b, h])])
            assert abs(lse[b, h] - inp.sm_scale * float(q @ row)) < 1e-12


def test_equal_scores_return_mean_of_visible_rows():
    wl = custom("equal", 14, 3, [20, 5], [6, 8], 256, fixed_parents=((-1, 0, 1, 1, 0, 4), (-1, 0, 0, 2, 3, 3, 5, 6)))
    inp = generate(wl)
    inp.q_latent[:] = 0
    inp.q_rope[:] = 0
    anc, out, lse, vis = _oracle_all(inp)
    for b in range(2):
        q0, q1 = int(inp.qo_indptr[b]), int(inp.qo_indptr[b + 1])
        k0, k1 = int(inp.kv_indptr[b]), int(inp.kv_indptr[b + 1])
        L = wl.prefixes[b]
        mask = brute.visibility(inp.parents[q0:q1], L)
        rows = bf16_bits_to_f64(inp.kv_pool[inp.kv_indices[k0:k1]])[:, :512]
        for t in range(q1 - q0):
            mean = rows[mask[t]].mean(axis=0)
            for h in range(3):
                np.testing.assert_allclose(out[q0 + t, h], mean, rtol=0, atol=1e-13)
                assert abs(lse[q0 + t, h] - np.log(mask[t].sum())) < 1e-13


def test_permuting_pool_rows_with_indices_changes_nothing():
    wl = custom("perm", 15, 4, [33, 9], [7, 12], 300)
    inp = generate(wl)
    _, out, lse, vis = _oracle_all(inp)
    perm = np.random.default_rng(99).permutation(inp.kv_pool.shape[0])
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    inp.kv_pool = inp.kv_pool[perm]                 # new slot s holds old row perm[s]
    inp.kv_indices = inv[inp.kv_indices].astype(np.int32)
    _, out2, lse2, vis2 = _oracle_all(inp)
    assert np.array_equal(out, out2)
    assert np.array_equal(lse, lse2)
    assert np.array_equal(vis, vis2)


# ----------------------------------------------------------------------------- brute force

@pytest.mark.parametrize("name", ["tiny", "custom"])
def test_numpy_brute_force_agrees(name):
    if name == "tiny":
        inp = generate(WORKLOADS["tiny"])
    else:
        inp = generate(custom("bf", 16, 6, [0, 70, 3], [3, 13, 1], 200))
    _, out, lse, _ = _oracle_all(inp)
    ref_out, ref_lse = brute.verify(inp)
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- merge identity

@pytest.mark.parametrize("cuts", [[30], [1, 40, 41], [0, 64, 70], [45, 46, 47, 48]])
def test_merged_partial_states_equal_one_shot(cuts):
    wl = custom("merge", 17, 4, [44], [9], 128)
    inp = generate(wl)
    anc, out, lse, _ = _oracle_all(inp)
    N = wl.kv_lens[0]
    bounds = [0] + list(cuts) + [N]
    ms, ls, os_ = [], [], []
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        m, l, o = oracle.partial_rows(inp, anc, lo, hi)
        ms.append(m), ls.append(l), os_.append(o)
    mout, mlse = oracle.merge_states(np.stack(ms), np.stack(ls), np.stack(os_))
    np.testing.assert_allclose(mout.reshape(out.shape), out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(mlse.reshape(lse.shape), lse, rtol=0, atol=1e-12)


def test_partial_state_without_visible_keys_is_empty():
    wl = custom("empty", 18, 2, [10], [5], 64, fixed_parents=(-1, 0, 0, 0, 0))
    inp = generate(wl)
    anc = oracle.ancestor_masks(inp.parents, inp.qo_indptr)
    # positions 12..14 are tree nodes 2..4: node 1 sees none of them
    m, l, o = oracle.partial_rows(inp, anc, 12, 15, rows=np.array([1 * 2 + 0, 1 * 2 + 1], np.int64))
    assert np.isneginf(m).all() and (l == 0).all() and (o == 0).all()
    out, lse = oracle.merge_states(m[None], l[None], o[None])
    assert (out == 0).all() and np.isneginf(lse).all()
