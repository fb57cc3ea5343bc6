"""CPU tests of the C-ABI library: it loads, exports what the header declares,
validates plans and arguments with the documented codes, and its host tree
mask helper matches the oracle bit for bit. No kernel is launched here."""
import ctypes
import os
import re

import numpy as np
import pytest

import mla_speculative_verify_absorb_b200 as va
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "verify_attn.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(verify_attn_\w+)\s*\(", text, flags=re.M)))


def test_library_exports_every_declared_symbol():
    lib = va.load_library()
    names = _declared_functions()
    assert len(names) >= 7
    for name in names:
        assert hasattr(lib, name), name
    assert os.path.dirname(va.lib_path()).startswith(ROOT)


def test_strerror_covers_codes():
    for code in range(0, -7, -1):
        s = va.verify_attn_strerror(code)
        assert s and "unknown" not in s
    assert "unknown" in va.verify_attn_strerror(-99)


def _params(**kw):
    base = dict(max_batch=1, num_heads=64, max_tree=64, d_latent=512, d_rope=64, num_sms=148,
                max_kv_per_req=65600, max_total_kv=65600, pool_slots=262144, sm_scale=192 ** -0.5)
    base.update(kw)
    return va.VerifyAttnParams(**base)


def test_plan_long_context_layout():
    plan, ws = va.verify_attn_plan(_params())
    assert plan.version == 2
    assert plan.num_clusters == 74                  # one CTA pair per two SMs
    assert plan.row_tiles_per_req == 32             # 64 nodes x 64 heads / 128
    assert plan.num_slots == 74 + 32
    assert plan.ws_meta_offset == 256
    assert plan.ws_partial_offset % 256 == 0
    assert plan.keys_per_tile == 256
    assert plan.ws_stage_offset % 1024 == 0
    assert plan.ws_stage_offset >= plan.ws_partial_offset + plan.num_slots * 128 * 512 * 4
    assert plan.stage_rows == 256 * ((65600 + 255) // 256 + 1)   # whole key tiles, one spare per request
    assert ws == plan.ws_bytes == plan.ws_stage_offset + plan.stage_rows * 576 * 2
    assert 0 < plan.split_smem_bytes <= 232448


def test_plan_caps_clusters_by_work():
    plan, _ = va.verify_attn_plan(_params(num_heads=8, max_tree=4, max_kv_per_req=260, max_total_kv=260,
                                          pool_slots=4096))
    assert plan.num_clusters == 2                   # 1 row tile x 2 key tiles of 256


@pytest.mark.parametrize("kw,code", [
    (dict(d_latent=256), -2), (dict(d_rope=32), -2), (dict(max_tree=65), -2), (dict(num_heads=2048), -2),
    (dict(max_tree=0), -1), (dict(num_heads=0), -1), (dict(max_batch=0), -1),
    (dict(max_kv_per_req=10), -1), (dict(pool_slots=0), -1), (dict(sm_scale=0.0), -1),
    (dict(sm_scale=float("inf")), -1), (dict(max_total_kv=1), -1), (dict(num_sms=1), -1),
])
def test_plan_rejects_bad_maxima(kw, code):
    with pytest.raises(va.VerifyAttnError) as e:
        va.verify_attn_plan(_params(**kw))
    assert e.value.code == code


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="uses fake device pointers; host-only check")
def test_run_rejects_bad_arguments_without_launching():
    plan, ws = va.verify_attn_plan(_params())
    lib = va.load_library()
    args = va.VerifyAttnArgs(q_latent=16, q_latent_stride_tok=64 * 512, q_latent_stride_head=512,
                             q_rope=16, q_rope_stride_tok=64 * 64, q_rope_stride_head=64,
                             kv_pool=16, kv_row_stride=576, kv_indices=16, kv_indptr=16, qo_indptr=16,
                             tree_anc=16, batch=1, out=16, out_stride_tok=64 * 512, out_stride_head=512)
    P = ctypes.byref
    # workspace too small
    assert lib.verify_attn_run(P(plan), P(args), 256, ws - 1, None) == -3
    # batch above the plan
    args.batch = 2
    assert lib.verify_attn_run(P(plan), P(args), 256, ws, None) == -1
    args.batch = 1
    # misaligned pool pointer, short pool rows, odd strides
    args.kv_pool = 8
    assert lib.verify_attn_run(P(plan), P(args), 256, ws, None) == -1
    args.kv_pool = 16
    args.kv_row_stride = 568
    assert lib.verify_attn_run(P(plan), P(args), 256, ws, None) == -1
    args.kv_row_stride = 576
    args.q_rope_stride_head = 60
    assert lib.verify_attn_run(P(plan), P(args), 256, ws, None) == -1
    args.q_rope_stride_head = 64
    # reduce needs an output
    args.out = None
    assert lib.verify_attn_reduce(P(plan), P(args), 256, ws, None) == -1
    # a plan that was never filled
    assert lib.verify_attn_run(P(va.VerifyAttnPlan()), P(args), 256, ws, None) == -1
    assert lib.verify_attn_run(P(plan), None, 256, ws, None) == -1


def test_tree_mask_helper_matches_oracle():
    rng = np.random.default_rng(7)
    for T in (1, 2, 3, 9, 33, 64):
        for _ in range(5):
            parents = np.full(T, -1, np.int32)
            for i in range(1, T):
                parents[i] = rng.integers(0, i)
            ours = va.verify_attn_build_tree_mask(parents)
            ref = oracle.ancestor_masks(parents, np.array([0, T], np.int32))
            assert np.array_equal(ours, ref)


@pytest.mark.parametrize("parents", [[0], [-1, 1], [-1, 0, 3], [-1, -1], list(range(-1, 64))])
def test_tree_mask_helper_rejects_malformed(parents):
    with pytest.raises(va.VerifyAttnError) as e:
        va.verify_attn_build_tree_mask(np.asarray(parents, np.int32))
    assert e.value.code == -1


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="uses fake device pointers; host-only check")
def test_variant_entry_points_reject_bad_arguments_without_launching():
    """Relocation, tree block and both merges validate before any launch."""
    lib = va.load_library()
    P = ctypes.byref
    d = va.VerifyAttnDefragArgs(kv_pool=16, kv_row_stride=576, pool_slots=100, kv_indices=16, kv_indptr=16,
                                dst_begin=16, batch=1, budget=4, max_total_kv=10, status=None)
    for field, bad in (("kv_pool", 8), ("kv_row_stride", 570), ("kv_row_stride", 560), ("batch", 0),
                       ("budget", -1), ("pool_slots", 0), ("max_total_kv", -1), ("dst_begin", None)):
        good = getattr(d, field)
        setattr(d, field, bad)
        assert lib.verify_attn_defrag(P(d), None) == -1, field
        setattr(d, field, good)
    assert lib.verify_attn_defrag(None, None) == -1

    m = va.VerifyAttnMergeArgs(o_a=16, o_a_stride_tok=4096, o_a_stride_head=512, lse_a=16, o_b=16,
                               o_b_stride_tok=4096, o_b_stride_head=512, lse_b=16, o_b_f32=0, out=16,
                               out_stride_tok=4096, out_stride_head=512, lse=None, max_tokens=4, num_tokens=None,
                               num_heads=8)
    for field, bad in (("o_a", 8), ("out", None), ("lse_b", None), ("o_b_stride_head", 4), ("num_heads", 0),
                       ("num_heads", 2048), ("max_tokens", -1)):
        good = getattr(m, field)
        setattr(m, field, bad)
        assert lib.verify_attn_merge_states(P(m), None) == -1, field
        setattr(m, field, good)
    m.max_tokens = 0                                        # nothing to merge: no launch, success
    assert lib.verify_attn_merge_states(P(m), None) == 0

    s = va.VerifyAttnMergeStackedArgs(o=16, lse_states=16, num_states=2, num_heads=8, out=16,
                                      out_stride_tok=4096, out_stride_head=512, lse=None, max_tokens=4,
                                      num_tokens=None)
    for field, bad in (("num_states", 0), ("num_states", 1025), ("o", 8), ("out_stride_tok", 100),
                       ("lse_states", None), ("max_tokens", -2)):
        good = getattr(s, field)
        setattr(s, field, bad)
        assert lib.verify_attn_merge_stacked(P(s), None) == -1, field
        setattr(s, field, good)
    s.max_tokens = 0
    assert lib.verify_attn_merge_stacked(P(s), None) == 0

    plan, ws = va.verify_attn_plan(_params())
    args = va.VerifyAttnArgs(q_latent=16, q_latent_stride_tok=64 * 512, q_latent_stride_head=512,
                             q_rope=16, q_rope_stride_tok=64 * 64, q_rope_stride_head=64,
                             kv_pool=16, kv_row_stride=576, kv_indices=16, kv_indptr=16, qo_indptr=16,
                             tree_anc=16, batch=1, out=16, out_stride_tok=64 * 512, out_stride_head=512, lse=None)
    # the tree block needs an LSE output, and an output of one kind or the other
    assert lib.verify_attn_tree_block(P(plan), P(args), 1, None, None, 256, ws, None) == -1
    args.lse = 16
    args.out = None
    assert lib.verify_attn_tree_block(P(plan), P(args), 1, None, None, 256, ws, None) == -1
    assert lib.verify_attn_tree_block(P(plan), P(args), 1, None, 8, 256, ws, None) == -1   # misaligned fp32 out
    assert lib.verify_attn_tree_block(P(plan), P(args), 1, None, 16, 256, ws - 1, None) == -3
