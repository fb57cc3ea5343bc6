"""The split-verify variant against the oracle.

Page "The Architecture Detective", section "The Split Verify Design": dense
prefix attention, a tiny masked tree-block attention and an LSE merge give
the same result as the one-pass verify attention. Each of the variant's
kernels is checked on its own (tree block against the oracle's partial state
over the tree keys, merge against the oracle's merge of states) and the
composition against the oracle's full rows, within the same tolerances as
the fused path.
"""
import numpy as np
import pytest
import torch

import mla_speculative_verify_absorb_b200 as va
import oracle
from gpu_common import LSE_ABS, MAX_ABS, REL_L2, compare, make_attention, product_anc
from workloads import WORKLOADS, custom, generate
from workloads import device as wdev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _strict(anc, inp):
    """Masks without each node's own bit (what the tree block attends with exclude_self)."""
    out = np.asarray(anc, dtype=np.uint64).copy()
    for b in range(len(inp.qo_indptr) - 1):
        q0, q1 = int(inp.qo_indptr[b]), int(inp.qo_indptr[b + 1])
        for t in range(q1 - q0):
            out[q0 + t] &= ~(np.uint64(1) << np.uint64(t))
    return out


def _tree_block_ref(inp, anc_keys):
    """Oracle (out, lse) over each request's tree keys [L_b, N_b) with masks anc_keys."""
    H = inp.q_latent.shape[1]
    n = int(inp.qo_indptr[-1]) * H
    out = np.zeros((n, 512))
    lse = np.full(n, -np.inf)
    for b in range(len(inp.qo_indptr) - 1):
        q0, q1 = int(inp.qo_indptr[b]), int(inp.qo_indptr[b + 1])
        N = int(inp.kv_indptr[b + 1] - inp.kv_indptr[b])
        L = N - (q1 - q0)
        rows = np.arange(q0 * H, q1 * H, dtype=np.int64)
        m, l, o = oracle.partial_rows(inp, anc_keys, L, N, rows=rows)
        ok = l > 0
        out[rows[ok]] = o[ok] / l[ok, None]
        lse[rows[ok]] = m[ok] + np.log(l[ok])
    return out, lse


@pytest.mark.parametrize("exclude_self,f32", [(True, False), (False, False), (True, True)])
def test_tree_block_matches_oracle(exclude_self, f32):
    inp = generate(custom("treeblock", 71, 16, [300, 0, 1000], [17, 5, 64], 8192))
    anc = product_anc(inp)
    attn = make_attention(inp.workload)
    d = wdev.to_device(inp, anc)
    self_anc = torch.zeros(inp.q_latent.shape[0], dtype=torch.int64, device="cuda")
    out_f32 = torch.full((inp.q_latent.shape[0], 16, 512), 7.0, dtype=torch.float32, device="cuda")
    args = attn.make_args(*wdev.positional(d), lse=d["lse"], visible_count=d["visible_count"])
    attn.tree_block(args, exclude_self, int(self_anc.data_ptr()), torch.cuda.current_stream().cuda_stream,
                    out_f32_ptr=int(out_f32.data_ptr()) if f32 else None)
    torch.cuda.synchronize()
    assert attn.status()[0] == 0
    ref, ref_lse = _tree_block_ref(inp, _strict(anc, inp) if exclude_self else anc)
    res = out_f32 if f32 else d["out"]
    out = res.float().cpu().numpy().astype(np.float64).reshape(-1, 512)
    if f32:   # fp32 accumulation over at most 64 keys: far inside the bf16 bound
        ok = ~np.isinf(ref_lse)
        assert np.abs(out[ok] - ref[ok]).max() <= 1e-4 * max(1.0, np.abs(ref[ok]).max())
    lse = d["lse"].cpu().numpy().astype(np.float64).reshape(-1)
    empty = np.isinf(ref_lse)
    if exclude_self:
        assert empty.any()                                  # the roots attend no strict ancestor
    assert np.all(np.isneginf(lse[empty])) and np.all(out[empty] == 0)
    compare(out[~empty], ref[~empty], lse[~empty], ref_lse[~empty])
    tokens = inp.q_latent.shape[0]
    t_local = np.concatenate([np.arange(int(inp.qo_indptr[b + 1] - inp.qo_indptr[b]))
                              for b in range(len(inp.qo_indptr) - 1)])
    assert np.array_equal(self_anc.cpu().numpy().view(np.uint64), np.uint64(1) << t_local.astype(np.uint64))
    _, _, vis = oracle.verify_rows(inp, oracle.ancestor_masks(inp.parents, inp.qo_indptr),
                                   rows=np.arange(tokens, dtype=np.int64) * inp.q_latent.shape[1])
    assert np.array_equal(d["visible_count"].cpu().numpy(), vis)


@pytest.mark.parametrize("b_f32", [False, True])
def test_merge_states_matches_oracle(b_f32):
    rng = np.random.default_rng(72)
    T, H = 37, 8
    o = [torch.from_numpy(rng.standard_normal((T, H, 512), dtype=np.float32)).to(torch.bfloat16).cuda()
         for _ in range(2)]
    if b_f32:   # an fp32 second state whose values are not bf16-representable
        o[1] = torch.from_numpy(rng.standard_normal((T, H, 512), dtype=np.float32)).cuda()
    lse = [rng.standard_normal((T, H)).astype(np.float32) * 4 for _ in range(2)]
    lse[0][0, :] = -np.inf                                  # one side empty
    lse[1][1, :] = -np.inf
    lse[0][2, :] = lse[1][2, :] = -np.inf                  # both empty
    d_lse = [torch.from_numpy(x).cuda() for x in lse]
    out = torch.empty_like(o[0])
    out_lse = torch.empty((T, H), dtype=torch.float32, device="cuda")
    count = torch.tensor([T - 5], dtype=torch.int32, device="cuda")   # the device count limits the rows
    out.fill_(3.0)
    m = va.VerifyAttnMergeArgs(
        o_a=o[0].data_ptr(), o_a_stride_tok=H * 512, o_a_stride_head=512, lse_a=d_lse[0].data_ptr(),
        o_b=o[1].data_ptr(), o_b_stride_tok=H * 512, o_b_stride_head=512, lse_b=d_lse[1].data_ptr(),
        o_b_f32=int(b_f32),
        out=out.data_ptr(), out_stride_tok=H * 512, out_stride_head=512, lse=out_lse.data_ptr(),
        max_tokens=T, num_tokens=count.data_ptr(), num_heads=H)
    va.verify_attn_merge_states(m, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    n = (T - 5) * H
    ms = np.stack([x.reshape(-1)[:n] for x in lse]).astype(np.float64)
    ls = np.where(np.isneginf(ms), 0.0, 1.0)
    os_ = np.stack([x.float().cpu().numpy().reshape(-1, 512)[:n] for x in o]).astype(np.float64)
    ref, ref_lse = oracle.merge_states(ms, ls, os_)
    got = out.float().cpu().numpy().reshape(-1, 512).astype(np.float64)
    got_lse = out_lse.cpu().numpy().reshape(-1).astype(np.float64)
    assert np.all(got[n:] == 3.0)                           # rows past the device count untouched
    both_empty = np.isneginf(ref_lse)
    assert both_empty.sum() == H
    assert np.all(got[:n][both_empty] == 0) and np.all(np.isneginf(got_lse[:n][both_empty]))
    ok = ~both_empty
    assert np.abs(got[:n][ok] - ref[ok]).max() <= 2 ** -7 * np.abs(ref[ok]).max()
    assert np.abs(got_lse[:n][ok] - ref_lse[ok]).max() <= 1e-4 * max(1.0, np.abs(ref_lse[ok]).max())


@pytest.mark.parametrize("name", ["tiny", "tp8", "ragged_small"])
def test_split_verify_matches_oracle(name):
    if name == "ragged_small":
        inp = generate(custom("sv_ragged", 73, 32, [0, 777, 4000, 12], [3, 64, 9, 1], 16384))
    else:
        inp = generate(WORKLOADS[name])
    anc = product_anc(inp)
    attn = make_attention(inp.workload)
    d = wdev.to_device(inp, anc)
    attn.split_verify(*wdev.positional(d), lse=d["lse"], visible_count=d["visible_count"])
    torch.cuda.synchronize()
    code, bits = attn.status()
    assert code == 0, f"status {code} bits {bits:#x}"
    ref, ref_lse, ref_vis = oracle.verify_rows(inp, oracle.ancestor_masks(inp.parents, inp.qo_indptr))
    out = d["out"].float().cpu().numpy().astype(np.float64).reshape(-1, 512)
    lse = d["lse"].cpu().numpy().astype(np.float64).reshape(-1)
    compare(out, ref, lse, ref_lse)
    H = inp.q_latent.shape[1]
    assert np.array_equal(d["visible_count"].cpu().numpy(), ref_vis[::H])


def test_split_verify_long_sampled_rows():
    inp = generate(WORKLOADS["long"])
    anc = product_anc(inp)
    attn = make_attention(inp.workload)
    d = wdev.to_device(inp, anc)
    attn.split_verify(*wdev.positional(d), lse=d["lse"])
    torch.cuda.synchronize()
    assert attn.status()[0] == 0
    H = inp.q_latent.shape[1]
    rows = np.random.default_rng(74).choice(inp.q_latent.shape[0] * H, 96, replace=False).astype(np.int64)
    rows[:H] = np.arange(H)                                 # all heads of the root
    ref, ref_lse, _ = oracle.verify_rows(inp, oracle.ancestor_masks(inp.parents, inp.qo_indptr), rows=rows)
    out = d["out"].float().cpu().numpy().astype(np.float64).reshape(-1, 512)[rows]
    lse = d["lse"].cpu().numpy().astype(np.float64).reshape(-1)[rows]
    compare(out, ref, lse, ref_lse)
