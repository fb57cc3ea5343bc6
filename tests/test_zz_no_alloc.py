"""GPU test of verify_attn_forward_static, the entry point for callers that
cannot allocate device memory (allocation-free serving loops, runtimes that
own the device heap, plugins handed only their tensors).

It must give the same result as the regular run + reduce pair with a
caller-allocated workspace, on two calls in a row (the library's fixed
workspace keeps the previous call's contents), and it must refuse plans whose
workspace exceeds its fixed size. This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import mla_speculative_verify_absorb_b200 as va
from gpu_common import MAX_ABS, REL_L2, make_attention, product_anc
from workloads import WORKLOADS, custom, generate
from workloads import device as wdev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _check_close(a, b):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(a).all()
    assert np.abs(a - b).max() <= MAX_ABS
    assert np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30) <= REL_L2


@pytest.mark.parametrize("name", ["tiny", "tp8", "batch3", "long"])
def test_static_workspace_matches_allocated_workspace(name):
    wl = WORKLOADS.get(name) or custom("batch3", 41, 16, [0, 300, 1000], [7, 64, 20], 4096)
    inp = generate(wl)
    anc = product_anc(inp)
    attn = make_attention(wl)
    assert attn.ws_bytes <= va.VERIFY_ATTN_STATIC_WS_BYTES

    ref = wdev.to_device(inp, anc)
    attn(*wdev.positional(ref), lse=ref["lse"], visible_count=ref["visible_count"])
    torch.cuda.synchronize()
    assert attn.status()[0] == 0

    d = wdev.to_device(inp, anc)
    status = torch.full((1,), 0xFFFF, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        d["out"].zero_()
        d["lse"].zero_()
        d["visible_count"].zero_()
        args = attn.make_args(*wdev.positional(d), lse=d["lse"], visible_count=d["visible_count"])
        va.verify_attn_forward_static(attn.plan, args, status.data_ptr(), stream)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        _check_close(d["out"], ref["out"])
        assert torch.equal(d["visible_count"], ref["visible_count"])
        assert (d["lse"] - ref["lse"]).abs().max().item() <= 2e-3


def test_static_workspace_rejects_large_plans():
    wl = WORKLOADS["ragged"]
    params = va.VerifyAttnParams(max_batch=wl.batch, num_heads=wl.num_heads, max_tree=max(wl.tree_sizes),
                                 d_latent=512, d_rope=64, num_sms=0, max_kv_per_req=max(wl.kv_lens),
                                 max_total_kv=wl.total_kv, pool_slots=wl.pool_slots, sm_scale=wl.sm_scale)
    plan, ws = va.verify_attn_plan(params)
    assert ws > va.VERIFY_ATTN_STATIC_WS_BYTES
    args = va.VerifyAttnArgs()
    with pytest.raises(va.VerifyAttnError) as e:
        va.verify_attn_forward_static(plan, args, None, 0)
    assert e.value.code == -3
