"""verify_attn_gather followed by verify_attn_split is verify_attn_run.

The two halves of the split path are exposed so a caller (and the bench) can
time or schedule them apart; run is defined as exactly that sequence, so the
outputs must be bit-identical, and the result must still match the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import compare, make_attention, product_anc, sample_rows
from workloads import WORKLOADS, generate
from workloads import device as wdev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.mark.parametrize("name", ["tiny", "full_scattered"])
def test_gather_then_split_equals_run(name):
    wl = WORKLOADS[name]
    inp = generate(wl)
    anc = product_anc(inp)
    attn = make_attention(wl)
    s = torch.cuda.current_stream().cuda_stream

    a = wdev.to_device(inp, anc)
    args_a = attn.make_args(*wdev.positional(a), lse=a["lse"], visible_count=a["visible_count"])
    attn.run(args_a, s)
    attn.reduce(args_a, s)
    torch.cuda.synchronize()
    assert attn.status()[0] == 0

    b = wdev.to_device(inp, anc)
    args_b = attn.make_args(*wdev.positional(b), lse=b["lse"], visible_count=b["visible_count"])
    attn.gather(args_b, s)
    attn.split(args_b, s)
    attn.reduce(args_b, s)
    torch.cuda.synchronize()
    assert attn.status()[0] == 0

    assert torch.equal(a["out"], b["out"])
    assert torch.equal(a["lse"], b["lse"])
    assert torch.equal(a["visible_count"], b["visible_count"])

    ref_anc = oracle.ancestor_masks(inp.parents, inp.qo_indptr)
    rows = sample_rows(inp, 16, seed=11)
    ref, ref_lse, _ = oracle.verify_rows(inp, ref_anc, rows=rows)
    out = b["out"].float().cpu().numpy().astype(np.float64).reshape(-1, 512)[rows]
    lse = b["lse"].cpu().numpy().astype(np.float64).reshape(-1)[rows]
    compare(out, ref, lse, ref_lse)
