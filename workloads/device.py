"""Copy a generated workload to the GPU as torch tensors (plumbing only).

No attention arithmetic and no tree-mask construction happens here: the
caller supplies the ancestor masks from whichever side it exercises.
"""
from __future__ import annotations

import numpy as np
import torch


def to_device(inp, anc: np.ndarray, device="cuda", pinned: bool = False):
    """Device tensors of one call plus an empty bf16 output, lse and counts."""
    def up(a, dtype=None):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if dtype is not None:
            t = t.view(dtype)
        if pinned:
            t = t.pin_memory()
        return t.to(device, non_blocking=pinned)

    H = inp.q_latent.shape[1]
    sum_t = inp.q_latent.shape[0]
    d = {
        "q_latent": up(inp.q_latent.view(np.int16), torch.bfloat16),
        "q_rope": up(inp.q_rope.view(np.int16), torch.bfloat16),
        "kv_pool": up(inp.kv_pool.view(np.int16), torch.bfloat16),
        "kv_indices": up(inp.kv_indices.astype(np.int32)),
        "kv_indptr": up(inp.kv_indptr.astype(np.int32)),
        "qo_indptr": up(inp.qo_indptr.astype(np.int32)),
        "tree_anc": up(np.asarray(anc, dtype=np.uint64).view(np.int64)),
    }
    d["out"] = torch.empty((sum_t, H, 512), dtype=torch.bfloat16, device=device)
    d["lse"] = torch.empty((sum_t, H), dtype=torch.float32, device=device)
    d["visible_count"] = torch.empty((sum_t,), dtype=torch.int32, device=device)
    return d


def positional(d):
    """Tensors in the order VerifyAttention expects."""
    return (d["q_latent"], d["q_rope"], d["kv_pool"], d["kv_indices"], d["kv_indptr"], d["qo_indptr"],
            d["tree_anc"], d["out"])
