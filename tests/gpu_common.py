"""Helpers shared by the GPU tests: run the CUDA path through the C ABI and
compare with the oracle. The CUDA side builds its tree masks with the
library's own host helper; the oracle side uses the oracle's."""
from __future__ import annotations

import numpy as np
import torch

import mla_speculative_verify_absorb_b200 as va
import oracle
from workloads import device as wdev

MAX_ABS = 1e-2     # max |out - oracle| for bf16 outputs
REL_L2 = 5e-3      # ||out - oracle||_2 / ||oracle||_2
LSE_ABS = 2e-3     # natural-log LSE, fp32 path vs float64


def product_anc(inp) -> np.ndarray:
    parts = []
    for b in range(len(inp.qo_indptr) - 1):
        q0, q1 = int(inp.qo_indptr[b]), int(inp.qo_indptr[b + 1])
        parts.append(va.verify_attn_build_tree_mask(inp.parents[q0:q1]))
    return np.concatenate(parts)


def make_attention(wl, **over):
    kw = dict(max_batch=wl.batch, num_heads=wl.num_heads, max_tree=max(wl.tree_sizes),
              max_kv_per_req=max(wl.kv_lens), max_total_kv=wl.total_kv, pool_slots=wl.pool_slots,
              sm_scale=wl.sm_scale)
    kw.update(over)
    return va.VerifyAttention(**kw)


def run_gpu(inp, attn=None, anc=None):
    """(out f64 [sumT,H,512], lse f64 [sumT,H], visible int [sumT], anc) from the CUDA path."""
    wl = inp.workload
    attn = attn or make_attention(wl)
    anc = product_anc(inp) if anc is None else anc
    d = wdev.to_device(inp, anc)
    attn(*wdev.positional(d), lse=d["lse"], visible_count=d["visible_count"])
    torch.cuda.synchronize()
    code, bits = attn.status()
    assert code == 0, f"device status {code} bits {bits:#x}"
    out = d["out"].float().cpu().numpy().astype(np.float64)
    lse = d["lse"].cpu().numpy().astype(np.float64)
    vis = d["visible_count"].cpu().numpy()
    return out, lse, vis, anc


def compare(out, ref, lse=None, ref_lse=None):
    assert np.isfinite(out).all()
    err = np.abs(out - ref)
    rel = np.linalg.norm(out - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err.max() <= MAX_ABS, f"max abs err {err.max():.3e}"
    assert rel <= REL_L2, f"rel L2 {rel:.3e}"
    if lse is not None:
        lerr = np.abs(lse - ref_lse)
        assert lerr.max() <= LSE_ABS, f"lse err {lerr.max():.3e}"
    return float(err.max()), float(rel)


def closed_form_counts(inp, anc):
    """L_b + popcount(anc) per token, from the oracle's masks."""
    counts = np.zeros(len(anc), dtype=np.int64)
    for b in range(len(inp.qo_indptr) - 1):
        q0, q1 = int(inp.qo_indptr[b]), int(inp.qo_indptr[b + 1])
        L = int(inp.kv_indptr[b + 1] - inp.kv_indptr[b]) - (q1 - q0)
        for t in range(q0, q1):
            counts[t] = L + bin(int(anc[t])).count("1")
    return counts


def sample_rows(inp, n_per_request: int, seed: int = 0) -> np.ndarray:
    """Query rows (token*H + head) spread over every request, first/last tiles included."""
    rng = np.random.default_rng(seed)
    H = inp.q_latent.shape[1]
    rows = []
    for b in range(len(inp.qo_indptr) - 1):
        q0, q1 = int(inp.qo_indptr[b]), int(inp.qo_indptr[b + 1])
        lo, hi = q0 * H, q1 * H
        pick = {lo, hi - 1, lo + min(127, hi - lo - 1), hi - 1 - min(127, hi - lo - 1)}
        pick.update(int(x) for x in rng.integers(lo, hi, size=n_per_request))
        rows.extend(sorted(pick))
    return np.asarray(rows, dtype=np.int64)


def oracle_all(inp):
    anc = oracle.ancestor_masks(inp.parents, inp.qo_indptr)
    out, lse, vis = oracle.verify_rows(inp, anc)
    H = inp.q_latent.shape[1]
    return anc, out.reshape(-1, H, 512), lse.reshape(-1, H), vis.reshape(-1, H)
