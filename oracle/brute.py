"""Dense numpy brute force of the verify attention -- TEST INFRASTRUCTURE.

A second, independently written statement of the same definition as
``mla_verify_oracle.c`` for tiny inputs only: it builds the whole boolean
visibility matrix of a request from the parent array (walking parents, not
from bitmasks), forms every score with one einsum over the 576-wide
concatenation, masks with -inf, and normalises with an explicit
exp / sum. Used as the "brute force" pin of the C oracle.
"""
from __future__ import annotations

import numpy as np


def _f64(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def visibility(parents, prefix_len: int) -> np.ndarray:
    """bool [T, L+T]: row t marks the KV positions tree node t may attend."""
    T = len(parents)
    vis = np.zeros((T, prefix_len + T), dtype=bool)
    vis[:, :prefix_len] = True
    for t in range(T):
        node = t
        while node != -1:
            vis[t, prefix_len + node] = True
            node = int(parents[node])
    return vis


def verify(inp):
    """(out [sumT, H, 512], lse [sumT, H]) in float64 for every query."""
    H = inp.q_latent.shape[1]
    q = np.concatenate([_f64(inp.q_latent), _f64(inp.q_rope)], axis=-1)      # [sumT, H, 576]
    out = np.zeros(inp.q_latent.shape, dtype=np.float64)
    lse = np.zeros((inp.q_latent.shape[0], H), dtype=np.float64)
    for b in range(len(inp.qo_indptr) - 1):
        q0, q1 = int(inp.qo_indptr[b]), int(inp.qo_indptr[b + 1])
        k0, k1 = int(inp.kv_indptr[b]), int(inp.kv_indptr[b + 1])
        T, N = q1 - q0, k1 - k0
        rows = _f64(inp.kv_pool[inp.kv_indices[k0:k1]])                      # [N, 576]
        scores = inp.sm_scale * np.einsum("thd,nd->thn", q[q0:q1], rows)      # [T, H, N]
        vis = visibility(inp.parents[q0:q1], N - T)                            # [T, N]
        scores = np.where(vis[:, None, :], scores, -np.inf)
        mx = scores.max(axis=-1, keepdims=True)
        w = np.exp(scores - mx)
        denom = w.sum(axis=-1, keepdims=True)
        out[q0:q1] = np.einsum("thn,nd->thd", w / denom, rows[:, :512])
        lse[q0:q1] = (mx + np.log(denom))[..., 0]
    return out, lse
