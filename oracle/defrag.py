"""CPU oracle for the KV relocation (defragmentation) step -- TEST INFRASTRUCTURE.

Only ``tests/`` and ``bench.py``'s CPU leg may import this module; the CUDA
library never does.

Definition (page "The Execution Phase", section "Tier 0 KV Defragmentation":
Tier 1 is live relocation of a request's fragmented page_size=1 slots into
contiguous ones under a copy budget; the pages give no algorithm, so this
states the plainest one): for every request b with KV positions
[kv_indptr[b], kv_indptr[b+1]) and n_b = min(N_b, budget), position j < n_b
moves to slot dst_begin[b] + j: the 576-wide latent row is copied there
(unless it is already there) and kv_indices is rewritten to that slot.
Positions j >= n_b, other requests' rows and all other slots are untouched.
The caller guarantees that a destination run holds no slot that any position
still references elsewhere.
"""
from __future__ import annotations

import numpy as np

D_QK = 576


def defrag(pool: np.ndarray, kv_indices: np.ndarray, kv_indptr: np.ndarray, dst_begin: np.ndarray,
           budget: int):
    """Return (new_pool, new_kv_indices); inputs are not modified.

    pool: uint16 [pool_slots, >= 576] (bf16 bit patterns); kv_indices int32.
    """
    pool = pool.copy()
    idx = np.asarray(kv_indices, dtype=np.int32).copy()
    src_pool = pool.copy()          # every copy reads the rows as they were before the call
    for b in range(len(kv_indptr) - 1):
        k0, k1 = int(kv_indptr[b]), int(kv_indptr[b + 1])
        n = min(k1 - k0, int(budget))
        for j in range(n):
            src, dst = int(idx[k0 + j]), int(dst_begin[b]) + j
            if src != dst:
                pool[dst, :D_QK] = src_pool[src, :D_QK]
            idx[k0 + j] = dst
    return pool, idx
