"""Seeded synthetic inputs for MLA-absorb tree-verify attention.

This module only draws numbers and lays them out. It holds none of the
attention arithmetic, builds no tree mask and computes nothing that either
the CPU oracle (``oracle/``) or the CUDA path computes: both sides receive the
same bytes from here and derive everything else with their own code.

Workload shapes follow the problem statement of the pages ("The Execution
Phase: From Plan to 3-6x Decode Speedup on Blackwell Consumer GPUs", section
"The Transition: From Planning to Execution": MLA-absorb attention with a
custom tree mask; page "The Architecture Detective", section "The Context: A
Bottleneck Confirmed": page_size=1 KV, non-contiguous tree tokens). The
concrete dimensions (q_latent 512 + q_rope 64 per head, c_kv 512 + k_rope 64
per token, bf16, page_size=1 pool addressed through kv_indices, one uint64
ancestor-or-self bitmask per query) are the workload's given constants.

Draw recipe (numpy ``default_rng(seed)``, PCG64), in this order:

1. per request, the tree parents: fixed lists are taken as given; a random
   tree draws ``parent[i]`` uniformly from the earlier nodes whose depth is
   below the cap (root depth 1), or from all earlier nodes without a cap;
2. for scattered layouts, one permutation of all pool slots; request b takes
   the next ``N_b = L_b + T_b`` entries (prefix positions first, then tree
   nodes in node order); contiguous layouts use slots ``0..N-1`` in order;
3. q_latent ``[sumT, H, 512]`` then q_rope ``[sumT, H, 64]`` as float32
   N(0,1), times ``q_scale``, rounded to bf16 (round-to-nearest-even);
4. the referenced latent rows ``[sum N_b, 576]`` in kv order as float32 N(0,1)
   rounded to bf16, written to ``pool[kv_indices]``.

Pool slots no request references hold a bf16 NaN so that a wrong gather
poisons the output instead of passing silently.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np

D_LATENT = 512
D_ROPE = 64
D_QK = D_LATENT + D_ROPE
BF16_NAN = np.uint16(0x7FC0)
DEFAULT_SCALE = 192.0 ** -0.5


@dataclass(frozen=True)
class Workload:
    """One synthetic verify call: per-request prefixes and tree sizes."""

    name: str
    seed: int
    num_heads: int
    prefixes: tuple
    tree_sizes: tuple
    pool_slots: int
    layout: str = "scattered"          # "scattered" | "contiguous"
    max_depth: Optional[int] = None    # depth cap counted in nodes (root = 1)
    fixed_parents: Optional[tuple] = None  # one tuple for all requests, or one per request
    q_scale: float = 1.0
    sm_scale: float = DEFAULT_SCALE

    @property
    def batch(self) -> int:
        return len(self.prefixes)

    @property
    def kv_lens(self) -> list:
        return [int(l) + int(t) for l, t in zip(self.prefixes, self.tree_sizes)]

    @property
    def total_kv(self) -> int:
        return sum(self.kv_lens)

    @property
    def total_q(self) -> int:
        return sum(int(t) for t in self.tree_sizes)


def _wl(name, seed, H, prefixes, trees, pool, **kw) -> Workload:
    return Workload(name=name, seed=seed, num_heads=H, prefixes=tuple(prefixes),
                    tree_sizes=tuple(trees), pool_slots=pool, **kw)


#: The five workloads of the problem statement, by name.
WORKLOADS = {
    # 1 request, H=8, T=4 fixed tree, L=256, pool 4096, scattered slots.
    "tiny": _wl("tiny", 1, 8, [256], [4], 4096, fixed_parents=(-1, 0, 0, 1)),
    # Per-rank slice of a 64-head model under 8-way tensor parallelism.
    "tp8": _wl("tp8", 2, 8, [4096], [16], 65536, max_depth=8),
    # All 64 heads on one GPU, contiguous and scattered slot lists; q scaled by 0.5.
    "full_contiguous": _wl("full_contiguous", 3, 64, [16384], [32], 262144,
                           layout="contiguous", q_scale=0.5),
    "full_scattered": _wl("full_scattered", 3, 64, [16384], [32], 262144,
                          layout="scattered", q_scale=0.5),
    # 65k-token prefix, T=64 tree of depth <= 16; the graph-captured call.
    "long": _wl("long", 4, 64, [65536], [64], 262144, max_depth=16),
    # 4 requests sharing one pool, interleaved scattered slots.
    "ragged": _wl("ragged", 5, 64, [8192, 32768, 131072, 200000], [32] * 4, 400000),
}


def random_parents(rng: np.random.Generator, T: int, max_depth: Optional[int]) -> np.ndarray:
    """Draw a random tree over T nodes: node 0 is the root (parent -1)."""
    parents = np.full(T, -1, dtype=np.int32)
    depth = [1]
    for i in range(1, T):
        cand = [j for j in range(i) if max_depth is None or depth[j] < max_depth]
        p = cand[int(rng.integers(len(cand)))]
        parents[i] = p
        depth.append(depth[p] + 1)
    return parents


def _to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern, round to nearest even (inputs are finite)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


@dataclass
class Inputs:
    """Host arrays of one verify call (bf16 values held as uint16 bit patterns)."""

    workload: Workload
    q_latent: np.ndarray      # uint16 [sumT, H, 512]
    q_rope: np.ndarray        # uint16 [sumT, H, 64]
    kv_pool: np.ndarray       # uint16 [pool_slots, 576]
    kv_indices: np.ndarray    # int32 [sum N_b]
    kv_indptr: np.ndarray     # int32 [B+1]
    qo_indptr: np.ndarray     # int32 [B+1]
    parents: np.ndarray       # int32 [sumT], request-local node ids, root -1
    sm_scale: float = DEFAULT_SCALE
    extra: dict = field(default_factory=dict)


def generate(wl: Workload, rows_chunk: int = 65536) -> Inputs:
    """Materialise a workload with the draw recipe in the module docstring."""
    rng = np.random.default_rng(wl.seed)
    B, H = wl.batch, wl.num_heads
    parents = []
    for b in range(B):
        T = int(wl.tree_sizes[b])
        if wl.fixed_parents is not None:
            fp = wl.fixed_parents
            per_request = len(fp) > 0 and isinstance(fp[0], (tuple, list))
            p = np.asarray(fp[b] if per_request else fp, dtype=np.int32)
            if p.shape[0] != T:
                raise ValueError("fixed parents do not match the tree size")
        else:
            p = random_parents(rng, T, wl.max_depth)
        parents.append(p)
    parents = np.concatenate(parents).astype(np.int32)

    kv_lens = wl.kv_lens
    total_kv = sum(kv_lens)
    if total_kv > wl.pool_slots:
        raise ValueError("pool too small for the workload")
    if wl.layout == "scattered":
        perm = rng.permutation(wl.pool_slots).astype(np.int32)
        kv_indices = perm[:total_kv].copy()
    elif wl.layout == "contiguous":
        kv_indices = np.arange(total_kv, dtype=np.int32)
    else:
        raise ValueError(wl.layout)
    kv_indptr = np.zeros(B + 1, dtype=np.int32)
    kv_indptr[1:] = np.cumsum(kv_lens)
    qo_indptr = np.zeros(B + 1, dtype=np.int32)
    qo_indptr[1:] = np.cumsum([int(t) for t in wl.tree_sizes])
    sum_t = int(qo_indptr[-1])

    q_lat = _to_bf16_bits(rng.standard_normal((sum_t, H, D_LATENT), dtype=np.float32) * np.float32(wl.q_scale))
    q_rope = _to_bf16_bits(rng.standard_normal((sum_t, H, D_ROPE), dtype=np.float32) * np.float32(wl.q_scale))

    pool = np.full((wl.pool_slots, D_QK), BF16_NAN, dtype=np.uint16)
    for start in range(0, total_kv, rows_chunk):
        stop = min(total_kv, start + rows_chunk)
        rows = rng.standard_normal((stop - start, D_QK), dtype=np.float32)
        pool[kv_indices[start:stop]] = _to_bf16_bits(rows)

    return Inputs(workload=wl, q_latent=q_lat, q_rope=q_rope, kv_pool=pool,
                  kv_indices=kv_indices, kv_indptr=kv_indptr, qo_indptr=qo_indptr,
                  parents=parents, sm_scale=wl.sm_scale)


def custom(name: str, seed: int, num_heads: int, prefixes: Sequence[int], tree_sizes: Sequence[int],
           pool_slots: int, **kw) -> Workload:
    """A workload with explicit shapes (used for edge cases and small parity runs)."""
    return _wl(name, seed, num_heads, list(prefixes), list(tree_sizes), pool_slots, **kw)
