"""KV-sequence sharding of one verify call across ranks (one process per GPU).

Each of R ranks attends a disjoint part of every query row's visible keys and
returns its state (o_r, lse_r); the states are gathered along a leading axis
over ``torch.distributed`` (NCCL on GPUs) and merged by the library's stacked
LSE merge (page "The Breakthrough", section "The Message in Context":
KV-split partial results combined by a reduce; page "The Architecture
Detective", section "The Split Verify Design": LSE merge of disjoint key
sets).

Partition of one request with prefix L and tree T (``shard_ranges``): the
prefix is cut into R' = min(R, max(1, L // T)) near-equal chunks, so that
every chunk has at least T keys. Ranks 0 .. R'-2 take the first R'-1 chunks
with every key visible; rank R-1 takes the last chunk plus the tree block
under the request's ancestor masks; any other rank holds an empty state
(lse = -inf). A rank's chunk runs through the library's own attention call
as a one-request call of N' = chunk keys whose last T keys take the mask
(1 << T) - 1, i.e. all visible: a dense pass.

Everything here is argument marshalling and ``torch.distributed`` plumbing;
the attention, the reduce and the merge run in the CUDA library.
"""
from __future__ import annotations

from typing import List, Tuple

from ._binding import (VERIFY_ATTN_D_LATENT, VerifyAttention, VerifyAttnError, VerifyAttnMergeStackedArgs,
                       verify_attn_merge_stacked)


def shard_ranges(L: int, T: int, R: int) -> List[Tuple[int, int]]:
    """KV position ranges [lo, hi) of ranks 0..R-1 for one request (prefix L, tree T)."""
    if L < 0 or T < 1 or R < 1:
        raise ValueError("need L >= 0, T >= 1, R >= 1")
    active = min(R, max(1, L // T))
    cuts = [i * L // active for i in range(active + 1)]
    ranges = [(0, 0)] * R
    for i in range(active - 1):
        ranges[i] = (cuts[i], cuts[i + 1])
    ranges[R - 1] = (cuts[active - 1], L + T)
    return ranges


def max_shard_keys(max_prefix: int, max_tree: int, R: int) -> int:
    """Upper bound of hi - lo over every L <= max_prefix and T <= max_tree:
    a chunk has at most ceil(max_prefix / R) keys when all R ranks are
    active and fewer than 2 T otherwise; the last rank adds the tree."""
    return max(-(-max_prefix // R), 2 * max_tree) + max_tree


def gather_states(o_local, lse_local, o_all, lse_all, group=None):
    """Gather every rank's (o, lse) into [R, ...] buffers, rank-major."""
    import torch.distributed as dist

    dist.all_gather_into_tensor(o_all.reshape(-1), o_local.reshape(-1), group=group)
    dist.all_gather_into_tensor(lse_all.reshape(-1), lse_local.reshape(-1), group=group)


class ShardedVerify:
    """One request's verify attention with its KV split over ``world`` ranks.

    ``local_state(rank, ...)`` computes one rank's state; ``merge`` combines
    stacked states; ``__call__`` does both with the exchange in between (the
    rank comes from the process group). One plan, sized for the longest
    shard, serves every rank. Small per-shape tensors (shard lengths, dense
    masks) are created on first use and reused, so repeated calls of one
    shape launch only library kernels and the two all-gathers.
    """

    def __init__(self, *, world: int, num_heads: int, max_tree: int, max_prefix: int, pool_slots: int,
                 sm_scale: float, device=None):
        import torch

        self.world = int(world)
        self.device = torch.device("cuda") if device is None else torch.device(device)
        keys = max_shard_keys(max_prefix, max_tree, self.world)
        self.attn = VerifyAttention(max_batch=1, num_heads=num_heads, max_tree=max_tree, max_kv_per_req=keys,
                                    max_total_kv=keys, pool_slots=pool_slots, sm_scale=sm_scale, device=self.device)
        self.num_heads = num_heads
        self.max_tree = max_tree
        H, D = num_heads, VERIFY_ATTN_D_LATENT
        self._shape_cache = {}
        self._o_local = torch.empty((max_tree, H, D), dtype=torch.bfloat16, device=self.device)
        self._lse_local = torch.empty((max_tree, H), dtype=torch.float32, device=self.device)
        self._o_empty = torch.zeros((max_tree, H, D), dtype=torch.bfloat16, device=self.device)
        self._lse_empty = torch.full((max_tree, H), float("-inf"), dtype=torch.float32, device=self.device)
        self._o_all = torch.empty((self.world * max_tree * H * D,), dtype=torch.bfloat16, device=self.device)
        self._lse_all = torch.empty((self.world * max_tree * H,), dtype=torch.float32, device=self.device)

    def _shape(self, n_keys: int, T: int):
        """Device tensors kv_indptr = [0, n_keys], qo_indptr = [0, T], dense masks (1 << T) - 1."""
        import torch

        key = (n_keys, T)
        if key not in self._shape_cache:
            self._shape_cache[key] = (
                torch.tensor([0, n_keys], dtype=torch.int32, device=self.device),
                torch.tensor([0, T], dtype=torch.int32, device=self.device),
                torch.full((T,), ((1 << T) - 1) if T < 64 else -1, dtype=torch.int64, device=self.device),
            )
        return self._shape_cache[key]

    def local_state(self, rank: int, q_latent, q_rope, kv_pool, kv_indices, tree_anc, o, lse, stream: int) -> bool:
        """State of `rank` over its shard into o (bf16 [T, H, 512]) and lse
        (fp32 [T, H]); returns False, writing nothing, for an empty shard."""
        T = int(q_latent.shape[0])
        N = int(kv_indices.shape[0])
        lo, hi = shard_ranges(N - T, T, self.world)[rank]
        if hi == lo:
            return False
        kv_indptr, qo_indptr, dense = self._shape(hi - lo, T)
        anc = tree_anc if rank == self.world - 1 else dense
        args = self.attn.make_args(q_latent, q_rope, kv_pool, kv_indices[lo:hi], kv_indptr, qo_indptr, anc, o,
                                   lse=lse)
        self.attn.run(args, stream)
        self.attn.reduce(args, stream)
        return True

    def merge(self, o_all, lse_all, out, lse=None, stream: int = 0):
        """Merge stacked states o_all [R, T, H, 512], lse_all [R, T, H] into out (and lse)."""
        args = VerifyAttnMergeStackedArgs(
            o=int(o_all.data_ptr()), lse_states=int(lse_all.data_ptr()), num_states=int(o_all.shape[0]),
            num_heads=self.num_heads, out=int(out.data_ptr()), out_stride_tok=out.stride(0),
            out_stride_head=out.stride(1), lse=None if lse is None else int(lse.data_ptr()),
            max_tokens=int(o_all.shape[1]), num_tokens=None)
        verify_attn_merge_stacked(args, stream)

    def stacked(self, T: int):
        """Views [R, T, H, 512] and [R, T, H] of the exchange buffers."""
        H, D = self.num_heads, VERIFY_ATTN_D_LATENT
        return (self._o_all[: self.world * T * H * D].view(self.world, T, H, D),
                self._lse_all[: self.world * T * H].view(self.world, T, H))

    def __call__(self, q_latent, q_rope, kv_pool, kv_indices, tree_anc, out, lse=None, group=None, stream=None):
        """This rank's share of the call, the exchange and the merge; every
        rank ends with the whole output."""
        import torch
        import torch.distributed as dist

        rank = dist.get_rank(group)
        if dist.get_world_size(group) != self.world:
            raise VerifyAttnError(-1, "ShardedVerify: process group size differs from the plan")
        T = int(q_latent.shape[0])
        if T > self.max_tree:
            raise VerifyAttnError(-1, "ShardedVerify: tree larger than the plan")
        s = torch.cuda.current_stream(self.device).cuda_stream if stream is None else stream
        o_local, lse_local = self._o_local[:T], self._lse_local[:T]
        if not self.local_state(rank, q_latent, q_rope, kv_pool, kv_indices, tree_anc, o_local, lse_local, s):
            o_local, lse_local = self._o_empty[:T], self._lse_empty[:T]
        o_all, lse_all = self.stacked(T)
        gather_states(o_local, lse_local, o_all, lse_all, group)
        self.merge(o_all, lse_all, out, lse, s)
        return out
