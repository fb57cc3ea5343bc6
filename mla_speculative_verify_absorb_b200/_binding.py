"""ctypes binding of ``include/verify_attn.h`` -- argument marshalling only.

Every function here has the same name and meaning as its C counterpart; the
C header documents layouts, ownership and error codes. ``VerifyAttention``
is a convenience holder for a plan plus a torch-allocated workspace that
fills ``verify_attn_args`` from torch tensors (device pointers and element
strides) and calls ``verify_attn_run`` then ``verify_attn_reduce``.
"""
from __future__ import annotations

import ctypes
import threading

import numpy as np

from . import build as _build

VERIFY_ATTN_D_LATENT = 512
VERIFY_ATTN_D_ROPE = 64
VERIFY_ATTN_MAX_TREE = 64
VERIFY_ATTN_STATIC_WS_BYTES = 128 << 20

_i32, _i64, _u32, _f32, _vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_float, ctypes.c_void_p


class VerifyAttnParams(ctypes.Structure):
    _fields_ = [
        ("max_batch", _i32), ("num_heads", _i32), ("max_tree", _i32), ("d_latent", _i32), ("d_rope", _i32),
        ("num_sms", _i32), ("max_kv_per_req", _i64), ("max_total_kv", _i64), ("pool_slots", _i64),
        ("sm_scale", _f32), ("reserved", _i32),
    ]


class VerifyAttnPlan(ctypes.Structure):
    _fields_ = [
        ("version", _i32), ("num_heads", _i32), ("max_batch", _i32), ("max_tree", _i32),
        ("max_kv_per_req", _i64), ("max_total_kv", _i64), ("pool_slots", _i64), ("sm_scale", _f32),
        ("num_clusters", _i32), ("rows_per_tile", _i32), ("keys_per_tile", _i32), ("row_tiles_per_req", _i32),
        ("num_slots", _i32), ("ws_meta_offset", _i64), ("ws_partial_offset", _i64), ("ws_bytes", _i64),
        ("split_smem_bytes", _i32), ("reserved0", _i32), ("ws_stage_offset", _i64), ("stage_rows", _i64),
        ("reserved", _i32 * 2),
    ]


class VerifyAttnArgs(ctypes.Structure):
    _fields_ = [
        ("q_latent", _vp), ("q_latent_stride_tok", _i64), ("q_latent_stride_head", _i64),
        ("q_rope", _vp), ("q_rope_stride_tok", _i64), ("q_rope_stride_head", _i64),
        ("kv_pool", _vp), ("kv_row_stride", _i64),
        ("kv_indices", _vp), ("kv_indptr", _vp), ("qo_indptr", _vp), ("tree_anc", _vp),
        ("batch", _i32), ("reserved0", _i32),
        ("out", _vp), ("out_stride_tok", _i64), ("out_stride_head", _i64),
        ("lse", _vp), ("visible_count", _vp),
    ]


class VerifyAttnDefragArgs(ctypes.Structure):
    _fields_ = [
        ("kv_pool", _vp), ("kv_row_stride", _i64), ("pool_slots", _i64), ("kv_indices", _vp), ("kv_indptr", _vp),
        ("dst_begin", _vp), ("batch", _i32), ("budget", _i32), ("max_total_kv", _i64), ("status", _vp),
    ]


class VerifyAttnMergeArgs(ctypes.Structure):
    _fields_ = [
        ("o_a", _vp), ("o_a_stride_tok", _i64), ("o_a_stride_head", _i64), ("lse_a", _vp),
        ("o_b", _vp), ("o_b_stride_tok", _i64), ("o_b_stride_head", _i64), ("lse_b", _vp), ("o_b_f32", _i32),
        ("out", _vp), ("out_stride_tok", _i64), ("out_stride_head", _i64), ("lse", _vp),
        ("max_tokens", _i64), ("num_tokens", _vp), ("num_heads", _i32),
    ]


class VerifyAttnMergeStackedArgs(ctypes.Structure):
    _fields_ = [
        ("o", _vp), ("lse_states", _vp), ("num_states", _i32), ("num_heads", _i32), ("out", _vp),
        ("out_stride_tok", _i64), ("out_stride_head", _i64), ("lse", _vp), ("max_tokens", _i64),
        ("num_tokens", _vp),
    ]


class VerifyAttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {verify_attn_strerror(code)} (code {code})")


_lock = threading.Lock()
_lib = None

EXPORTS = (
    "verify_attn_plan", "verify_attn_workspace_init", "verify_attn_run", "verify_attn_gather", "verify_attn_split",
    "verify_attn_reduce",
    "verify_attn_build_tree_mask", "verify_attn_build_tree_mask_device", "verify_attn_status",
    "verify_attn_forward_static", "verify_attn_defrag", "verify_attn_tree_block", "verify_attn_merge_states",
    "verify_attn_merge_stacked", "verify_attn_strerror",
)


def lib_path() -> str:
    return _build.LIB_PATH


def load_library():
    """Build (if missing or stale) and load the CUDA library; raises on failure."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            lib = ctypes.CDLL(path)
            P = ctypes.POINTER
            lib.verify_attn_plan.argtypes = [P(VerifyAttnParams), P(VerifyAttnPlan), P(ctypes.c_size_t)]
            lib.verify_attn_workspace_init.argtypes = [P(VerifyAttnPlan), _vp, ctypes.c_size_t, _vp]
            lib.verify_attn_run.argtypes = [P(VerifyAttnPlan), P(VerifyAttnArgs), _vp, ctypes.c_size_t, _vp]
            lib.verify_attn_gather.argtypes = [P(VerifyAttnPlan), P(VerifyAttnArgs), _vp, ctypes.c_size_t, _vp]
            lib.verify_attn_split.argtypes = [P(VerifyAttnPlan), P(VerifyAttnArgs), _vp, ctypes.c_size_t, _vp]
            lib.verify_attn_reduce.argtypes = [P(VerifyAttnPlan), P(VerifyAttnArgs), _vp, ctypes.c_size_t, _vp]
            lib.verify_attn_build_tree_mask.argtypes = [_vp, _i32, _vp]
            lib.verify_attn_build_tree_mask_device.argtypes = [_vp, _vp, _i32, _vp, _vp, _vp]
            lib.verify_attn_status.argtypes = [_vp, _vp, P(_u32)]
            lib.verify_attn_forward_static.argtypes = [P(VerifyAttnPlan), P(VerifyAttnArgs), _vp, _vp]
            lib.verify_attn_defrag.argtypes = [P(VerifyAttnDefragArgs), _vp]
            lib.verify_attn_tree_block.argtypes = [P(VerifyAttnPlan), P(VerifyAttnArgs), ctypes.c_int, _vp, _vp,
                                                   _vp, ctypes.c_size_t, _vp]
            lib.verify_attn_merge_states.argtypes = [P(VerifyAttnMergeArgs), _vp]
            lib.verify_attn_merge_stacked.argtypes = [P(VerifyAttnMergeStackedArgs), _vp]
            lib.verify_attn_strerror.argtypes = [ctypes.c_int]
            lib.verify_attn_strerror.restype = ctypes.c_char_p
            for name in EXPORTS[:-1]:
                getattr(lib, name).restype = ctypes.c_int
            _lib = lib
    return _lib


def verify_attn_strerror(code: int) -> str:
    return load_library().verify_attn_strerror(int(code)).decode()


def _check(code: int, where: str):
    if code != 0:
        raise VerifyAttnError(code, where)


def verify_attn_plan(params: VerifyAttnParams):
    """Return (plan, workspace bytes)."""
    plan = VerifyAttnPlan()
    nbytes = ctypes.c_size_t(0)
    _check(load_library().verify_attn_plan(ctypes.byref(params), ctypes.byref(plan), ctypes.byref(nbytes)),
           "verify_attn_plan")
    return plan, int(nbytes.value)


def verify_attn_workspace_init(plan, ws_ptr: int, ws_bytes: int, stream: int = 0):
    _check(load_library().verify_attn_workspace_init(ctypes.byref(plan), ws_ptr, ws_bytes, stream),
           "verify_attn_workspace_init")


def verify_attn_run(plan, args: VerifyAttnArgs, ws_ptr: int, ws_bytes: int, stream: int = 0):
    _check(load_library().verify_attn_run(ctypes.byref(plan), ctypes.byref(args), ws_ptr, ws_bytes, stream),
           "verify_attn_run")


def verify_attn_gather(plan, args: VerifyAttnArgs, ws_ptr: int, ws_bytes: int, stream: int = 0):
    _check(load_library().verify_attn_gather(ctypes.byref(plan), ctypes.byref(args), ws_ptr, ws_bytes, stream),
           "verify_attn_gather")


def verify_attn_split(plan, args: VerifyAttnArgs, ws_ptr: int, ws_bytes: int, stream: int = 0):
    _check(load_library().verify_attn_split(ctypes.byref(plan), ctypes.byref(args), ws_ptr, ws_bytes, stream),
           "verify_attn_split")


def verify_attn_reduce(plan, args: VerifyAttnArgs, ws_ptr: int, ws_bytes: int, stream: int = 0):
    _check(load_library().verify_attn_reduce(ctypes.byref(plan), ctypes.byref(args), ws_ptr, ws_bytes, stream),
           "verify_attn_reduce")


def verify_attn_forward_static(plan, args: VerifyAttnArgs, status_ptr=None, stream: int = 0):
    """Split + reduce with the library's own fixed workspace (no allocation)."""
    _check(load_library().verify_attn_forward_static(ctypes.byref(plan), ctypes.byref(args), status_ptr, stream),
           "verify_attn_forward_static")


def verify_attn_build_tree_mask(parents) -> np.ndarray:
    """uint64 ancestor-or-self masks of one tree (host helper)."""
    p = np.ascontiguousarray(parents, dtype=np.int32)
    anc = np.zeros(p.shape[0], dtype=np.uint64)
    _check(load_library().verify_attn_build_tree_mask(p.ctypes.data, int(p.shape[0]), anc.ctypes.data),
           "verify_attn_build_tree_mask")
    return anc


def verify_attn_build_tree_mask_device(parents_ptr: int, qo_indptr_ptr: int, batch: int, anc_ptr: int,
                                       status_ptr=None, stream: int = 0):
    """Ancestor masks of a batch of trees on the device (asynchronous)."""
    _check(load_library().verify_attn_build_tree_mask_device(parents_ptr, qo_indptr_ptr, int(batch), anc_ptr,
                                                             status_ptr, stream), "verify_attn_build_tree_mask_device")


def verify_attn_defrag(args: VerifyAttnDefragArgs, stream: int = 0):
    """Relocate each request's leading KV positions into its destination run (asynchronous)."""
    _check(load_library().verify_attn_defrag(ctypes.byref(args), stream), "verify_attn_defrag")


def verify_attn_tree_block(plan, args: VerifyAttnArgs, exclude_self: bool, self_anc_ptr, out_f32_ptr, ws_ptr: int,
                           ws_bytes: int, stream: int = 0):
    """Masked tree-block attention of the split-verify variant (asynchronous)."""
    _check(load_library().verify_attn_tree_block(ctypes.byref(plan), ctypes.byref(args), int(bool(exclude_self)),
                                                 self_anc_ptr, out_f32_ptr, ws_ptr, ws_bytes, stream),
           "verify_attn_tree_block")


def verify_attn_merge_states(args: VerifyAttnMergeArgs, stream: int = 0):
    """Two-state LSE merge (asynchronous)."""
    _check(load_library().verify_attn_merge_states(ctypes.byref(args), stream), "verify_attn_merge_states")


def verify_attn_merge_stacked(args: VerifyAttnMergeStackedArgs, stream: int = 0):
    """Stacked R-state LSE merge (asynchronous)."""
    _check(load_library().verify_attn_merge_stacked(ctypes.byref(args), stream), "verify_attn_merge_stacked")


def verify_attn_status(ws_ptr: int, stream: int = 0):
    """(code, raw status bits) of a workspace; synchronises `stream`."""
    detail = _u32(0)
    code = load_library().verify_attn_status(ws_ptr, stream, ctypes.byref(detail))
    return int(code), int(detail.value)


# ----------------------------------------------------------------------------- torch convenience

def _ptr(t):
    return None if t is None else int(t.data_ptr())


def defrag(kv_pool, kv_indices, kv_indptr, dst_begin, budget: int, status=None, max_total_kv=None, stream=None):
    """Relocate KV rows with device tensors: kv_pool bf16 [slots, >=576] and kv_indices int32 are
    rewritten in place; kv_indptr / dst_begin int32; status an optional uint32/int32 device word."""
    import torch

    s = torch.cuda.current_stream(kv_pool.device).cuda_stream if stream is None else stream
    args = VerifyAttnDefragArgs(
        kv_pool=_ptr(kv_pool), kv_row_stride=kv_pool.stride(0), pool_slots=kv_pool.shape[0],
        kv_indices=_ptr(kv_indices), kv_indptr=_ptr(kv_indptr), dst_begin=_ptr(dst_begin),
        batch=int(kv_indptr.shape[0]) - 1, budget=int(budget),
        max_total_kv=int(kv_indices.shape[0]) if max_total_kv is None else int(max_total_kv),
        status=_ptr(status))
    verify_attn_defrag(args, s)
    return args


class VerifyAttention:
    """A plan plus its workspace; call with device tensors to run split + reduce."""

    def __init__(self, *, max_batch: int, num_heads: int, max_tree: int, max_kv_per_req: int,
                 max_total_kv: int, pool_slots: int, sm_scale: float, device=None, num_sms: int = 0):
        import torch

        self.params = VerifyAttnParams(max_batch=max_batch, num_heads=num_heads, max_tree=max_tree,
                                       d_latent=VERIFY_ATTN_D_LATENT, d_rope=VERIFY_ATTN_D_ROPE, num_sms=num_sms,
                                       max_kv_per_req=max_kv_per_req, max_total_kv=max_total_kv,
                                       pool_slots=pool_slots, sm_scale=sm_scale)
        self.plan, self.ws_bytes = verify_attn_plan(self.params)
        self.device = torch.device("cuda") if device is None else torch.device(device)
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.device)
        verify_attn_workspace_init(self.plan, _ptr(self.workspace), self.ws_bytes,
                                   torch.cuda.current_stream(self.device).cuda_stream)

    def make_args(self, q_latent, q_rope, kv_pool, kv_indices, kv_indptr, qo_indptr, tree_anc, out,
                  lse=None, visible_count=None) -> VerifyAttnArgs:
        """Fill the C argument struct from tensors (bf16 tensors or uint16 bit views)."""
        return VerifyAttnArgs(
            q_latent=_ptr(q_latent), q_latent_stride_tok=q_latent.stride(0), q_latent_stride_head=q_latent.stride(1),
            q_rope=_ptr(q_rope), q_rope_stride_tok=q_rope.stride(0), q_rope_stride_head=q_rope.stride(1),
            kv_pool=_ptr(kv_pool), kv_row_stride=kv_pool.stride(0),
            kv_indices=_ptr(kv_indices), kv_indptr=_ptr(kv_indptr), qo_indptr=_ptr(qo_indptr),
            tree_anc=_ptr(tree_anc), batch=int(kv_indptr.shape[0]) - 1,
            out=_ptr(out), out_stride_tok=out.stride(0), out_stride_head=out.stride(1),
            lse=_ptr(lse), visible_count=_ptr(visible_count))

    def run(self, args: VerifyAttnArgs, stream: int):
        verify_attn_run(self.plan, args, _ptr(self.workspace), self.ws_bytes, stream)

    def gather(self, args: VerifyAttnArgs, stream: int):
        verify_attn_gather(self.plan, args, _ptr(self.workspace), self.ws_bytes, stream)

    def split(self, args: VerifyAttnArgs, stream: int):
        verify_attn_split(self.plan, args, _ptr(self.workspace), self.ws_bytes, stream)

    def reduce(self, args: VerifyAttnArgs, stream: int):
        verify_attn_reduce(self.plan, args, _ptr(self.workspace), self.ws_bytes, stream)

    def __call__(self, *tensors, lse=None, visible_count=None, stream=None):
        import torch

        s = torch.cuda.current_stream(self.device).cuda_stream if stream is None else stream
        args = self.make_args(*tensors, lse=lse, visible_count=visible_count)
        self.run(args, s)
        self.reduce(args, s)
        return args

    def tree_block(self, args: VerifyAttnArgs, exclude_self: bool, self_anc_ptr, stream: int, out_f32_ptr=None):
        verify_attn_tree_block(self.plan, args, exclude_self, self_anc_ptr, out_f32_ptr, _ptr(self.workspace),
                               self.ws_bytes, stream)

    def split_verify(self, q_latent, q_rope, kv_pool, kv_indices, kv_indptr, qo_indptr, tree_anc, out,
                     lse=None, visible_count=None, stream=None):
        """The split-verify variant: tree block (strict ancestors), dense pass
        (prefix + own key) and LSE merge, three library calls on one stream.
        Same inputs and results as ``__call__`` (up to rounding). Scratch for
        the intermediate states is allocated once, sized by the plan."""
        import torch

        s = torch.cuda.current_stream(self.device).cuda_stream if stream is None else stream
        tokens = int(q_latent.shape[0])
        H = self.params.num_heads
        if getattr(self, "_sv", None) is None:
            cap = self.params.max_batch * self.params.max_tree
            self._sv = {
                "o_t": torch.empty((cap, H, VERIFY_ATTN_D_LATENT), dtype=torch.float32, device=self.device),
                "lse_t": torch.empty((cap, H), dtype=torch.float32, device=self.device),
                "lse_p": torch.empty((cap, H), dtype=torch.float32, device=self.device),
                "self_anc": torch.empty((cap,), dtype=torch.int64, device=self.device),
            }
        sv = self._sv
        if tokens > sv["self_anc"].shape[0]:
            raise VerifyAttnError(-1, "split_verify: more tokens than the plan allows")
        o_t, lse_t, lse_p, self_anc = sv["o_t"][:tokens], sv["lse_t"][:tokens], sv["lse_p"][:tokens], sv["self_anc"]
        a_t = self.make_args(q_latent, q_rope, kv_pool, kv_indices, kv_indptr, qo_indptr, tree_anc, out,
                             lse=lse_t, visible_count=visible_count)
        self.tree_block(a_t, True, _ptr(self_anc), s, out_f32_ptr=_ptr(o_t))
        a_d = self.make_args(q_latent, q_rope, kv_pool, kv_indices, kv_indptr, qo_indptr, self_anc[:tokens], out,
                             lse=lse_p)
        self.run(a_d, s)
        self.reduce(a_d, s)
        batch = int(kv_indptr.shape[0]) - 1
        m = VerifyAttnMergeArgs(
            o_a=_ptr(out), o_a_stride_tok=out.stride(0), o_a_stride_head=out.stride(1), lse_a=_ptr(lse_p),
            o_b=_ptr(o_t), o_b_stride_tok=o_t.stride(0), o_b_stride_head=o_t.stride(1), lse_b=_ptr(lse_t), o_b_f32=1,
            out=_ptr(out), out_stride_tok=out.stride(0), out_stride_head=out.stride(1), lse=_ptr(lse),
            max_tokens=tokens, num_tokens=_ptr(qo_indptr) + 4 * batch, num_heads=H)
        verify_attn_merge_states(m, s)
        return a_d

    def status(self, stream=None):
        import torch

        s = torch.cuda.current_stream(self.device).cuda_stream if stream is None else stream
        return verify_attn_status(_ptr(self.workspace), s)
