"""B200-native MLA-absorb tree-verify attention.

The computation runs in the CUDA library ``lib/libverify_attn.so`` (built
from ``csrc/`` for sm_100a); this package only marshals arguments to its C
ABI (``include/verify_attn.h``) through ctypes. There is no fallback: if the
library cannot be built or loaded, importing the binding raises.
"""
from ._binding import (  # noqa: F401
    VERIFY_ATTN_D_LATENT,
    VERIFY_ATTN_D_ROPE,
    VERIFY_ATTN_MAX_TREE,
    VERIFY_ATTN_STATIC_WS_BYTES,
    VerifyAttnArgs,
    VerifyAttnDefragArgs,
    VerifyAttnMergeArgs,
    VerifyAttnMergeStackedArgs,
    VerifyAttnError,
    VerifyAttnParams,
    VerifyAttnPlan,
    VerifyAttention,
    defrag,
    lib_path,
    load_library,
    verify_attn_build_tree_mask,
    verify_attn_build_tree_mask_device,
    verify_attn_defrag,
    verify_attn_forward_static,
    verify_attn_gather,
    verify_attn_merge_stacked,
    verify_attn_merge_states,
    verify_attn_plan,
    verify_attn_reduce,
    verify_attn_run,
    verify_attn_split,
    verify_attn_status,
    verify_attn_strerror,
    verify_attn_tree_block,
    verify_attn_workspace_init,
)
