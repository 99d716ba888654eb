"""Block-sparse video attention for B200 (sm_100a): fused QK-RMSNorm + 3D RoPE,
SubBlock block selection and block-sparse attention, behind a C ABI
(include/sbattn.h) with a thin torch binding."""

from .api import (AttentionLayer, SBAttnError, adaln_modulate, attention_flops, check_status, forward,  # noqa: F401
                  keep_count, select_blocks_noalloc,
                  nblocks, qk_norm_rope, select_blocks, select_blocks_pooled, select_blocks_threshold,
                  select_workspace_bytes, swiglu)

__all__ = ["AttentionLayer", "SBAttnError", "adaln_modulate", "attention_flops", "check_status", "forward",
           "keep_count", "select_blocks_noalloc",
           "nblocks", "qk_norm_rope", "select_blocks", "select_blocks_pooled", "select_blocks_threshold",
           "select_workspace_bytes", "swiglu"]
