"""attn25: exact fused attention for B200 (sm_100a) behind a small C ABI.

The compute runs in libattn25.so (hand-written sm_100a kernels); this package
is its ctypes binding plus helpers that allocate the caller-owned buffers
with PyTorch.  Importing it fails if the library has not been built.
"""
from __future__ import annotations

import torch

from .abi import (  # noqa: F401
    ATTN_ERR_TIMEOUT,
    EXPORTED,
    LIB,
    LIB_PATH,
    MASK_BITMAP,
    MASK_CAUSAL,
    MASK_DOCUMENT,
    MASK_SLIDING_WINDOW,
    MASK_VARLEN,
    MOD_ALIBI,
    MOD_CAUSAL,
    MOD_DOCUMENT,
    MOD_LOCAL_BOOST,
    MOD_NONE,
    MOD_SLIDING_WINDOW,
    MOD_SOFTCAP,
    WALK_CLUSTER_LAUNCH_CONTROL,
    WALK_DEFAULT,
    WALK_STATIC,
    AttnError,
    BlockMask,
    ModParams,
    attn_block_mask_bind,
    attn_block_mask_bytes,
    attn_bwd,
    attn_bwd_deterministic,
    attn_bwd_deterministic_workspace_size,
    attn_bwd_strided,
    attn_bwd_noalloc,
    attn_bwd_noalloc_max_workspace,
    attn_bwd_workspace_size,
    attn_check_wait_timeout,
    attn_fp8_rotate_quantize,
    attn_fwd,
    attn_fwd_fp8,
    attn_fwd_strided,
    attn_get_status,
    attn_set_wait_limit_ms,
    attn_set_work_walk,
    attn_strerror,
    build_block_mask,
)
from .counts import useful_elements, useful_flops  # noqa: F401


def new_block_mask(mod_kind, mod_params, B, Sq, Skv, device="cuda", stream=None) -> BlockMask:
    """Allocate a block-mask buffer with torch, bind it and build it on the GPU."""
    nbytes = attn_block_mask_bytes(B, Sq, Skv)
    buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
    off = (-buf.data_ptr()) % 256
    buf = buf[off:off + nbytes]
    mask = attn_block_mask_bind(buf, B, Sq, Skv)
    build_block_mask(mod_kind, mod_params, B, Sq, Skv, mask, stream)
    return mask


def new_bwd_workspace(B, Hq, Sq, D, device="cuda", deterministic=False) -> torch.Tensor:
    """A 256-byte-aligned workspace of attn_bwd_workspace_size bytes (or, with
    deterministic=True, attn_bwd_deterministic_workspace_size bytes)."""
    nbytes = (attn_bwd_deterministic_workspace_size if deterministic else attn_bwd_workspace_size)(B, Hq, Sq, D)
    buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
    off = (-buf.data_ptr()) % 256
    return buf[off:off + nbytes]
