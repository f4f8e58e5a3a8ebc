"""fp64 CPU oracle for fused attention — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline arm of
``bench.py`` may import this package.  The CUDA library never calls it and it
never calls the CUDA library.
"""
from .attention import (  # noqa: F401
    MOD_ALIBI,
    MOD_CAUSAL,
    MOD_DOCUMENT,
    MOD_LOCAL_BOOST,
    MOD_NONE,
    MOD_SLIDING_WINDOW,
    MOD_SOFTCAP,
    MASK_BITMAP,
    MASK_CAUSAL,
    MASK_DOCUMENT,
    MASK_SLIDING_WINDOW,
    MASK_VARLEN,
    has_bitmap,
    has_document,
    has_mask,
    split_mod,
    alibi_slope,
    attention_backward,
    attention_forward,
    attention_probs,
    online_forward,
    score_mod,
    useful_elements,
    useful_flops,
)
from .block_sparsity import block_mask, classify_tiles  # noqa: F401
from .fp8 import (  # noqa: F401
    attention_forward_fp8,
    fwht,
    hadamard,
    prep_fp32,
    quantize_e4m3,
    quantize_per_head,
    rotation,
)
