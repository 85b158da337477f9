"""B200-native paged tree-attention verify and paged KV-append (libtaco_attn + a thin binding).

The compute path is the C-ABI library ``libtaco_attn.so`` built from ``csrc/`` for sm_100a; the
functions below only marshal torch tensors into its pointers and sizes.
"""
from ._lib import (  # noqa: F401
    PrefixCache,
    TACO_OPT_GRID_CTAS,
    TACO_OPT_KERNEL,
    TACO_OPT_L2_PREFETCH,
    TACO_OPT_TEST_STALL,
    TACO_OPT_SEG_COST,
    TACO_OPT_COMBINE,
    TacoError,
    check_device,
    check_noalloc,
    load,
    logits_argmax,
    lookahead_propose,
    lookahead_update_copy_len,
    paged_kv_append,
    paged_kv_append_e4m3,
    paged_tree_attention,
    paged_tree_attention_append,
    paged_tree_attention_e4m3,
    paged_tree_attention_noalloc,
    release_workspace,
    set_option,
    tree_greedy_accept,
    tree_mask_from_parents,
    version,
    last_call_launches,
)
