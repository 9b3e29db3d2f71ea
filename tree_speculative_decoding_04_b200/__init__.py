"""Teacher-side verification step of tree speculative decoding on NVIDIA B200.

Four calls, each a hand-written sm_100a CUDA kernel behind a C ABI
(``include/treeverify.h``): ``tree_build_mask``, ``tree_attention``,
``tree_accept`` and ``kv_commit_realign``.  This package only marshals torch
tensors into those calls (``_lib``) and offers a host-side driver of one whole
verification step (``verifier``).
"""
from ._lib import (  # noqa: F401
    ATTN_PREFIX_READY,
    ATTN_ROPE,
    EXPORTS,
    LIB_PATH,
    MAX_TREE_ROWS,
    SEQ_BAD_GEOMETRY,
    SEQ_BAD_PARENT,
    SEQ_TIMEOUT,
    SEQ_TOO_DEEP,
    TVError,
    attention_workspace,
    kv_commit_realign,
    layer_pointers,
    load,
    set_wait_limit_ns,
    tree_accept,
    tree_accept_lm_head,
    lm_head_workspace,
    tree_attention,
    tree_attention_workspace_size,
    tree_build_mask,
    tree_kv_write,
)
