"""paged_kv_cache_404_b200: PagedAttention's data-parallel hot path for B200.

A C ABI library (libpagedkv.so, see include/pagedkv.h) with the CUDA calls
paged_kv_write, paged_attention_decode, copy_blocks and swap_blocks, and a
native host block manager; this package is its thin Python binding (torch is used for device
memory and streams only).
"""
from ._lib import PagedKVError, lib  # noqa: F401
from .block_manager import BlockManager  # noqa: F401
from .ops import (  # noqa: F401
    BLOCK_SIZE,
    copy_blocks,
    decode_workspace,
    decode_workspace_bytes,
    decode_workspace_bytes_shared,
    paged_attention_decode,
    paged_attention_decode_shared,
    paged_attention_prefill,
    paged_attention_decode_noalloc,
    paged_kv_write,
    swap_blocks,
)
