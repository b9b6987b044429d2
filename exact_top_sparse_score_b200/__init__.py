"""Exact Top-k sparse decode attention on B200 (sm_100a).

The compute lives in ``libtopk_attn.so`` (hand-written CUDA behind a C ABI,
declared in ``include/topk_attn.h``).  This package is a thin ctypes binding:
it checks tensors, allocates outputs with torch when the caller passes none,
and forwards pointers and the current CUDA stream.  There is no CPU path:
every call fails if the library is missing or a tensor is not on a CUDA
device.
"""
from ._binding import (  # noqa: F401
    TKA_BF16,
    TKA_F32,
    DEV_BAD_PAGE,
    DEV_BAD_SEQ_LEN,
    DEV_INTERNAL,
    DEV_TIMEOUT,
    TopkAttnError,
    block_attn_workspace_size,
    library_path,
    load_library,
    topk_attn_decode,
    topk_attn_decode_certified,
    topk_attn_decode_paged,
    topk_attn_decode_static,
    topk_attn_static_workspace_capacity,
    topk_attn_debug_set_wait_limit,
    topk_attn_device_status,
    topk_attn_last_device_status,
    topk_attn_workspace_size,
    topk_block_attn_decode,
    topk_block_pool_keys,
    topk_hisa_attn_decode,
    topk_indexer_attn_decode,
)
