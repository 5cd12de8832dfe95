"""B200-native paged KV cache: decode attention, slot-mapping scatter, copy-on-write.

Thin Python binding over ``libpagedkv.so`` (C ABI in ``include/pagedkv.h``).
Every step of the GPU path runs in the library's CUDA kernels; this module only
checks tensor dtypes/shapes/devices and passes pointers.  PyTorch is used for
device memory and streams.  There is no CPU fallback: if the library is
missing, every call raises.

Functions mirror the C names:
    paged_attention_decode, paged_attention_decode_append (fused: new K/V row
    written, then attended), paged_attention_decode_shared_prefix + prefix_groups
    (shared prefixes read once per group), paged_attention_workspace_bytes,
    reshape_and_cache,
    copy_blocks, device_errors, BlockManager (bm_*), paged_decode_step_host and
    DecodeSession / decode_step (one step from host buffers: inputs uploaded,
    copy-on-write copies, fused append + attention, output downloaded),
    LayeredDecodeStep (every layer's decode as one CUDA graph).
"""
from ._native import (  # noqa: F401
    BlockManager,
    DecodeSession,
    PagedKVError,
    copy_blocks,
    decode_step,
    device_errors,
    library_path,
    load_library,
    paged_attention_decode,
    paged_attention_decode_append,
    paged_attention_decode_shared_prefix,
    paged_attention_partition_tokens,
    paged_attention_shared_prefix_workspace_bytes,
    paged_attention_workspace_bytes,
    paged_decode_step_host,
    paged_decode_step_staging_bytes,
    prefix_groups,
    reshape_and_cache,
    selftest_wait_timeout,
    DEVERR_BLOCK_ID,
    DEVERR_CONTEXT_LEN,
    DEVERR_SLOT,
    DEVERR_TIMEOUT,
    DEVERR_INTERNAL,
    DEVERR_PREFIX,
    GROUP_WIDTH,
)
from .graph import LayeredDecodeStep  # noqa: F401,E402
