"""B200-native paged KV-cache attention: thin Python binding over ``libpagedkv.so``.

The library (``csrc/``, declared in ``include/pagedkv.h``) holds every kernel
of the path; this package only marshals torch tensors' device pointers and
the current CUDA stream into its C-ABI calls.  Importing the package does not
load the library; the first call does, and fails loudly if it is missing.
"""
from ._binding import (  # noqa: F401
    FP8_E4M3,
    FP8_POOL_DTYPES,
    PagedKVError,
    copy_blocks,
    decode_multi_partition_size,
    decode_partition_size,
    decode_workspace_size,
    prefill_fp8_workspace_size,
    get_device_error,
    library_path,
    load_library,
    paged_attention_decode,
    paged_attention_decode_fp8,
    paged_attention_decode_step,
    paged_attention_decode_step_fp8,
    paged_attention_decode_multi,
    paged_attention_decode_multi_step,
    paged_attention_prefill_chunk,
    paged_attention_prefill_chunk_fp8,
    reshape_and_cache,
    reshape_and_cache_fp8,
    set_wait_limit_ns,
    DEFAULT_WAIT_LIMIT_NS,
    swap_blocks,
)
