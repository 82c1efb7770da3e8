"""B200-native paged KV-cache decode: the Python face of ``libpagedkv.so``.

    from paged_kv_cache_468_b200 import kv_cache_write, paged_attention_decode

Importing the package loads nothing; the CUDA library is opened on the first
call that needs it, and a missing or unloadable library raises at that point.
There is no CPU fallback.
"""
from .pagedkv import (  # noqa: F401
    BF16,
    F16,
    BlockAllocator,
    PagedKVError,
    copy_blocks,
    decode_cascade_plan,
    decode_plan,
    decode_workspace_bytes,
    device_flags,
    hbm_gather_probe,
    hbm_read_probe,
    kv_cache_write,
    lib,
    paged_attention_decode,
    paged_attention_decode_cascade,
    paged_attention_prefill,
    selftest_bounded_wait,
    version,
)
