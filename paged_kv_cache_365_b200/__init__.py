"""B200-native paged KV-cache decode: slot-mapped append, copy-on-write block
copy, paged single-query attention with split-K partitions, block swapping
to a host pool, and a host block allocator -- behind the C ABI of libpkv.so
(include/pkv.h).

Importing the package loads libpkv.so; it raises ImportError when the library
has not been built.  There is no CPU or Python fallback.
"""
from ._lib import (ERR_BLOCK_RANGE, ERR_CONTEXT_RANGE, ERR_COPY_RANGE, ERR_SLOT_RANGE,  # noqa: F401
                   ERR_TIMEOUT, LIB_PATH, PkvError)
from .api import (BLOCK_SIZE, DEFAULT_PARTITION, BlockAllocator, PagedKVCache, copy_blocks,  # noqa: F401
                  copy_blocks_check, decode_workspace_bytes, get_error, kv_append, kv_cache_bytes,
                  paged_attention_decode, paged_attention_decode_static_ws, paged_attention_decode_prefix,
                  decode_prefix_workspace_bytes, common_prefix_pages, swap_blocks, swap_blocks_check,
                  paged_attention_multi, multi_workspace_bytes, kv_append_fp8, paged_attention_decode_fp8,
                  kv_append_copy, cow_copy_rows, selftest_bounded_wait, cascade_prefix_pages,
                  partition_tokens, decode_step, paged_attention_decode_prefix_fp8,
                  decode_prefix_fp8_workspace_bytes, paged_attention_multi_fp8, decode_step_fp8)
