"""libpagedattn: paged KV cache decode attention for B200 (sm_100a).

    from paged_kv_cache_361_b200 import PagedKVCache          # serving-loop API
    from paged_kv_cache_361_b200 import binding               # thin C-ABI binding

The compute runs in the CUDA kernels of libpagedattn.so (built in-tree by
paged_kv_cache_361_b200.build); there is no CPU or eager fallback.
"""
from .binding import (BlockManager, PagedAttnError, pa_copy_blocks, pa_decode, pa_decode_partition_tokens,  # noqa: F401
                      pa_decode_workspace_bytes, pa_get_device_error, pa_reshape_and_cache)
from .cache import PagedKVCache  # noqa: F401
