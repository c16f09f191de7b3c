"""B200-native paged-KV decode / prefill attention (sm_100a).

The computation lives in libpagedkv.so (CUDA, C ABI in include/pagedkv.h);
this package is a thin ctypes binding plus seeded input generators.  Importing
the package does not load the library; the first call does, and raises if the
library has not been built -- there is no CPU fallback.
"""
from .binding import (  # noqa: F401
    PagedKVError,
    SPLIT_TOKENS,
    TILE_TOKENS,
    kv_append,
    kv_append_varlen,
    library_path,
    merge_partials,
    paged_attn_partials,
    partials_size,
    paged_decode_attn,
    paged_decode_attn_append,
    paged_decode_attn_static_ws,
    paged_prefill_attn,
    paged_prefill_attn_bwd,
    paged_varlen_attn,
    strerror,
    varlen_workspace_size,
    workspace_size,
)
