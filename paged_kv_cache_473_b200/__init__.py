"""B200 (sm_100a) paged KV cache: KV append and paged decode attention.

The compute lives in ``libpagedattn.so`` (C ABI, include/pagedattn.h); this
package is its Python binding plus seeded synthetic batch generators
(``workloads``) and the in-tree build step (``build``).
"""

from ._binding import (  # noqa: F401
    BlockManager,
    copy_blocks,
    DEVERR_BLOCK,
    DEVERR_CONTEXT,
    DEVERR_LAYOUT,
    DEVERR_SLOT,
    DEVERR_TIMEOUT,
    KERNELS,
    PagedAttnError,
    decode,
    decode_cascade,
    decode_cascade_workspace_size,
    decode_multi,
    decode_multi_workspace_size,
    decode_splitk,
    decode_splitk_noalloc,
    decode_step,
    decode_splitk_partition,
    decode_splitk_workspace_size,
    check_bounded_wait,
    device_errors,
    error_string,
    last_launch_count,
    lib,
    prefill,
    write_kv,
)

__all__ = [
    "BlockManager",
    "copy_blocks",
    "write_kv",
    "decode",
    "decode_cascade",
    "decode_cascade_workspace_size",
    "decode_multi",
    "decode_multi_workspace_size",
    "decode_splitk",
    "decode_splitk_noalloc",
    "decode_step",
    "decode_splitk_partition",
    "decode_splitk_workspace_size",
    "check_bounded_wait",
    "device_errors",
    "error_string",
    "last_launch_count",
    "prefill",
    "PagedAttnError",
]
