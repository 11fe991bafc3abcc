"""B200 (sm_100a) paged KV cache: KV append and paged decode attention.

The compute lives in ``libpagedattn.so`` (C ABI, include/pagedattn.h); this
package is its Python binding plus seeded synthetic batch generators
(``workloads``) and the in-tree build step (``build``).  The library is opened
on the first call into it (or the first read of ``lib``), so importing the
package, or only its input generators, maps no GPU code.
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
    last_decode_schedule,
    last_launch_count,
    prefill,
    write_kv,
)


def __getattr__(name):  # ``lib``: the opened library, resolved on first use
    if name == "lib":
        from . import _binding

        return _binding.lib
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")


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
    "last_decode_schedule",
    "last_launch_count",
    "prefill",
    "PagedAttnError",
]
