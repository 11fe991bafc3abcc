"""ctypes binding of ``libpagedattn.so`` (include/pagedattn.h).

Argument marshalling only: shapes, raw device pointers and the current CUDA
stream go to the C ABI; every step of the computation runs in the library's
kernels.  torch provides device memory (the optional ``out`` tensors and the
split-K workspace) and streams.  The binding refuses to run if the library is
missing or cannot be built; there is no fallback path.

The library is opened on first use (the first call, or the first read of
``lib``), not at import, so that importing the package for its input
generators (``workloads``) maps no GPU code.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import build as _build

PA_F32, PA_BF16 = 0, 1
PA_OK, PA_ERR_INVALID, PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE, PA_ERR_CUDA = 0, 1, 2, 3, 4
# pa_schedule_t (include/pagedattn.h)
SCHEDULES = {0: "none", 1: "single", 2: "grid", 3: "dynamic", 4: "dynamic_merged"}
KERNELS = {"auto": 0, "cuda_core": 1, "mma": 2}
DEVERR_SLOT, DEVERR_BLOCK, DEVERR_CONTEXT, DEVERR_TIMEOUT, DEVERR_LAYOUT = 1, 2, 4, 8, 16

_c_i32, _c_i64, _c_f32, _c_sz, _c_vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: status {status} ({error_string(status)})")


def _load_library() -> ctypes.CDLL:
    path = _build.LIB
    if not _build.up_to_date():
        try:
            path = _build.build()
        except Exception as e:  # noqa: BLE001
            if not os.path.exists(path):
                raise ImportError(f"libpagedattn.so is missing and could not be built: {e}") from e
    lib = ctypes.CDLL(path)
    lib.pa_write_kv.argtypes = [_c_vp, _c_vp, _c_vp, _c_i32, _c_vp, _c_vp, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32,
                                _c_vp]
    lib.pa_write_kv.restype = _c_i32
    dec = [_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_f32, _c_f32,
           _c_i32, _c_vp, _c_i32]
    lib.pa_decode.argtypes = dec + [_c_i32, _c_vp]
    lib.pa_decode.restype = _c_i32
    lib.pa_decode_splitk.argtypes = dec + [_c_i32, _c_i32, _c_vp, _c_sz, _c_i32, _c_vp]
    lib.pa_decode_splitk.restype = _c_i32
    lib.pa_decode_step.argtypes = [_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_i32, _c_i32, _c_i32, _c_i32,
                                   _c_i32, _c_i32, _c_i32, _c_f32, _c_f32, _c_i32, _c_vp, _c_i32, _c_i32, _c_i32,
                                   _c_vp, _c_sz, _c_i32, _c_vp]
    lib.pa_decode_step.restype = _c_i32
    lib.pa_decode_splitk_noalloc.argtypes = dec + [_c_i32, _c_i32, _c_i32, _c_vp]
    lib.pa_decode_splitk_noalloc.restype = _c_i32
    lib.pa_decode_splitk_partition.argtypes = [_c_i32, _c_i32, _c_i32, _c_i32]
    lib.pa_decode_splitk_partition.restype = _c_i32
    lib.pa_decode_splitk_workspace_size.argtypes = [_c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32]
    lib.pa_decode_splitk_workspace_size.restype = _c_sz
    lib.pa_decode_multi.argtypes = [_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32,
                                    _c_i32, _c_i32, _c_f32, _c_f32, _c_i32, _c_vp, _c_i32, _c_i32, _c_i32, _c_vp, _c_sz,
                                    _c_vp]
    lib.pa_decode_multi.restype = _c_i32
    lib.pa_decode_multi_workspace_size.argtypes = [_c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32]
    lib.pa_decode_multi_workspace_size.restype = _c_sz
    lib.pa_prefill.argtypes = [_c_vp, _c_vp, _c_vp, _c_vp, _c_vp, _c_i32, _c_i32, _c_vp, _c_vp, _c_vp, _c_vp, _c_i32,
                               _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_f32, _c_f32, _c_i32, _c_vp, _c_i32,
                               _c_vp]
    lib.pa_prefill.restype = _c_i32
    lib.pa_copy_blocks.argtypes = [_c_vp, _c_vp, _c_vp, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_vp]
    lib.pa_copy_blocks.restype = _c_i32
    # host block manager (include/block_manager.h)
    lib.pa_bm_create.argtypes = [_c_i32, _c_i32]
    lib.pa_bm_create.restype = _c_vp
    lib.pa_bm_destroy.argtypes = [_c_vp]
    lib.pa_bm_destroy.restype = None
    lib.pa_bm_num_free.argtypes = [_c_vp]
    lib.pa_bm_num_free.restype = _c_i32
    lib.pa_bm_blocks_needed.argtypes = [_c_vp, _c_vp, _c_i32]
    lib.pa_bm_blocks_needed.restype = _c_i32
    lib.pa_bm_add_sequence.argtypes = [_c_vp, _c_i64, _c_vp, _c_i32, _c_vp]
    lib.pa_bm_add_sequence.restype = _c_i32
    lib.pa_bm_append_slots.argtypes = [_c_vp, _c_vp, _c_vp, _c_i32, _c_vp, _c_vp, _c_vp]
    lib.pa_bm_append_slots.restype = _c_i32
    lib.pa_bm_fork.argtypes = [_c_vp, _c_i64, _c_i64]
    lib.pa_bm_fork.restype = _c_i32
    lib.pa_bm_free_sequence.argtypes = [_c_vp, _c_i64]
    lib.pa_bm_free_sequence.restype = _c_i32
    lib.pa_bm_length.argtypes = [_c_vp, _c_i64]
    lib.pa_bm_length.restype = _c_i32
    lib.pa_bm_block_tables.argtypes = [_c_vp, _c_vp, _c_i32, _c_i32, _c_vp, _c_vp]
    lib.pa_bm_block_tables.restype = _c_i32
    lib.pa_bm_slots.argtypes = [_c_vp, _c_i64, _c_i32, _c_i32, _c_vp]
    lib.pa_bm_slots.restype = _c_i32
    lib.pa_bm_ref_count.argtypes = [_c_vp, _c_i32]
    lib.pa_bm_ref_count.restype = _c_i32
    lib.pa_decode_cascade.argtypes = dec + [_c_i32, _c_i32, _c_i32, _c_i32, _c_vp, _c_sz, _c_vp]
    lib.pa_decode_cascade.restype = _c_i32
    lib.pa_decode_cascade_workspace_size.argtypes = [_c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32]
    lib.pa_decode_cascade_workspace_size.restype = _c_sz
    lib.pa_check_bounded_wait.argtypes = [ctypes.c_uint64, _c_vp]
    lib.pa_check_bounded_wait.restype = _c_i32
    lib.pa_device_errors.argtypes = [ctypes.POINTER(ctypes.c_uint32), _c_i32]
    lib.pa_device_errors.restype = _c_i32
    lib.pa_error_string.argtypes = [_c_i32]
    lib.pa_error_string.restype = ctypes.c_char_p
    lib.pa_last_launch_count.argtypes = []
    lib.pa_last_launch_count.restype = _c_i32
    lib.pa_last_decode_schedule.argtypes = []
    lib.pa_last_decode_schedule.restype = _c_i32
    return lib


_lib_handle: Optional[ctypes.CDLL] = None


def _lib() -> ctypes.CDLL:
    """The opened library (opened, and built if stale, on first use)."""
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = _load_library()
    return _lib_handle


def __getattr__(name):  # module attribute ``lib``, resolved on first use
    if name == "lib":
        return _lib()
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")


def error_string(status: int) -> str:
    return _lib().pa_error_string(int(status)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return PA_F32
    if t.dtype == torch.bfloat16:
        return PA_BF16
    raise TypeError(f"paged attention takes float32 or bfloat16 tensors, got {t.dtype}")


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _check(status: int, what: str) -> None:
    if status != PA_OK:
        raise PagedAttnError(status, what)


def write_kv(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor, k_cache: torch.Tensor,
             v_cache: torch.Tensor, stream=None) -> None:
    """Append ``k``/``v`` rows ``[N, Hkv, D]`` into the caches at ``slot_mapping`` (int64)."""
    nb, hkv, bs, d = k_cache.shape
    st = _lib().pa_write_kv(_ptr(k), _ptr(v), _ptr(slot_mapping), slot_mapping.numel(), _ptr(k_cache), _ptr(v_cache),
                         nb, bs, hkv, d, _dtype_code(k_cache), _stream(stream))
    _check(st, "pa_write_kv")


def _decode_common(q, k_cache, block_tables, out):
    B, hq, d = q.shape
    nb, hkv, bs, d2 = k_cache.shape
    if out is None:
        out = torch.empty_like(q)
    return B, hq, d, nb, hkv, bs, out


def decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
           context_lens: torch.Tensor, scale: float, softcap: float = 0.0, window: int = 0,
           out: Optional[torch.Tensor] = None, kernel: str = "auto", stream=None) -> torch.Tensor:
    """Paged decode attention, one CTA per (sequence, kv head).  Returns ``out``."""
    B, hq, d, nb, hkv, bs, out = _decode_common(q, k_cache, block_tables, out)
    st = _lib().pa_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens), B, hq, hkv, d,
                       bs, block_tables.shape[1], nb, float(scale), float(softcap), int(window), _ptr(out),
                       _dtype_code(q), KERNELS[kernel], _stream(stream))
    _check(st, "pa_decode")
    return out


def decode_splitk_partition(batch: int, num_kv_heads: int, max_context_len: int, partition_tokens: int = 0) -> int:
    return _lib().pa_decode_splitk_partition(batch, num_kv_heads, max_context_len, partition_tokens)


def decode_splitk_workspace_size(batch: int, num_q_heads: int, head_dim: int, max_context_len: int,
                                 partition_tokens: int = 0, num_kv_heads: int = 1) -> int:
    return _lib().pa_decode_splitk_workspace_size(batch, num_q_heads, head_dim, max_context_len, partition_tokens,
                                               num_kv_heads)


def decode_splitk(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
                  context_lens: torch.Tensor, scale: float, softcap: float = 0.0, window: int = 0, *,
                  max_context_len: int, partition_tokens: int = 0, out: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, kernel: str = "auto", stream=None) -> torch.Tensor:
    """Split-K (flash-decoding) paged decode with the log-sum-exp combine.

    ``max_context_len`` is a host-side bound on every ``context_lens[b]``.
    ``partition_tokens=0`` lets the library schedule the work (the dynamic work
    queue on the tensor-core path).  The workspace (device memory) must be
    zero-filled before its first use; it is allocated zeroed with torch if not
    given.
    """
    B, hq, d, nb, hkv, bs, out = _decode_common(q, k_cache, block_tables, out)
    if workspace is None:  # (a given workspace's size is checked by the library)
        need = decode_splitk_workspace_size(B, hq, d, max_context_len, partition_tokens, hkv)
        workspace = torch.zeros(max(need, 16), dtype=torch.uint8, device=q.device)
    wbytes = workspace.numel() * workspace.element_size()
    st = _lib().pa_decode_splitk(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens), B, hq,
                              hkv, d, bs, block_tables.shape[1], nb, float(scale), float(softcap), int(window),
                              _ptr(out), _dtype_code(q), int(partition_tokens), int(max_context_len),
                              _ptr(workspace), wbytes, KERNELS[kernel], _stream(stream))
    _check(st, "pa_decode_splitk")
    return out


def decode_cascade_workspace_size(batch: int, num_q_heads: int, head_dim: int, max_context_len: int,
                                  prefix_len: int, partition_tokens: int = 0, num_kv_heads: int = 1) -> int:
    return _lib().pa_decode_cascade_workspace_size(batch, num_q_heads, head_dim, max_context_len, prefix_len,
                                                partition_tokens, num_kv_heads)


def decode_cascade(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
                   context_lens: torch.Tensor, scale: float, softcap: float = 0.0, window: int = 0, *,
                   n_sharers: int, prefix_len: int, max_context_len: int, partition_tokens: int = 0,
                   out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """Split-K decode where sequences ``0 .. n_sharers-1`` share their first
    ``prefix_len`` positions (same blocks): the prefix is read once per kv head
    for all of them, then merged with each sequence's own range."""
    B, hq, d, nb, hkv, bs, out = _decode_common(q, k_cache, block_tables, out)
    need = decode_cascade_workspace_size(B, hq, d, max_context_len, prefix_len, partition_tokens, hkv)
    if workspace is None:
        workspace = torch.zeros(max(need, 16), dtype=torch.uint8, device=q.device)
    wbytes = workspace.numel() * workspace.element_size()
    st = _lib().pa_decode_cascade(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens), B, hq,
                               hkv, d, bs, block_tables.shape[1], nb, float(scale), float(softcap), int(window),
                               _ptr(out), _dtype_code(q), int(n_sharers), int(prefix_len), int(partition_tokens),
                               int(max_context_len), _ptr(workspace), wbytes, _stream(stream))
    _check(st, "pa_decode_cascade")
    return out


def decode_step(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor,
                v_cache: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                softcap: float = 0.0, window: int = 0, *, split: bool = True, max_context_len: int = 0,
                partition_tokens: int = 0, out: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None, kernel: str = "auto", stream=None) -> torch.Tensor:
    """One decode step: append ``k_new``/``v_new`` ``[B, Hkv, D]`` at position
    ``context_lens[b] - 1`` of each sequence and attend, in one pass.

    ``split=False``: one CTA per (sequence, kv head).  ``split=True``: split-K
    with the combine (``max_context_len`` required; workspace allocated with
    torch if not given).
    """
    B, hq, d, nb, hkv, bs, out = _decode_common(q, k_cache, block_tables, out)
    ptoks = int(partition_tokens) if split else -1
    wptr, wbytes = None, 0
    if split:
        if max_context_len <= 0:
            raise ValueError("decode_step(split=True) needs max_context_len")
        if workspace is None:  # (a given workspace's size is checked by the library)
            need = decode_splitk_workspace_size(B, hq, d, max_context_len, partition_tokens, hkv)
            workspace = torch.zeros(max(need, 16), dtype=torch.uint8, device=q.device)
        wptr, wbytes = _ptr(workspace), workspace.numel() * workspace.element_size()
    st = _lib().pa_decode_step(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                            _ptr(context_lens), B, hq, hkv, d, bs, block_tables.shape[1], nb, float(scale),
                            float(softcap), int(window), _ptr(out), _dtype_code(q), ptoks, int(max_context_len), wptr,
                            wbytes, KERNELS[kernel], _stream(stream))
    _check(st, "pa_decode_step")
    return out


def decode_multi_workspace_size(batch: int, q_len: int, num_q_heads: int, head_dim: int, max_context_len: int,
                                partition_tokens: int = 0, num_kv_heads: int = 1) -> int:
    return _lib().pa_decode_multi_workspace_size(batch, q_len, num_q_heads, head_dim, max_context_len, partition_tokens,
                                              num_kv_heads)


def decode_multi(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
                 context_lens: torch.Tensor, scale: float, softcap: float = 0.0, window: int = 0, *,
                 split: bool = True, max_context_len: int = 0, partition_tokens: int = 0,
                 out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """Attention of ``q`` ``[B, T, Hq, D]`` (T new tokens per sequence, already
    appended to the cache at positions ``L-T .. L-1``) with a causal mask.

    ``split=False``: one CTA per (sequence, kv head).  ``split=True``: split-K
    with the combine (``max_context_len`` required; the workspace is allocated
    zeroed with torch if not given).
    """
    B, T, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    if out is None:
        out = torch.empty_like(q)
    ptoks = int(partition_tokens) if split else -1
    wptr, wbytes = None, 0
    if split:
        if max_context_len <= 0:
            raise ValueError("decode_multi(split=True) needs max_context_len")
        need = decode_multi_workspace_size(B, T, hq, d, max_context_len, partition_tokens, hkv)
        if workspace is None:
            workspace = torch.zeros(max(need, 16), dtype=torch.uint8, device=q.device)
        wptr, wbytes = _ptr(workspace), workspace.numel() * workspace.element_size()
    st = _lib().pa_decode_multi(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens), B, T, hq,
                             hkv, d, bs, block_tables.shape[1], nb, float(scale), float(softcap), int(window),
                             _ptr(out), _dtype_code(q), ptoks, int(max_context_len), wptr, wbytes, _stream(stream))
    _check(st, "pa_decode_multi")
    return out


def prefill(q: torch.Tensor, k_new: Optional[torch.Tensor], v_new: Optional[torch.Tensor],
            slot_mapping: Optional[torch.Tensor], cu_q_lens: torch.Tensor, k_cache: torch.Tensor,
            v_cache: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
            softcap: float = 0.0, window: int = 0, *, max_q_len: int, out: Optional[torch.Tensor] = None,
            stream=None) -> torch.Tensor:
    """Paged prefill: append ``k_new``/``v_new`` ``[total, Hkv, D]`` at
    ``slot_mapping`` (skipped when both are None), then sequence b's query
    rows ``q[cu_q_lens[b]:cu_q_lens[b+1]]`` -- its last positions -- attend
    causally.  ``max_q_len`` bounds every sequence's row count."""
    total, hq, d = q.shape
    nb, hkv, bs, _ = k_cache.shape
    if out is None:
        out = torch.empty_like(q)
    st = _lib().pa_prefill(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), _ptr(cu_q_lens), total,
                        int(max_q_len), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
                        cu_q_lens.numel() - 1, hq, hkv, d, bs, block_tables.shape[1], nb, float(scale),
                        float(softcap), int(window), _ptr(out), _dtype_code(q), _stream(stream))
    _check(st, "pa_prefill")
    return out


def copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor, pairs: torch.Tensor, stream=None) -> None:
    """Copy whole blocks inside both caches: ``pairs`` is a device int32
    ``[n, 2]`` tensor of (src, dst) block ids (copy-on-write)."""
    nb, hkv, bs, d = k_cache.shape
    pairs = pairs.to(torch.int32).contiguous()
    st = _lib().pa_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(pairs), pairs.shape[0], nb, bs, hkv, d,
                            _dtype_code(k_cache), _stream(stream))
    _check(st, "pa_copy_blocks")


def _i64_array(xs):
    xs = [int(x) for x in xs]
    return (ctypes.c_int64 * max(1, len(xs)))(*xs), len(xs)


class BlockManager:
    """The library's host block manager (include/block_manager.h): on-demand
    allocation, reference counts, fork, copy-on-write and a prefix cache of
    full blocks.  Host memory only; the copy-on-write pairs it returns are
    carried out on the GPU with :func:`copy_blocks`."""

    def __init__(self, num_blocks: int, block_size: int):
        self._h = _lib().pa_bm_create(int(num_blocks), int(block_size))
        if not self._h:
            raise PagedAttnError(PA_ERR_INVALID, "pa_bm_create")
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)

    def close(self) -> None:
        if self._h:
            _lib().pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001
            pass

    @property
    def num_free(self) -> int:
        return _lib().pa_bm_num_free(self._h)

    def blocks_needed(self, num_tokens: int, token_ids=None) -> int:
        arr = _i64_array(token_ids)[0] if token_ids is not None else None
        return _lib().pa_bm_blocks_needed(self._h, arr, int(num_tokens))

    def add_sequence(self, seq_id: int, num_tokens: int, token_ids=None) -> int:
        """Register a prompt; returns how many leading positions came from the prefix cache."""
        arr = None
        if token_ids is not None:
            arr, n = _i64_array(token_ids)
            if n != num_tokens:
                raise ValueError("token_ids must hold num_tokens ids")
        cached = ctypes.c_int32(0)
        _check(_lib().pa_bm_add_sequence(self._h, int(seq_id), arr, int(num_tokens), ctypes.byref(cached)),
               "pa_bm_add_sequence")
        return cached.value

    def append_slots(self, seq_ids, token_ids=None):
        """One decode step: returns (slots int64 [n], copy-on-write pairs int32 [k, 2])."""
        ids, n = _i64_array(seq_ids)
        toks = _i64_array(token_ids)[0] if token_ids is not None else None
        slots = (ctypes.c_int64 * max(1, n))()
        cow = (ctypes.c_int32 * max(2, 2 * n))()
        ncow = ctypes.c_int32(0)
        _check(_lib().pa_bm_append_slots(self._h, ids, toks, n, slots, cow, ctypes.byref(ncow)), "pa_bm_append_slots")
        k = ncow.value
        return (torch.tensor(list(slots)[:n], dtype=torch.int64),
                torch.tensor(list(cow)[: 2 * k], dtype=torch.int32).reshape(k, 2))

    def fork(self, parent_id: int, child_id: int) -> None:
        _check(_lib().pa_bm_fork(self._h, int(parent_id), int(child_id)), "pa_bm_fork")

    def free(self, seq_id: int) -> None:
        _check(_lib().pa_bm_free_sequence(self._h, int(seq_id)), "pa_bm_free_sequence")

    def length(self, seq_id: int) -> int:
        return _lib().pa_bm_length(self._h, int(seq_id))

    def block_tables(self, seq_ids, max_blocks: int):
        """(tables int32 [n, max_blocks], -1 padded; context_lens int32 [n]) on the host."""
        ids, n = _i64_array(seq_ids)
        tables = torch.empty((n, int(max_blocks)), dtype=torch.int32)
        lens = torch.empty((n,), dtype=torch.int32)
        _check(_lib().pa_bm_block_tables(self._h, ids, n, int(max_blocks), tables.data_ptr(), lens.data_ptr()),
               "pa_bm_block_tables")
        return tables, lens

    def slots(self, seq_id: int, start: int, count: int) -> torch.Tensor:
        out = torch.empty((int(count),), dtype=torch.int64)
        _check(_lib().pa_bm_slots(self._h, int(seq_id), int(start), int(count), out.data_ptr() if count else None),
               "pa_bm_slots")
        return out

    def ref_count(self, block: int) -> int:
        return _lib().pa_bm_ref_count(self._h, int(block))


# PA_NOALLOC_SCRATCH_BYTES of include/pagedattn.h (a CPU test checks that the two agree).
NOALLOC_SCRATCH_BYTES = 16 << 20


def decode_splitk_noalloc(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                          block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float, softcap: float = 0.0,
                          window: int = 0, *, max_context_len: int, partition_tokens: int = 0,
                          out: torch.Tensor, kernel: str = "auto", stream=None) -> torch.Tensor:
    """``decode_splitk`` for callers that must not allocate device memory: the
    split-K scratch is the library's own fixed array, and ``out`` must be given.
    Calls must not overlap on the GPU (they share that array)."""
    B, hq, d, nb, hkv, bs, out = _decode_common(q, k_cache, block_tables, out)
    st = _lib().pa_decode_splitk_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
                                      B, hq, hkv, d, bs, block_tables.shape[1], nb, float(scale), float(softcap),
                                      int(window), _ptr(out), _dtype_code(q), int(partition_tokens),
                                      int(max_context_len), KERNELS[kernel], _stream(stream))
    _check(st, "pa_decode_splitk_noalloc")
    return out


def device_errors(clear: bool = True) -> int:
    """OR of the PA_DEVERR_* bits raised on the current device (synchronises)."""
    bits = ctypes.c_uint32(0)
    _check(_lib().pa_device_errors(ctypes.byref(bits), 1 if clear else 0), "pa_device_errors")
    return bits.value


def check_bounded_wait(limit_ns: int = 1_000_000, stream=None) -> None:
    """Launch the bounded-wait check (a wait nothing completes, given up after
    ``limit_ns``); read the resulting PA_DEVERR_TIMEOUT with device_errors()."""
    _check(_lib().pa_check_bounded_wait(int(limit_ns), _stream(stream)), "pa_check_bounded_wait")


def last_launch_count() -> int:
    return _lib().pa_last_launch_count()


def last_decode_schedule() -> str:
    """Name of the schedule the last decode call on this thread ran
    ("dynamic_merged", "dynamic", "grid", "single", or "none")."""
    return SCHEDULES.get(_lib().pa_last_decode_schedule(), "unknown")
