"""CPU oracle for the paged KV cache append and paged decode attention.

TEST INFRASTRUCTURE.  Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  The library
(``paged_kv_cache_473_b200``) never imports it and shares no code with it.

The arithmetic lives in ``paged_attention_oracle.c`` (plain C, fp64, OpenMP over
output rows); this module compiles it with gcc on first use and marshals torch
CPU tensors into it.  The functions below follow these passages:

* ``write_kv`` -- nano-vllm (ovshake) README, "Key Concepts Explained: KV Cache"
  and "Key Concepts Explained: PagedAttention".
* ``decode`` -- the same README, "X-Ray Mode" (GQA head sharing, scores
  ``Q K^T / sqrt(d)``) and "PagedAttention"; flex-nano-vllm README (paged
  attention through a page table, Gemma 2).  Softmax, softcap and window
  readings are stated in the C file's header.
* ``decode_multi`` -- several query tokens per sequence with a causal mask
  (the README's "Features": chunked prefill, speculative decoding); each query
  token is the decode above over the positions up to its own.
* ``prefill`` -- ``write_kv`` of a prompt's (or chunk's) rows followed by
  ``decode_multi`` per sequence ("Key Concepts Explained: KV Cache": prefill
  computes and stores the prompt's keys and values).

Pins (tests/test_oracle_pins.py): agreement with torch's fp64
``scaled_dot_product_attention`` on contiguous K/V, permutation invariance over
physical blocks, L = 1 returning V, identical keys giving mean(V), an infinite
softcap equal to no softcap, softcap saturation and two-token closed forms,
window special cases, the page-table example drawn on the nano-vllm README and
incremental decoding equal to causal attention; for ``decode_multi``,
agreement with torch's fp64 attention under an explicit causal (and window)
mask on contiguous K/V, the T = 1 case equal to ``decode`` bit for bit, and
causality (changing later positions leaves a row unchanged).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "paged_attention_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, BF16 = 0, 1
_ERRORS = {1: "bad arguments", 2: "slot out of range", 3: "block id out of range", 4: "context length out of range",
           5: "out of memory"}


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        vp, i32, i64p, i32p, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_double
        lib.oracle_write_kv.argtypes = [vp, vp, i64p, i32, vp, vp, i32, i32, i32, i32, i32]
        lib.oracle_write_kv.restype = i32
        lib.oracle_decode.argtypes = [vp, i32, vp, vp, i32, i32p, i32p, i32, i32, i32, i32, i32, i32, i32, dbl, dbl,
                                      i32, i32p, i32, vp]
        lib.oracle_decode.restype = i32
        lib.oracle_decode_multi.argtypes = [vp, i32, vp, vp, i32, i32p, i32p, i32, i32, i32, i32, i32, i32, i32, i32,
                                            dbl, dbl, i32, i32p, i32, vp]
        lib.oracle_decode_multi.restype = i32
        lib.oracle_num_threads.restype = i32
        lib.oracle_set_num_threads.argtypes = [i32]
        _lib = lib
    return _lib


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(n)


def _code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"oracle takes fp32 or bf16, got {t.dtype}")


def _cpu(t: torch.Tensor) -> torch.Tensor:
    t = t.detach()
    if t.device.type != "cpu":
        t = t.cpu()
    return t.contiguous()


def _check(status: int) -> None:
    if status != 0:
        raise ValueError(f"oracle: {_ERRORS.get(status, status)}")


def write_kv(k_new: torch.Tensor, v_new: torch.Tensor, slot_mapping: torch.Tensor, k_cache: torch.Tensor,
             v_cache: torch.Tensor) -> None:
    """Append rows into CPU cache tensors in place (byte copy per slot)."""
    assert k_cache.device.type == "cpu" and k_cache.is_contiguous() and v_cache.is_contiguous()
    k_new, v_new = _cpu(k_new), _cpu(v_new)
    slots = _cpu(slot_mapping).to(torch.int64)
    nb, hkv, bs, d = k_cache.shape
    assert k_new.dtype == k_cache.dtype == v_cache.dtype == v_new.dtype
    n = slots.numel()
    assert k_new.shape == (n, hkv, d) and v_new.shape == (n, hkv, d)
    _check(_load().oracle_write_kv(k_new.data_ptr(), v_new.data_ptr(), slots.data_ptr(), n, k_cache.data_ptr(),
                                   v_cache.data_ptr(), nb, bs, hkv, d, _code(k_cache)))


def decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
           context_lens: torch.Tensor, scale: float, softcap: float = 0.0, window: int = 0,
           rows: Optional[Sequence[tuple]] = None) -> np.ndarray:
    """fp64 decode attention.  Returns ``[B, Hq, D]`` (or ``[len(rows), D]``).

    ``scale`` and ``softcap`` are rounded to fp32 first, as the GPU library
    receives them, and then widened exactly.
    """
    q, k_cache, v_cache = _cpu(q), _cpu(k_cache), _cpu(v_cache)
    bt = _cpu(block_tables).to(torch.int32)
    cl = _cpu(context_lens).to(torch.int32)
    B, hq, d = q.shape
    nb, hkv, bs, d2 = k_cache.shape
    assert d == d2 and v_cache.shape == k_cache.shape and k_cache.dtype == v_cache.dtype
    scale64 = float(np.float32(scale))
    cap64 = float(np.float32(softcap)) if np.isfinite(softcap) else float(softcap)
    if rows is None:
        out = np.zeros((B, hq, d), dtype=np.float64)
        rows_arr, n_rows = None, 0
    else:
        rows_arr = torch.tensor([list(r) for r in rows], dtype=torch.int32).reshape(-1, 2).contiguous()
        n_rows = rows_arr.shape[0]
        out = np.zeros((n_rows, d), dtype=np.float64)
    st = _load().oracle_decode(q.data_ptr(), _code(q), k_cache.data_ptr(), v_cache.data_ptr(), _code(k_cache),
                               bt.data_ptr(), cl.data_ptr(), B, hq, hkv, d, bs, bt.shape[1], nb, scale64, cap64,
                               int(window), None if rows_arr is None else rows_arr.data_ptr(), n_rows,
                               out.ctypes.data)
    _check(st)
    return out


def decode_multi(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
                 context_lens: torch.Tensor, scale: float, softcap: float = 0.0, window: int = 0,
                 rows: Optional[Sequence[tuple]] = None) -> np.ndarray:
    """fp64 multi-query attention: ``q`` is ``[B, T, Hq, D]``; query token j
    of sequence b sits at position ``L - T + j`` and attends causally.
    Returns ``[B, T, Hq, D]`` (or ``[len(rows), D]`` for ``(b, j, h)`` rows)."""
    q, k_cache, v_cache = _cpu(q), _cpu(k_cache), _cpu(v_cache)
    bt = _cpu(block_tables).to(torch.int32)
    cl = _cpu(context_lens).to(torch.int32)
    B, T, hq, d = q.shape
    nb, hkv, bs, d2 = k_cache.shape
    assert d == d2 and v_cache.shape == k_cache.shape and k_cache.dtype == v_cache.dtype
    scale64 = float(np.float32(scale))
    cap64 = float(np.float32(softcap)) if np.isfinite(softcap) else float(softcap)
    if rows is None:
        out = np.zeros((B, T, hq, d), dtype=np.float64)
        rows_arr, n_rows = None, 0
    else:
        rows_arr = torch.tensor([list(r) for r in rows], dtype=torch.int32).reshape(-1, 3).contiguous()
        n_rows = rows_arr.shape[0]
        out = np.zeros((n_rows, d), dtype=np.float64)
    st = _load().oracle_decode_multi(q.data_ptr(), _code(q), k_cache.data_ptr(), v_cache.data_ptr(), _code(k_cache),
                                     bt.data_ptr(), cl.data_ptr(), B, T, hq, hkv, d, bs, bt.shape[1], nb, scale64,
                                     cap64, int(window), None if rows_arr is None else rows_arr.data_ptr(), n_rows,
                                     out.ctypes.data)
    _check(st)
    return out


def prefill(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, slot_mapping: torch.Tensor,
            cu_q_lens: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
            context_lens: torch.Tensor, scale: float, softcap: float = 0.0, window: int = 0) -> np.ndarray:
    """Paged prefill: append the new rows (``write_kv``, in place on the CPU
    caches), then sequence b's query rows ``[cu[b], cu[b+1])`` -- its last
    ``T_b`` positions -- attend causally (``decode_multi`` with ``T = T_b``).
    Returns ``[total, Hq, D]`` fp64."""
    if k_new is not None:
        write_kv(k_new, v_new, slot_mapping, k_cache, v_cache)
    cu = [int(x) for x in _cpu(cu_q_lens)]
    q = _cpu(q)
    tables, lens = _cpu(block_tables), _cpu(context_lens)
    out = np.zeros((q.shape[0], q.shape[1], q.shape[2]), dtype=np.float64)
    for b in range(len(cu) - 1):
        T = cu[b + 1] - cu[b]
        if T == 0:
            continue
        out[cu[b]:cu[b + 1]] = decode_multi(q[cu[b]:cu[b + 1]].unsqueeze(0), k_cache, v_cache, tables[b:b + 1],
                                            lens[b:b + 1], scale, softcap, window)[0]
    return out


def decode_batch(batch, softcap: Optional[float] = None, window: Optional[int] = None, rows=None) -> np.ndarray:
    """``decode`` on a ``workloads.Batch`` with its own scale/softcap/window."""
    w = batch.workload
    return decode(batch.q, batch.k_cache, batch.v_cache, batch.block_tables, batch.context_lens, w.scale,
                  w.softcap if softcap is None else softcap, w.window if window is None else window, rows=rows)
