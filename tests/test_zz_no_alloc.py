"""The allocation-free split-K entry point, pa_decode_splitk_noalloc.

Some callers cannot allocate device memory where they decode: code inside a
stream capture that forbids allocation, a serving loop that cannot pay for an
allocation's synchronisation, or a host whose device memory belongs to an
allocator the library cannot reach.  For them the library keeps a fixed
split-K scratch array of its own.  This file checks, through the C ABI, that
the entry point gives bit for bit the answer of pa_decode_splitk with a caller
workspace (the same kernels and partition run), and that both lie within the
decode tolerance of the CPU oracle, on two calls in a row with different
inputs (the second call meets the scratch the first one left behind).  It
covers a shape whose partitions are merged inside the decode kernel, one
merged by the combine kernel after the dynamic schedule, and one on the fixed
partition grid; the Python wrapper is checked too, and requests larger than the
array are refused.  It is collected last, so that a run that stops at the first
failure has run every other test first.
"""

import ctypes

import pytest
import torch

import oracle
import paged_kv_cache_473_b200 as pa
from paged_kv_cache_473_b200 import _binding as bnd
from paged_kv_cache_473_b200 import workloads as wl
from tests.gpu_helpers import assert_close, bits, to_dev

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines, never run there
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _call_noalloc(b, w, out, partition_tokens, max_ctx):
    return bnd.lib.pa_decode_splitk_noalloc(
        b.q.data_ptr(), b.k_cache.data_ptr(), b.v_cache.data_ptr(), b.block_tables.data_ptr(),
        b.context_lens.data_ptr(), b.q.shape[0], w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
        b.block_tables.shape[1], b.k_cache.shape[0], ctypes.c_float(w.scale), ctypes.c_float(w.softcap), w.window,
        out.data_ptr(), bnd.PA_BF16, partition_tokens, max_ctx, 0, torch.cuda.current_stream().cuda_stream)


# (workload, batch size / length bound, partition): how the partitions are merged
CASES = [
    ("tinyllama_1b", dict(batch=48), 0, "dynamic_merged"),          # work queue, merged inside the decode kernel
    ("llama3_8b", dict(batch=24, max_len=3000), 0, "dynamic"),      # work queue, merged by the combine kernel
    ("tinyllama_1b", dict(batch=16), 128, "grid"),                  # fixed partition grid and the combine kernel
]


@pytest.mark.parametrize("name,kw,partition_tokens,schedule", CASES)
def test_noalloc_equals_the_workspace_entry_point_and_the_oracle_on_two_calls(name, kw, partition_tokens, schedule):
    w = wl.WORKLOADS[name].replace(prefix_share=0.0)
    pa.device_errors(clear=True)
    for call, seed in enumerate((w.seed, w.seed + 1)):  # different inputs on the second call
        b_cpu = wl.make_batch(w, seed=seed, prefilled=True, **kw)
        b = to_dev(b_cpu)
        max_ctx = b_cpu.max_context_len
        need = pa.decode_splitk_workspace_size(b.q.shape[0], w.num_q_heads, w.head_dim, max_ctx, partition_tokens,
                                               w.num_kv_heads)
        assert need <= bnd.NOALLOC_SCRATCH_BYTES
        ref = pa.decode_splitk(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale, w.softcap,
                               w.window, max_context_len=max_ctx, partition_tokens=partition_tokens)
        out = torch.full_like(b.q, float("nan"))
        assert _call_noalloc(b, w, out, partition_tokens, max_ctx) == bnd.PA_OK
        assert pa.last_decode_schedule() == schedule
        torch.cuda.synchronize()
        assert torch.equal(bits(out), bits(ref)), f"call {call}: differs from pa_decode_splitk"
        want = oracle.decode(b_cpu.q, b_cpu.k_cache, b_cpu.v_cache, b_cpu.block_tables, b_cpu.context_lens, w.scale,
                             w.softcap, w.window)
        assert_close(out, want, torch.bfloat16, f"{name} call {call}")
        assert pa.device_errors() == 0


def test_noalloc_python_wrapper():
    """The binding's decode_splitk_noalloc: writes the given ``out`` and returns it."""
    w = wl.WORKLOADS["gemma2_2b"]
    b_cpu = wl.make_batch(w, batch=20, prefilled=True)
    b = to_dev(b_cpu)
    out = torch.full_like(b.q, float("nan"))
    got = pa.decode_splitk_noalloc(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale, w.softcap,
                                   w.window, max_context_len=b_cpu.max_context_len, partition_tokens=0, out=out)
    torch.cuda.synchronize()
    assert got.data_ptr() == out.data_ptr()
    want = oracle.decode(b_cpu.q, b_cpu.k_cache, b_cpu.v_cache, b_cpu.block_tables, b_cpu.context_lens, w.scale,
                         w.softcap, w.window)
    assert_close(out, want, torch.bfloat16, "python wrapper")
    assert pa.device_errors() == 0


def test_noalloc_refuses_requests_beyond_its_scratch():
    w = wl.WORKLOADS["long_splitk"]
    b = wl.make_batch(w, lengths=[16], device="cuda", prefilled=True)
    out = torch.empty_like(b.q)
    big = 1 << 28  # a context bound whose partials would not fit in the fixed scratch
    need = pa.decode_splitk_workspace_size(1, w.num_q_heads, w.head_dim, big, 64, w.num_kv_heads)
    assert need > bnd.NOALLOC_SCRATCH_BYTES
    assert _call_noalloc(b, w, out, 64, big) == bnd.PA_ERR_WORKSPACE
    with pytest.raises(pa.PagedAttnError):
        pa.decode_splitk_noalloc(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale,
                                 max_context_len=big, partition_tokens=64, out=out)
