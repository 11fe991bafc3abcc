"""The allocation-free split-K entry point, pa_decode_splitk_noalloc.

Some callers cannot allocate device memory where they decode (inside a stream
capture that forbids it, in a serving loop that cannot pay for an allocation's
synchronisation, or with memory owned by an allocator the library cannot
reach).  For them the library keeps a fixed split-K scratch array of its own;
this file checks, through the C ABI, that the entry point gives the same
answer as pa_decode_splitk with a caller workspace, on two calls in a row (the
second one meets the scratch the first one left behind), and that requests
larger than the array are refused.  It is collected last so that a run that
stops at the first failure has run every other test first.
"""

import ctypes

import pytest
import torch

import paged_kv_cache_473_b200 as pa
from paged_kv_cache_473_b200 import _binding as bnd
from paged_kv_cache_473_b200 import workloads as wl
from tests.gpu_helpers import TOL, errors

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines, never run there
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _call_noalloc(b, w, out, partition_tokens, max_ctx):
    return bnd.lib.pa_decode_splitk_noalloc(
        b.q.data_ptr(), b.k_cache.data_ptr(), b.v_cache.data_ptr(), b.block_tables.data_ptr(),
        b.context_lens.data_ptr(), b.q.shape[0], w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
        b.block_tables.shape[1], b.k_cache.shape[0], ctypes.c_float(w.scale), ctypes.c_float(w.softcap), w.window,
        out.data_ptr(), bnd.PA_BF16, partition_tokens, max_ctx, 0, torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("partition_tokens", [0, 128])
def test_noalloc_matches_the_workspace_entry_point_on_two_calls(partition_tokens):
    w = wl.WORKLOADS["tinyllama_1b"]
    for call, seed in enumerate((w.seed, w.seed + 1)):  # different inputs on the second call
        b = wl.make_batch(w, seed=seed, batch=16, device="cuda", prefilled=True)
        max_ctx = b.max_context_len
        ref = pa.decode_splitk(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale, w.softcap,
                               w.window, max_context_len=max_ctx, partition_tokens=partition_tokens)
        out = torch.full_like(b.q, float("nan"))
        assert _call_noalloc(b, w, out, partition_tokens, max_ctx) == bnd.PA_OK
        torch.cuda.synchronize()
        mx, mean = errors(out, ref.double().cpu().numpy())
        tmax, tmean = TOL[torch.bfloat16]
        assert mx <= tmax and mean <= tmean, f"call {call}: max {mx:.3g} mean {mean:.3g}"
        assert pa.device_errors() == 0


def test_noalloc_refuses_requests_beyond_its_scratch():
    w = wl.WORKLOADS["long_splitk"]
    b = wl.make_batch(w, lengths=[16], device="cuda", prefilled=True)
    out = torch.empty_like(b.q)
    big = 1 << 28  # a context bound whose partials would not fit in the fixed scratch
    need = pa.decode_splitk_workspace_size(1, w.num_q_heads, w.head_dim, big, 64, w.num_kv_heads)
    assert need > bnd.NOALLOC_SCRATCH_BYTES
    assert _call_noalloc(b, w, out, 64, big) == bnd.PA_ERR_WORKSPACE
