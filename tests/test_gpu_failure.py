"""Failure detection on the GPU without a fault: a wait that nothing completes
gives up after its bound and reports PA_DEVERR_TIMEOUT through the device
error word, and the context stays usable for the next call."""

import pytest
import torch

import paged_kv_cache_473_b200 as pa
from paged_kv_cache_473_b200 import workloads as wl
from tests.gpu_helpers import assert_close, oracle_step, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit_ns", [1_000_000, 20_000_000])
def test_bounded_wait_gives_up_and_reports(limit_ns):
    pa.device_errors(clear=True)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    pa.check_bounded_wait(limit_ns)
    end.record()
    torch.cuda.synchronize()
    assert pa.device_errors() & pa.DEVERR_TIMEOUT
    ms = start.elapsed_time(end)
    assert limit_ns / 1e6 <= ms < limit_ns / 1e6 + 50  # it waited its bound, then returned

    # The context is intact: a decode step right after is correct and raises nothing.
    w = wl.WORKLOADS["tinyllama_1b"]
    bc = wl.make_batch(w, batch=4, max_len=300)
    b = to_dev(bc)
    out = pa.decode_step(b.q, b.k_new, b.v_new, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale,
                         split=True, max_context_len=b.max_context_len)
    torch.cuda.synchronize()
    ref, _, _ = oracle_step(bc)
    assert_close(out, ref, torch.bfloat16, "decode after a timed-out wait")
    assert pa.device_errors() == 0
