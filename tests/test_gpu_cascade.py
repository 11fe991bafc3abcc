"""GPU parity of the cascade decode (pa_decode_cascade) against the CPU
oracle: batches where the first sequences share a prefix of full blocks (the
Llama-3-8B shape's 30% sharers of 64 prefix blocks, and the other heads).  The
cascade is an exact reformulation of decode, so the oracle is plain decode on
the same inputs; tolerances are the decode ones."""

import pytest
import torch

import oracle
import paged_kv_cache_473_b200 as pa
from paged_kv_cache_473_b200 import workloads as wl
from tests.gpu_helpers import assert_close, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_device_errors():
    if torch.cuda.is_available():
        pa.device_errors()
    yield


def _batch(name, **kw):
    w = wl.WORKLOADS[name]
    b_cpu, n_sh, plen = wl.order_for_cascade(wl.make_batch(w, prefilled=True, **kw))
    return w, b_cpu, to_dev(b_cpu), n_sh, plen


def _cascade(w, b, n_sh, plen, partition=0, window=None):
    win = w.window if window is None else window
    out = pa.decode_cascade(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale, w.softcap, win,
                            n_sharers=n_sh, prefix_len=plen, max_context_len=b.max_context_len,
                            partition_tokens=partition)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("partition", [0, 256, 512, 1024])
def test_cascade_llama3_prefix_sharing(partition):
    w, b_cpu, b, n_sh, plen = _batch("llama3_8b", batch=40, max_len=3000)
    assert n_sh >= 4 and plen == 1024
    out = _cascade(w, b, n_sh, plen, partition)
    assert pa.last_launch_count() == 3
    ref = oracle.decode_batch(b_cpu)
    assert_close(out, ref, torch.bfloat16, f"cascade P={partition}")
    assert pa.device_errors() == 0


@pytest.mark.parametrize("window", [100, 700, 1500])
def test_cascade_with_a_window(window):
    """Windows that start inside the prefix, and ones that skip it entirely."""
    w, b_cpu, b, n_sh, plen = _batch("llama3_8b", batch=24, max_len=3000)
    out = _cascade(w, b, n_sh, plen, 256, window=window)
    ref = oracle.decode_batch(b_cpu, window=window)
    assert_close(out, ref, torch.bfloat16, f"cascade window={window}")


@pytest.mark.parametrize("name,prefix_blocks", [("tinyllama_1b", 40), ("gemma2_2b", 4)])
def test_cascade_other_heads(name, prefix_blocks):
    """G = 8 (8 sharers per prefix CTA) and G = 2 with 128-token blocks, softcap 50."""
    w = wl.WORKLOADS[name].replace(prefix_share=0.5, prefix_blocks=prefix_blocks)
    b_cpu, n_sh, plen = wl.order_for_cascade(wl.make_batch(w, prefilled=True, batch=20))
    b = to_dev(b_cpu)
    assert n_sh >= 2 and plen > 0
    out = _cascade(w, b, n_sh, plen)
    ref = oracle.decode_batch(b_cpu)
    assert_close(out, ref, torch.bfloat16, f"cascade {name}")


def test_cascade_without_sharers_is_split_k():
    w, b_cpu, b, n_sh, plen = _batch("llama3_8b", batch=12, max_len=2000)
    out = pa.decode_cascade(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale, n_sharers=0,
                            prefix_len=plen, max_context_len=b.max_context_len)
    torch.cuda.synchronize()
    assert_close(out, oracle.decode_batch(b_cpu), torch.bfloat16, "cascade, no sharers")


def test_cascade_reports_a_sharer_whose_table_differs():
    w, b_cpu, b, n_sh, plen = _batch("llama3_8b", batch=24, max_len=3000)
    tables = b.block_tables.clone()
    tables[1, 3] = tables[n_sh, 0]  # sharer 1 points elsewhere inside the prefix
    pa.decode_cascade(b.q, b.k_cache, b.v_cache, tables, b.context_lens, w.scale, n_sharers=n_sh, prefix_len=plen,
                      max_context_len=b.max_context_len)
    torch.cuda.synchronize()
    assert pa.device_errors() & pa.DEVERR_BLOCK


def test_cascade_full_size_sampled_rows():
    w = wl.WORKLOADS["llama3_8b"]
    b, n_sh, plen = wl.order_for_cascade(wl.make_batch(w, prefilled=True, device="cuda"))
    out = pa.decode_cascade(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale, n_sharers=n_sh,
                            prefix_len=plen, max_context_len=b.max_context_len)
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(5)
    rows = [(int(i), int(h)) for i, h in zip(torch.randint(0, 128, (40,), generator=g),
                                             torch.randint(0, 32, (40,), generator=g))]
    rows += [(0, 0), (n_sh - 1, 31), (n_sh, 5)]
    ref = oracle.decode(b.q.cpu(), b.k_cache.cpu(), b.v_cache.cpu(), b.block_tables.cpu(), b.context_lens.cpu(),
                        w.scale, rows=rows)
    got = torch.stack([out[i, h] for i, h in rows])
    assert_close(got, ref, torch.bfloat16, "full-size cascade")
    assert pa.device_errors() == 0
