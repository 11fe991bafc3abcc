"""GPU parity of paged prefill (pa_prefill) against the CPU oracle: prompts (or
prompt chunks) of different lengths appended into the paged cache and attended
causally.  The append must be bit-exact; the attention within the decode
tolerances (bf16: max-abs 2e-2, mean-abs 2e-3)."""

import pytest
import torch

import oracle
import paged_kv_cache_473_b200 as pa
from paged_kv_cache_473_b200 import workloads as wl
from tests.gpu_helpers import assert_close, bits, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_device_errors():
    if torch.cuda.is_available():
        pa.device_errors()
    yield


def _run(name, lengths, q_lens, window=None, softcap=None, append=True):
    w = wl.WORKLOADS[name].replace(prefix_share=0.0)
    b_cpu = wl.make_batch(w, lengths=lengths, prefilled=True)
    x = wl.make_prefill_inputs(b_cpu, q_lens)
    b = to_dev(b_cpu)
    win = w.window if window is None else window
    cap = w.softcap if softcap is None else softcap
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    out = pa.prefill(dev["q"], dev["k_new"] if append else None, dev["v_new"] if append else None,
                     dev["slot_mapping"] if append else None, dev["cu_q_lens"], kc, vc, b.block_tables,
                     b.context_lens, w.scale, cap, win, max_q_len=x["max_q_len"])
    torch.cuda.synchronize()
    kc_ref, vc_ref = b_cpu.k_cache.clone(), b_cpu.v_cache.clone()
    ref = oracle.prefill(x["q"], x["k_new"] if append else None, x["v_new"], x["slot_mapping"], x["cu_q_lens"],
                         kc_ref, vc_ref, b_cpu.block_tables, b_cpu.context_lens, w.scale, cap, win)
    return w, out, ref, (kc, vc), (kc_ref, vc_ref)


@pytest.mark.parametrize("name", ["tinyllama_1b", "gemma2_2b", "llama3_8b"])
def test_prefill_prompts_from_scratch(name):
    """Whole prompts: every context position is new (T_b = L_b), ragged lengths
    spanning several query tiles and a partial last tile."""
    lengths = [1, 9, 64, 130, 257, 700]
    w, out, ref, (kc, vc), (kc_ref, vc_ref) = _run(name, lengths, lengths)
    assert pa.device_errors() == 0
    assert torch.equal(bits(kc), bits(kc_ref)) and torch.equal(bits(vc), bits(vc_ref))
    assert_close(out, ref, torch.bfloat16, f"prefill {name}")


@pytest.mark.parametrize("name", ["tinyllama_1b", "llama3_8b"])
def test_chunked_prefill_over_an_existing_context(name):
    """A chunk of new tokens on top of cached positions, and sequences with no
    new token in this call."""
    lengths = [300, 45, 1000, 17, 64]
    q_lens = [100, 45, 7, 0, 33]
    w, out, ref, (kc, vc), (kc_ref, vc_ref) = _run(name, lengths, q_lens)
    assert torch.equal(bits(kc), bits(kc_ref)) and torch.equal(bits(vc), bits(vc_ref))
    assert_close(out, ref, torch.bfloat16, f"chunked prefill {name}")


@pytest.mark.parametrize("window", [1, 16, 100])
def test_prefill_window_and_softcap(window):
    lengths = [200, 77]
    w, out, ref, _, _ = _run("gemma2_2b", lengths, [150, 77], window=window)
    assert_close(out, ref, torch.bfloat16, f"prefill window={window} softcap 50")


@pytest.mark.parametrize("name", ["tinyllama_1b", "llama3_8b"])
@pytest.mark.parametrize("window", [1, 33, 200])
def test_prefill_window_small_heads(name, window):
    """Sliding windows at head_dim 64 and 128: windows that start inside a
    64-token K/V tile and ones spanning several."""
    lengths = [300, 129, 17]
    w, out, ref, _, _ = _run(name, lengths, [260, 129, 17], window=window)
    assert_close(out, ref, torch.bfloat16, f"prefill {name} window={window}")


@pytest.mark.parametrize("name", ["tinyllama_1b", "llama3_8b"])
def test_prefill_softcap_small_heads(name):
    lengths = [200, 77]
    w, out, ref, _, _ = _run(name, lengths, lengths, softcap=30.0)
    assert_close(out, ref, torch.bfloat16, f"prefill {name} softcap 30")


@pytest.mark.parametrize("name", ["tinyllama_1b", "llama3_8b"])
def test_prefill_query_tile_edges(name):
    """Prompt lengths at the edges of a CTA's query tile (16 or 32 tokens with
    8 or 4 query heads per kv head) and of 64- and 128-token K/V spans: the
    last tile partly filled, and K/V ranges ending inside or at the end of a
    tile."""
    lengths = [15, 16, 17, 31, 32, 33, 63, 64, 65, 127, 128, 129]
    w, out, ref, (kc, vc), (kc_ref, vc_ref) = _run(name, lengths, lengths)
    assert torch.equal(bits(kc), bits(kc_ref)) and torch.equal(bits(vc), bits(vc_ref))
    assert_close(out, ref, torch.bfloat16, f"prefill edges {name}")


def test_prefill_attend_only():
    """k_new = v_new = NULL: the rows are already in the cache."""
    lengths = [120, 33]
    w, out, ref, _, _ = _run("llama3_8b", lengths, [40, 33], append=False)
    assert_close(out, ref, torch.bfloat16, "prefill without append")


def test_prefill_bad_offsets_are_reported_not_written():
    w = wl.WORKLOADS["tinyllama_1b"]
    b = wl.make_batch(w, lengths=[40, 40], prefilled=True, device="cuda")
    x = wl.make_prefill_inputs(b, [10, 10])
    cu = torch.tensor([0, 10, 30], dtype=torch.int32, device="cuda")  # past total_q = 20
    out = torch.full_like(x["q"], 7.0)
    pa.prefill(x["q"], None, None, None, cu, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale,
               max_q_len=20, out=out)
    torch.cuda.synchronize()
    assert pa.device_errors() & pa.DEVERR_CONTEXT
    assert torch.all(out[10:] == 7.0)  # the malformed sequence's rows are untouched


@pytest.mark.parametrize("name,lengths", [("llama3_8b", [1024] * 16), ("tinyllama_1b", [37, 2047, 512, 1300, 64, 999]),
                                          ("gemma2_2b", [1024, 333, 700])])
def test_prefill_full_size_sampled_rows(name, lengths):
    """The measured prefill workload (16 prompts x 1024 tokens) and ragged long
    prompts: sampled rows against the oracle (each row is a causal attention
    over up to 2047 positions)."""
    w = wl.WORKLOADS[name].replace(prefix_share=0.0)
    b = wl.make_batch(w, lengths=lengths, device="cuda")
    x = wl.make_prefill_inputs(b, lengths)
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    out = pa.prefill(x["q"], x["k_new"], x["v_new"], x["slot_mapping"], x["cu_q_lens"], kc, vc, b.block_tables,
                     b.context_lens, w.scale, w.softcap, w.window, max_q_len=x["max_q_len"])
    torch.cuda.synchronize()
    assert pa.device_errors() == 0
    cu = x["cu_q_lens"].tolist()
    g = torch.Generator().manual_seed(17)
    picks = []
    for bi, L in enumerate(lengths):
        for j in sorted(set([0, L - 1] + torch.randint(0, L, (4,), generator=g).tolist())):
            picks.append((bi, j, int(torch.randint(0, w.num_q_heads, (1,), generator=g))))
    # oracle: each picked row is a decode over its own prefix of the appended cache
    kc_cpu, vc_cpu = kc.cpu(), vc.cpu()
    tables, q = b.block_tables.cpu(), x["q"].cpu()
    for bi, j, h in picks:
        lens = torch.tensor([j + 1], dtype=torch.int32)
        ref = oracle.decode(q[cu[bi] + j].unsqueeze(0), kc_cpu, vc_cpu, tables[bi:bi + 1], lens, w.scale, w.softcap,
                            w.window, rows=[(0, h)])
        assert_close(out[cu[bi] + j, h].unsqueeze(0), ref, torch.bfloat16, f"{name} prompt {bi} token {j} head {h}")
