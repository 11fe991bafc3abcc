"""GPU parity of multi-query paged attention (pa_decode_multi) against the CPU
oracle: T new query tokens per sequence, already appended, attending causally
over the paged cache.  Each case runs the same seeded inputs through the C ABI
and through ``oracle.decode_multi`` and compares element by element within the
decode tolerances (bf16: max-abs 2e-2, mean-abs 2e-3)."""

import pytest
import torch

import oracle
import paged_kv_cache_473_b200 as pa
from paged_kv_cache_473_b200 import workloads as wl
from tests.gpu_helpers import assert_close, bits, to_dev

pytestmark = pytest.mark.gpu

REDUCED = {
    "tinyllama_1b": dict(batch=6),
    "gemma2_2b": dict(batch=6),
    "llama3_8b": dict(batch=8, max_len=3000),
    "long_splitk": dict(lengths=[16384 + 37, 1, 1000]),
}


@pytest.fixture(autouse=True)
def _clear_device_errors():
    if torch.cuda.is_available():
        pa.device_errors()
    yield


def _case(name, T, **extra):
    w = wl.WORKLOADS[name]
    kw = dict(REDUCED[name])
    kw.update(extra)
    if "lengths" in kw:
        kw.pop("batch", None)
    kw = {k: v for k, v in kw.items() if v is not None}
    b_cpu = wl.make_batch(w, prefilled=True, **kw)
    mq = wl.make_multi_queries(b_cpu, T)
    return w, b_cpu, to_dev(b_cpu), mq


def _run(w, b, q, split, partition, window=None, softcap=None, max_ctx=None):
    win = w.window if window is None else window
    cap = w.softcap if softcap is None else softcap
    mx = max_ctx if max_ctx is not None else max(1, b.max_context_len)
    out = pa.decode_multi(q.cuda(), b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale, cap, win,
                          split=split, max_context_len=mx, partition_tokens=partition)
    torch.cuda.synchronize()
    return out


def _ref(w, b_cpu, q, window=None, softcap=None, rows=None):
    win = w.window if window is None else window
    cap = w.softcap if softcap is None else softcap
    return oracle.decode_multi(q, b_cpu.k_cache, b_cpu.v_cache, b_cpu.block_tables, b_cpu.context_lens, w.scale,
                               cap, win, rows=rows)


@pytest.mark.parametrize("name,T", [("tinyllama_1b", 1), ("tinyllama_1b", 2), ("tinyllama_1b", 3), ("tinyllama_1b", 4),
                                    ("tinyllama_1b", 8), ("gemma2_2b", 5), ("gemma2_2b", 32), ("llama3_8b", 3),
                                    ("llama3_8b", 4), ("llama3_8b", 16), ("long_splitk", 4), ("long_splitk", 6)])
@pytest.mark.parametrize("split,partition", [(False, 0), (True, 0), (True, 64)])
def test_multi_parity(name, T, split, partition):
    w, b_cpu, b, mq = _case(name, T)
    out = _run(w, b, mq["q"], split, partition)
    ref = _ref(w, b_cpu, mq["q"])
    assert_close(out, ref, torch.bfloat16, f"multi {name} T={T} split={split} P={partition}")
    assert pa.device_errors() == 0


@pytest.mark.parametrize("window", [1, 3, 17, 200])
@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("T", [4, 6])
def test_multi_window_per_query_token(window, split, T):
    """Each query token has its own window start (T = 4: 16 query rows per kv
    head, the warp-per-item path when split; T = 6: the CTA-shared path)."""
    w, b_cpu, b, mq = _case("llama3_8b", T)
    out = _run(w, b, mq["q"], split, 64, window=window)
    ref = _ref(w, b_cpu, mq["q"], window=window)
    assert_close(out, ref, torch.bfloat16, f"multi window={window} split={split}")


@pytest.mark.parametrize("window", [1, 5, 40])
@pytest.mark.parametrize("T", [3, 4])
def test_multi_window_two_row_tiles(window, T):
    """head_dim 64 with 24 and 32 query rows per kv head: two 16-row tiles per
    warp on the warp-per-item path, the second partly padding at T = 3."""
    w, b_cpu, b, mq = _case("tinyllama_1b", T)
    out = _run(w, b, mq["q"], True, 0, window=window)
    ref = _ref(w, b_cpu, mq["q"], window=window)
    assert_close(out, ref, torch.bfloat16, f"multi two tiles window={window} T={T}")


@pytest.mark.parametrize("window", [1, 20, 300])
@pytest.mark.parametrize("T", [5, 8])
def test_multi_window_head_dim_256(window, T):
    """head_dim 256 (softcap 50) with 10 and 16 query rows per kv head: the
    rows kernel's one 16-row tile per warp, per-row windows."""
    w, b_cpu, b, mq = _case("gemma2_2b", T)
    out = _run(w, b, mq["q"], True, 0, window=window)
    ref = _ref(w, b_cpu, mq["q"], window=window)
    assert_close(out, ref, torch.bfloat16, f"multi head_dim 256 window={window} T={T}")


@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("name,T", [("tinyllama_1b", 5), ("tinyllama_1b", 2), ("tinyllama_1b", 4), ("llama3_8b", 4),
                                    ("gemma2_2b", 8)])
def test_multi_short_and_empty_sequences(split, name, T):
    """L = 0 rows, L < T (early query tokens see nothing: zero rows), L = T,
    ranges inside one slice and across block edges."""
    lengths = [0, 2, 5, 1, 17, 33, 64]
    w, b_cpu, b, mq = _case(name, T, lengths=lengths, max_len=None)
    out = _run(w, b, mq["q"], split, 64, max_ctx=64)
    ref = _ref(w, b_cpu, mq["q"])
    assert_close(out, ref, torch.bfloat16, f"multi short {name} T={T} split={split}")
    assert torch.count_nonzero(out[0]).item() == 0
    for i, L in enumerate(lengths):
        if L < T:  # query tokens before the first position
            assert torch.count_nonzero(out[i, : T - L]).item() == 0


def test_multi_softcap_and_verify_flow():
    """The speculative-verify flow: append the T draft rows with pa_write_kv
    (bit-exact against the oracle's append), then attend them causally."""
    w = wl.WORKLOADS["gemma2_2b"]
    T = 4
    b_cpu = wl.make_batch(w, batch=5, prefilled=True)
    mq = wl.make_multi_queries(b_cpu, T)
    b = to_dev(b_cpu)
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    pa.write_kv(mq["k_new"].cuda(), mq["v_new"].cuda(), mq["slot_mapping"].cuda(), kc, vc)
    out = pa.decode_multi(mq["q"].cuda(), kc, vc, b.block_tables, b.context_lens, w.scale, w.softcap, 0,
                          split=True, max_context_len=b_cpu.max_context_len, partition_tokens=0)
    torch.cuda.synchronize()
    kc_ref, vc_ref = b_cpu.k_cache.clone(), b_cpu.v_cache.clone()
    oracle.write_kv(mq["k_new"], mq["v_new"], mq["slot_mapping"], kc_ref, vc_ref)
    assert torch.equal(bits(kc), bits(kc_ref)) and torch.equal(bits(vc), bits(vc_ref))
    ref = oracle.decode_multi(mq["q"], kc_ref, vc_ref, b_cpu.block_tables, b_cpu.context_lens, w.scale, w.softcap, 0)
    assert_close(out, ref, torch.bfloat16, "multi verify flow, softcap 50")


def test_multi_block_permutation_invariance():
    w, b_cpu, b, mq = _case("llama3_8b", 4)
    q = mq["q"].cuda()
    base = pa.decode_multi(q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale, split=False)
    nb = b.k_cache.shape[0]
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(3)).cuda()
    kc2, vc2 = torch.empty_like(b.k_cache), torch.empty_like(b.v_cache)
    kc2[perm] = b.k_cache
    vc2[perm] = b.v_cache
    t2 = b.block_tables.clone()
    m = t2 >= 0
    t2[m] = perm[t2[m].long()].to(torch.int32)
    moved = pa.decode_multi(q, kc2, vc2, t2, b.context_lens, w.scale, split=False)
    torch.cuda.synchronize()
    assert torch.equal(bits(base), bits(moved))


@pytest.mark.parametrize("name,T", [("llama3_8b", 4), ("tinyllama_1b", 8)])
def test_multi_full_size_sampled_rows(name, T):
    """The full-size shape, library-chosen split; sampled rows against the oracle."""
    w = wl.WORKLOADS[name]
    b = wl.make_batch(w, prefilled=True, device="cuda")
    mq = wl.make_multi_queries(b, T)
    out = pa.decode_multi(mq["q"], b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale, w.softcap,
                          w.window, split=True, max_context_len=b.max_context_len, partition_tokens=0)
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(11)
    B = b.context_lens.numel()
    rows = [(int(i), int(j), int(h)) for i, j, h in zip(torch.randint(0, B, (40,), generator=g),
                                                         torch.randint(0, T, (40,), generator=g),
                                                         torch.randint(0, w.num_q_heads, (40,), generator=g))]
    L = b.context_lens.cpu()
    rows += [(int(L.argmax()), T - 1, 0), (int(L.argmin()), 0, w.num_q_heads - 1)]
    ref = oracle.decode_multi(mq["q"].cpu(), b.k_cache.cpu(), b.v_cache.cpu(), b.block_tables.cpu(), L, w.scale,
                              w.softcap, w.window, rows=rows)
    got = torch.stack([out[i, j, h] for i, j, h in rows])
    assert_close(got, ref, torch.bfloat16, f"{name} full-size multi T={T}")
    assert pa.device_errors() == 0
