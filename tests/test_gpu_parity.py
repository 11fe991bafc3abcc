"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle
on the same seeded inputs.

Append: bit-exact.  Decode: within max-abs / mean-abs 2e-2 / 2e-3 (bf16 inputs,
fp32 accumulation) or 1e-4 / 1e-5 (fp32), of the fp64 oracle.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_473_b200 as pa
from paged_kv_cache_473_b200 import workloads as wl
from tests.gpu_helpers import TOL, assert_close, bits, errors, gpu_step, oracle_step, to_dev
from tests.paging_helpers import scatter_to_pool

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines, never run there
    pytest.skip("needs a CUDA device", allow_module_level=True)

# Sizes the oracle finishes in seconds that still span many 16-token slices,
# several partitions and ragged tails.
REDUCED = {
    "tiny_fp32": dict(),
    "tinyllama_1b": dict(batch=8),
    "gemma2_2b": dict(batch=12),
    "llama3_8b": dict(batch=16, max_len=3000),
    "long_splitk": dict(lengths=[16384 + 37, 19999, 1, 1000]),
}


@pytest.fixture(autouse=True)
def _clear_device_errors():
    pa.device_errors(clear=True)
    yield


def _reduced(name, **extra):
    w = wl.WORKLOADS[name]
    kw = dict(REDUCED[name])
    kw.update(extra)
    b_cpu = wl.make_batch(w, **kw)
    return w, b_cpu, to_dev(b_cpu)


@pytest.mark.parametrize("name", list(wl.WORKLOADS))
def test_write_kv_is_bit_exact(name):
    w, b_cpu, b = _reduced(name)
    _, kc, vc = gpu_step(b)
    _, kc_ref, vc_ref = oracle_step(b_cpu)
    assert torch.equal(bits(kc), bits(kc_ref))
    assert torch.equal(bits(vc), bits(vc_ref))
    assert pa.device_errors() == 0


def test_write_kv_skips_padding_and_flags_bad_slots():
    w = wl.WORKLOADS["tinyllama_1b"]
    b_cpu = wl.make_batch(w, batch=4, max_len=300)
    b = to_dev(b_cpu)
    slots = b.slot_mapping.clone()
    slots[1] = -1
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    pa.write_kv(b.k_new, b.v_new, slots, kc, vc)
    kc_ref, vc_ref = b_cpu.k_cache.clone(), b_cpu.v_cache.clone()
    oracle.write_kv(b_cpu.k_new, b_cpu.v_new, slots.cpu(), kc_ref, vc_ref)
    assert torch.equal(bits(kc), bits(kc_ref)) and torch.equal(bits(vc), bits(vc_ref))
    assert pa.device_errors() == 0
    slots[2] = b.num_blocks * w.block_size  # one past the pool: skipped and reported
    kc2 = b.k_cache.clone()
    vc2 = b.v_cache.clone()
    pa.write_kv(b.k_new, b.v_new, slots, kc2, vc2)
    assert pa.device_errors() & pa.DEVERR_SLOT


@pytest.mark.parametrize("name", list(wl.WORKLOADS))
@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("kernel", ["auto", "cuda_core"])
def test_step_parity(name, split, kernel):
    w, b_cpu, b = _reduced(name)
    out, _, _ = gpu_step(b, kernel=kernel, split=split, partition=w.partition_tokens)
    ref, _, _ = oracle_step(b_cpu)
    assert_close(out, ref, w.torch_dtype, f"{name} split={split} kernel={kernel}")
    assert pa.device_errors() == 0


@pytest.mark.parametrize("window", [4096, 1, 64, 200, 300, 511])
@pytest.mark.parametrize("split", [False, True])
def test_gemma_softcap_and_sliding_window(window, split):
    w, b_cpu, b = _reduced("gemma2_2b")
    out, _, _ = gpu_step(b, split=split, partition=128, window=window)
    ref, _, _ = oracle_step(b_cpu, window=window)
    assert_close(out, ref, w.torch_dtype, f"window={window}")


@pytest.mark.parametrize("partition", [64, 256, 512, 1024])
def test_splitk_is_invariant_to_partition_size(partition):
    w, b_cpu, b = _reduced("long_splitk")
    out, _, _ = gpu_step(b, split=True, partition=partition)
    ref, _, _ = oracle_step(b_cpu)
    assert_close(out, ref, w.torch_dtype, f"partition={partition}")


@pytest.mark.parametrize("kernel", ["auto", "cuda_core"])
def test_one_partition_splitk_is_bit_identical_to_decode(kernel):
    w, b_cpu, b = _reduced("tinyllama_1b")
    a, _, _ = gpu_step(b, kernel=kernel)
    s, _, _ = gpu_step(b, kernel=kernel, split=True, partition=2048)
    assert torch.equal(bits(a), bits(s))


@pytest.mark.parametrize("kernel", ["auto", "cuda_core"])
@pytest.mark.parametrize("split", [False, True])
def test_block_permutation_invariance_is_bit_exact(kernel, split):
    w, b_cpu, b = _reduced("llama3_8b")
    base, kc, vc = gpu_step(b, kernel=kernel, split=split, partition=256)
    nb = kc.shape[0]
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(5)).cuda()
    kc2, vc2 = torch.empty_like(kc), torch.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    t2 = b.block_tables.clone()
    m = t2 >= 0
    t2[m] = perm[t2[m].long()].to(torch.int32)
    if split:
        out = pa.decode_splitk(b.q, kc2, vc2, t2, b.context_lens, w.scale, max_context_len=b.max_context_len,
                               partition_tokens=256, kernel=kernel)
    else:
        out = pa.decode(b.q, kc2, vc2, t2, b.context_lens, w.scale, kernel=kernel)
    torch.cuda.synchronize()
    assert torch.equal(bits(out), bits(base))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_context_of_length_one_returns_v_exactly(dtype, d):
    gen = torch.Generator().manual_seed(d)
    hkv, hq, B = 2, 8, 5
    ks = [torch.randn((1, hkv, d), generator=gen).to(dtype) for _ in range(B)]
    vs = [torch.randn((1, hkv, d), generator=gen).to(dtype) for _ in range(B)]
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 16, gen, dtype=dtype)
    q = (torch.randn((B, hq, d), generator=gen) * 30).to(dtype)
    kern = "auto"
    out = pa.decode(q.cuda(), kc.cuda(), vc.cuda(), tables.cuda(), cl.cuda(), 1 / math.sqrt(d), 10.0, 0, kernel=kern)
    torch.cuda.synchronize()
    for i in range(B):
        for h in range(hq):
            assert torch.equal(bits(out[i, h]), bits(vs[i][0, h // 4]))


def test_zero_length_context_gives_zero_rows():
    w, b_cpu, b = _reduced("tinyllama_1b", prefilled=True)
    cl = b.context_lens.clone()
    cl[3] = 0
    for split in (False, True):
        if split:
            out = pa.decode_splitk(b.q, b.k_cache, b.v_cache, b.block_tables, cl, w.scale,
                                   max_context_len=b.max_context_len, partition_tokens=64)
        else:
            out = pa.decode(b.q, b.k_cache, b.v_cache, b.block_tables, cl, w.scale)
        torch.cuda.synchronize()
        assert torch.count_nonzero(out[3]).item() == 0
        assert torch.isfinite(out.float()).all()


def test_infinite_softcap_is_bit_identical_to_no_softcap():
    w, b_cpu, b = _reduced("gemma2_2b")
    a, _, _ = gpu_step(b, softcap=0.0)
    c, _, _ = gpu_step(b, softcap=float("inf"))
    assert torch.equal(bits(a), bits(c))
    ref, _, _ = oracle_step(b_cpu, softcap=0.0)
    assert_close(a, ref, torch.bfloat16, "no softcap")


@pytest.mark.parametrize("split", [False, True])
def test_window_edges(split):
    """W = L-1, L, L+1 around one sequence's length, and W >= L equal to no window."""
    w, b_cpu, b = _reduced("tinyllama_1b")
    L0 = int(b_cpu.context_lens[0])
    base, _, _ = gpu_step(b, split=split, partition=64, window=0)
    for W in (L0 - 1, L0, L0 + 1, 1):
        out, _, _ = gpu_step(b, split=split, partition=64, window=W)
        ref, _, _ = oracle_step(b_cpu, window=W)
        assert_close(out, ref, torch.bfloat16, f"W={W}")
    big, _, _ = gpu_step(b, split=split, partition=64, window=1 << 20)
    assert torch.equal(bits(big), bits(base))


def test_identical_keys_give_mean_of_v():
    gen = torch.Generator().manual_seed(8)
    L, hkv, d = 700, 4, 128
    key = torch.randn((1, hkv, d), generator=gen)
    ks = [key.expand(L, hkv, d).clone().to(torch.bfloat16)]
    vs = [torch.randn((L, hkv, d), generator=gen).to(torch.bfloat16)]
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 16, gen, dtype=torch.bfloat16)
    q = torch.randn((1, 16, d), generator=gen).to(torch.bfloat16)
    out = pa.decode(q.cuda(), kc.cuda(), vc.cuda(), tables.cuda(), cl.cuda(), 0.09)
    torch.cuda.synchronize()
    for h in range(16):
        mean = vs[0][:, h // 4].double().mean(0).numpy()
        mx, _ = errors(out[0, h], mean)
        assert mx <= 2e-2


@pytest.mark.parametrize("hq,hkv", [(4, 4), (6, 2), (24, 3), (8, 1), (16, 2)])
@pytest.mark.parametrize("kernel", ["auto", "cuda_core"])
def test_group_sizes(hq, hkv, kernel):
    w = wl.WORKLOADS["llama3_8b"].replace(num_q_heads=hq, num_kv_heads=hkv, prefix_share=0.0)
    b_cpu = wl.make_batch(w, batch=6, max_len=900)
    b = to_dev(b_cpu)
    out, _, _ = gpu_step(b, kernel=kernel)
    ref, _, _ = oracle_step(b_cpu)
    assert_close(out, ref, torch.bfloat16, f"G={hq // hkv}")


@pytest.mark.parametrize("bs,d", [(16, 256), (32, 64), (64, 128), (256, 256), (256, 64)])
def test_block_sizes_and_head_dims(bs, d):
    w = wl.WORKLOADS["gemma2_2b"].replace(block_size=bs, head_dim=d)
    b_cpu = wl.make_batch(w, batch=5)
    b = to_dev(b_cpu)
    for split in (False, True):
        out, _, _ = gpu_step(b, split=split, partition=256)
        ref, _, _ = oracle_step(b_cpu)
        assert_close(out, ref, torch.bfloat16, f"bs={bs} d={d} split={split}")


def test_large_scores_stay_finite():
    w = wl.WORKLOADS["llama3_8b"]
    b_cpu = wl.make_batch(w, batch=6, max_len=1500, q_scale=100.0)
    b = to_dev(b_cpu)
    for split in (False, True):
        out, _, _ = gpu_step(b, split=split, partition=128)
        ref, _, _ = oracle_step(b_cpu)
        assert_close(out, ref, torch.bfloat16, f"q x100 split={split}")


def test_bad_block_id_and_long_context_are_reported_not_faulted():
    w, b_cpu, b = _reduced("tinyllama_1b")
    t = b.block_tables.clone()
    t[0, 0] = b.num_blocks + 5  # outside the pool: the tile is skipped
    pa.decode(b.q, b.k_cache, b.v_cache, t, b.context_lens, w.scale)
    assert pa.device_errors() & pa.DEVERR_BLOCK
    cl = b.context_lens.clone()
    cl[1] = b.max_blocks_per_seq * w.block_size + 1  # longer than the table: clamped
    pa.decode(b.q, b.k_cache, b.v_cache, b.block_tables, cl, w.scale)
    assert pa.device_errors() & pa.DEVERR_CONTEXT
    cl = b.context_lens.clone()
    pa.decode_splitk(b.q, b.k_cache, b.v_cache, b.block_tables, cl, w.scale,
                     max_context_len=int(cl.max().item()) - 1, partition_tokens=64)
    assert pa.device_errors() & pa.DEVERR_CONTEXT
    # The context stays usable.
    out, _, _ = gpu_step(b)
    ref, _, _ = oracle_step(b_cpu)
    assert_close(out, ref, torch.bfloat16, "after errors")
    assert pa.device_errors() == 0


# ---- full sizes, bench launch configuration, sampled rows -----------------------

FULL = ["tinyllama_1b", "gemma2_2b", "llama3_8b", "long_splitk"]
COUNTER_BYTES = 256 * 1024  # the split-K workspace's fixed counter region


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_rows(name):
    w = wl.WORKLOADS[name]
    b = wl.make_batch(w, device="cuda")
    cpu = dict(q=b.q.cpu(), k_new=b.k_new.cpu(), v_new=b.v_new.cpu(), slots=b.slot_mapping.cpu(),
               kc=b.k_cache.cpu(), vc=b.v_cache.cpu(), tables=b.block_tables.cpu(), lens=b.context_lens.cpu())
    out, _, _ = gpu_step(b, split=True, partition=w.partition_tokens)
    assert torch.isfinite(out.float()).all()
    assert pa.device_errors() == 0
    oracle.write_kv(cpu["k_new"], cpu["v_new"], cpu["slots"], cpu["kc"], cpu["vc"])
    g = torch.Generator().manual_seed(99)
    B, hq = w.batch, w.num_q_heads
    rows = [(int(i), int(h)) for i, h in zip(torch.randint(0, B, (48,), generator=g),
                                             torch.randint(0, hq, (48,), generator=g))]
    # Always include the longest and the shortest sequence.
    L = cpu["lens"]
    rows += [(int(L.argmax()), 0), (int(L.argmin()), hq - 1)]
    ref = oracle.decode(cpu["q"], cpu["kc"], cpu["vc"], cpu["tables"], cpu["lens"], w.scale, w.softcap, w.window,
                        rows=rows)
    got = torch.stack([out[i, h] for i, h in rows])
    assert_close(got, ref, w.torch_dtype, f"{name} full size, sampled rows")


# ---- fused decode step ------------------------------------------------------------


@pytest.mark.parametrize("name", list(wl.WORKLOADS))
@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("kernel", ["auto", "cuda_core"])
def test_fused_step_equals_append_then_decode_bit_for_bit(name, split, kernel):
    w, b_cpu, b = _reduced(name)
    ref_out, ref_kc, ref_vc = gpu_step(b, kernel=kernel, split=split, partition=w.partition_tokens)
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    out = pa.decode_step(b.q, b.k_new, b.v_new, kc, vc, b.block_tables, b.context_lens, w.scale, w.softcap,
                         w.window, split=split, max_context_len=max(1, b.max_context_len),
                         partition_tokens=w.partition_tokens, kernel=kernel)
    torch.cuda.synchronize()
    assert torch.equal(bits(out), bits(ref_out))
    assert torch.equal(bits(kc), bits(ref_kc)) and torch.equal(bits(vc), bits(ref_vc))
    ref, _, _ = oracle_step(b_cpu)
    assert_close(out, ref, w.torch_dtype, f"fused step {name} split={split} kernel={kernel}")
    assert pa.device_errors() == 0


@pytest.mark.parametrize("window", [0, 1, 100])
def test_fused_step_with_window_and_softcap(window):
    w, b_cpu, b = _reduced("gemma2_2b")
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    out = pa.decode_step(b.q, b.k_new, b.v_new, kc, vc, b.block_tables, b.context_lens, w.scale, w.softcap, window,
                         split=True, max_context_len=b.max_context_len, partition_tokens=128)
    torch.cuda.synchronize()
    ref, kc_ref, vc_ref = oracle_step(b_cpu, window=window)
    assert torch.equal(bits(kc), bits(kc_ref)) and torch.equal(bits(vc), bits(vc_ref))
    assert_close(out, ref, torch.bfloat16, f"fused step window={window}")


@pytest.mark.parametrize("name", FULL)
def test_full_size_fused_step_grid_schedule_sampled_rows(name):
    """The fused step on the fixed partition grid (the library's grid partition
    for the shape, given explicitly), at full size, on sampled rows.  The
    dynamic schedule that the benchmark times is compared on its whole output
    below."""
    w = wl.WORKLOADS[name]
    b = wl.make_batch(w, device="cuda")
    cpu = dict(q=b.q.cpu(), k_new=b.k_new.cpu(), v_new=b.v_new.cpu(), slots=b.slot_mapping.cpu(),
               kc=b.k_cache.cpu(), vc=b.v_cache.cpu(), tables=b.block_tables.cpu(), lens=b.context_lens.cpu())
    part = pa.decode_splitk_partition(w.batch, w.num_kv_heads, b.max_context_len, w.partition_tokens)
    out = pa.decode_step(b.q, b.k_new, b.v_new, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale,
                         w.softcap, w.window, split=True, max_context_len=b.max_context_len, partition_tokens=part)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    assert pa.device_errors() == 0
    oracle.write_kv(cpu["k_new"], cpu["v_new"], cpu["slots"], cpu["kc"], cpu["vc"])
    # The appended rows landed bit-exactly.
    L = cpu["lens"]
    bs = w.block_size
    for i in range(0, w.batch, max(1, w.batch // 16)):
        t = int(L[i]) - 1
        blk = int(cpu["tables"][i, t // bs])
        assert torch.equal(bits(b.k_cache[blk, :, t % bs]), bits(cpu["k_new"][i]))
        assert torch.equal(bits(b.v_cache[blk, :, t % bs]), bits(cpu["v_new"][i]))
    g = torch.Generator().manual_seed(7)
    rows = [(int(i), int(h)) for i, h in zip(torch.randint(0, w.batch, (48,), generator=g),
                                             torch.randint(0, w.num_q_heads, (48,), generator=g))]
    rows += [(int(L.argmax()), 1), (int(L.argmin()), 0)]
    ref = oracle.decode(cpu["q"], cpu["kc"], cpu["vc"], cpu["tables"], cpu["lens"], w.scale, w.softcap, w.window,
                        rows=rows)
    got = torch.stack([out[i, h] for i, h in rows])
    assert_close(got, ref, w.torch_dtype, f"{name} full-size fused step")


# ---- the benchmark's timed call, full size, whole output -----------------------------

# (workload, partition argument of bench.Runner): -1 is the workload's own
# schedule, the headline and per-shape lines of bench.py (the dynamic work
# queue, or the 512-token grid for the long split-K shape); the long shape is
# also timed on the dynamic schedule.
BENCH_STEPS = [("tinyllama_1b", -1), ("gemma2_2b", -1), ("llama3_8b", -1), ("long_splitk", -1), ("long_splitk", 0)]


@pytest.mark.parametrize("name,partition", BENCH_STEPS)
def test_full_size_timed_step_whole_output(name, partition):
    """The step bench.py times (bench.Runner.step: pa_decode_step with the
    runner's schedule, workspace and max_context_len), at the full workload
    size: every output element against the oracle (append, then decode),
    the whole cache after the step bit-exact against the oracle's append, and
    the workspace's counter region back at zero."""
    import bench

    w = wl.WORKLOADS[name]
    runner = bench.Runner(w, 0, "auto", True, partition, fused=True)
    b = runner.batch
    cpu = {k: getattr(b, k).cpu() for k in ("q", "k_new", "v_new", "slot_mapping", "k_cache", "v_cache",
                                            "block_tables", "context_lens")}
    runner.step(0)
    torch.cuda.synchronize()
    assert pa.device_errors() == 0
    if runner.partition == 0:
        assert int(runner.ws[:COUNTER_BYTES].view(torch.int32).abs().sum()) == 0
    oracle.write_kv(cpu["k_new"], cpu["v_new"], cpu["slot_mapping"], cpu["k_cache"], cpu["v_cache"])
    kc, vc = runner.pools[0]
    assert torch.equal(bits(kc), bits(cpu["k_cache"])), "key cache after the step"
    assert torch.equal(bits(vc), bits(cpu["v_cache"])), "value cache after the step"
    ref = oracle.decode(cpu["q"], cpu["k_cache"], cpu["v_cache"], cpu["block_tables"], cpu["context_lens"], w.scale,
                        w.softcap, w.window)
    assert_close(runner.out, ref, w.torch_dtype, f"{name} timed step (partition {runner.partition}), whole output")
    del runner
    torch.cuda.empty_cache()


# ---- dynamic (work-queue) split-K schedule ------------------------------------------
# partition_tokens == 0 on the tensor-core path: persistent CTAs claim
# (sequence, kv head, partition) items from a counter in the workspace.


@pytest.mark.parametrize("name", ["tinyllama_1b", "gemma2_2b", "llama3_8b", "long_splitk"])
@pytest.mark.parametrize("append", [False, True])
def test_dynamic_schedule_parity(name, append):
    w, b_cpu, b = _reduced(name)
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    if append:
        out = pa.decode_step(b.q, b.k_new, b.v_new, kc, vc, b.block_tables, b.context_lens, w.scale, w.softcap,
                             w.window, split=True, max_context_len=b.max_context_len, partition_tokens=0)
    else:
        pa.write_kv(b.k_new, b.v_new, b.slot_mapping, kc, vc)
        out = pa.decode_splitk(b.q, kc, vc, b.block_tables, b.context_lens, w.scale, w.softcap, w.window,
                               max_context_len=b.max_context_len, partition_tokens=0)
    torch.cuda.synchronize()
    ref, kc_ref, vc_ref = oracle_step(b_cpu)
    assert torch.equal(bits(kc), bits(kc_ref)) and torch.equal(bits(vc), bits(vc_ref))
    assert_close(out, ref, w.torch_dtype, f"dynamic {name} append={append}")
    assert pa.device_errors() == 0


@pytest.mark.parametrize("lengths", [[1, 2, 3], [0, 5, 0, 17], [1] * 40, [16, 32, 48, 64, 15, 17, 31, 33]])
def test_dynamic_schedule_short_and_empty_sequences(lengths):
    """Fewer items than CTAs, L = 0 rows, single-slice items."""
    w = wl.WORKLOADS["llama3_8b"].replace(prefix_share=0.0)
    b_cpu = wl.make_batch(w, lengths=lengths, prefilled=True)
    b = to_dev(b_cpu)
    out = pa.decode_splitk(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale,
                           max_context_len=max(1, max(lengths)), partition_tokens=0)
    torch.cuda.synchronize()
    ref, _, _ = oracle_step(b_cpu, append=False)
    assert_close(out, ref, torch.bfloat16, f"dynamic lengths={lengths}")
    for i, L in enumerate(lengths):
        if L == 0:
            assert torch.count_nonzero(out[i]).item() == 0


def test_dynamic_schedule_many_units_per_cta():
    """Many short sequences: thousands of items, prefix arrays of a large batch
    (the CTA-wide length scan)."""
    w = wl.WORKLOADS["llama3_8b"].replace(prefix_share=0.0, lengths=("uniform", 1, 40))
    b_cpu = wl.make_batch(w, batch=2000, prefilled=True)
    b = to_dev(b_cpu)
    out = pa.decode_splitk(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale,
                           max_context_len=b.max_context_len, partition_tokens=0)
    assert pa.last_decode_schedule() in ("dynamic", "dynamic_merged")
    torch.cuda.synchronize()
    rows = [(i, h) for i in range(0, 2000, 37) for h in (0, 13, 31)]
    ref = oracle.decode(b_cpu.q, b_cpu.k_cache, b_cpu.v_cache, b_cpu.block_tables, b_cpu.context_lens, w.scale,
                        rows=rows)
    got = torch.stack([out[i, h] for i, h in rows])
    assert_close(got, ref, torch.bfloat16, "dynamic, many items per CTA")
    assert pa.device_errors() == 0


def test_dynamic_schedule_block_permutation_invariance_and_workspace_reuse():
    w, b_cpu, b = _reduced("llama3_8b", prefilled=True)
    need = pa.decode_splitk_workspace_size(b.q.shape[0], w.num_q_heads, w.head_dim, b.max_context_len, 0,
                                           w.num_kv_heads)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")  # one workspace for every call
    kw = dict(max_context_len=b.max_context_len, partition_tokens=0, workspace=ws)
    base = pa.decode_splitk(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale, **kw)
    again = pa.decode_splitk(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale, **kw)
    nb = b.k_cache.shape[0]
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(9)).cuda()
    kc2, vc2 = torch.empty_like(b.k_cache), torch.empty_like(b.v_cache)
    kc2[perm] = b.k_cache
    vc2[perm] = b.v_cache
    t2 = b.block_tables.clone()
    m = t2 >= 0
    t2[m] = perm[t2[m].long()].to(torch.int32)
    moved = pa.decode_splitk(b.q, kc2, vc2, t2, b.context_lens, w.scale, **kw)
    torch.cuda.synchronize()
    assert torch.equal(bits(base), bits(again))
    assert torch.equal(bits(base), bits(moved))


def test_dynamic_schedule_counters_return_to_zero():
    """The merge and work counters live in the workspace and must read zero
    after every call: calls of different batches share one workspace, and every
    output row must be written (NaN-filled beforehand) and correct each time."""
    w = wl.WORKLOADS["tinyllama_1b"]
    # (batch, seed, partition_tokens): shapes shrink and grow, and a fixed-partition
    # call (grid schedule plus combine) writes its partials in between.
    calls = [(24, w.seed, 0), (9, w.seed + 5, 0), (24, w.seed + 6, 128), (24, w.seed, 0)]
    batches = [wl.make_batch(w, prefilled=True, batch=B, seed=sd) for B, sd, _ in calls]
    need = max(pa.decode_splitk_workspace_size(bc.q.shape[0], w.num_q_heads, w.head_dim, 2048, P, w.num_kv_heads)
               for bc, (_, _, P) in zip(batches, calls))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    outs = []
    for bc, (_, _, P) in zip(batches, calls):
        b = to_dev(bc)
        out = torch.full_like(b.q, float("nan"))
        pa.decode_splitk(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale,
                         max_context_len=2048, partition_tokens=P, out=out, workspace=ws)
        torch.cuda.synchronize()
        ref, _, _ = oracle_step(bc, append=False)
        assert not torch.isnan(out).any()
        assert_close(out, ref, torch.bfloat16, f"dynamic reuse batch={bc.q.shape[0]}")
        outs.append(out)
    assert torch.equal(bits(outs[0]), bits(outs[3]))
    assert pa.device_errors() == 0


@pytest.mark.parametrize("name,kw,max_ctx,schedule", [
    ("tinyllama_1b", dict(batch=48), None, "dynamic_merged"),  # fixed items cover the work, the last partial merges
    ("llama3_8b", dict(batch=64), None, "dynamic"),           # more items than 2 per warp (claims), combine kernel
    # at most 8 partitions but more than 2 items per warp: claims and the combine kernel
    ("gemma2_2b", dict(batch=256), None, "dynamic"),
    ("llama3_8b", dict(batch=128, max_len=2048), None, "dynamic"),
    ("tinyllama_1b", dict(batch=256), None, "dynamic"),
    # head_dim 64 merged by the combine: the 12-warp-per-SM configuration
    ("tinyllama_1b", dict(batch=128), None, "dynamic"),
])
def test_dynamic_schedule_counter_region_reads_zero_after_each_call(name, kw, max_ctx, schedule):
    """Whichever way the partitions are merged, and whether or not warps claim
    items from the work counter, the step matches the oracle and the
    workspace's counter region is all zero when the call ends (the next call
    relies on it)."""
    w = wl.WORKLOADS[name]
    bc = wl.make_batch(w, prefilled=False, **kw)
    b = to_dev(bc)
    mx = max_ctx or b.max_context_len
    need = pa.decode_splitk_workspace_size(bc.q.shape[0], w.num_q_heads, w.head_dim, mx, 0, w.num_kv_heads)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    for _ in range(2):
        out = pa.decode_step(b.q, b.k_new, b.v_new, kc, vc, b.block_tables, b.context_lens, w.scale, w.softcap,
                             w.window, split=True, max_context_len=mx, partition_tokens=0, workspace=ws)
        assert pa.last_decode_schedule() == schedule
        torch.cuda.synchronize()
        assert int(ws[:COUNTER_BYTES].view(torch.int32).abs().sum()) == 0
    ref, _, _ = oracle_step(bc)
    assert_close(out, ref, torch.bfloat16, f"{name} step")
    assert pa.device_errors() == 0


@pytest.mark.parametrize("batch,schedule", [(64, "dynamic_merged"), (48, "dynamic_merged")])
def test_in_kernel_merge_is_deterministic(batch, schedule):
    """At the headline shape (64 sequences, and at 48) the dynamic schedule
    merges each unit's partitions in the decode kernel, by whichever warp
    arrives last; the sums run in partition order, so repeated steps on the
    same inputs give the same bits."""
    w = wl.WORKLOADS["tinyllama_1b"]
    b = wl.make_batch(w, device="cuda", prefilled=True, batch=batch)
    need = pa.decode_splitk_workspace_size(batch, w.num_q_heads, w.head_dim, b.max_context_len, 0, w.num_kv_heads)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(12):
        outs.append(pa.decode_splitk(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale,
                                     max_context_len=b.max_context_len, partition_tokens=0, workspace=ws))
        assert pa.last_decode_schedule() == schedule
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(bits(o), bits(outs[0]))
    assert pa.device_errors() == 0


@pytest.mark.parametrize("window", [1, 100, 1000])
def test_dynamic_schedule_window(window):
    w, b_cpu, b = _reduced("tinyllama_1b", prefilled=True)
    out = pa.decode_splitk(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, w.scale, 0.0, window,
                           max_context_len=b.max_context_len, partition_tokens=0)
    torch.cuda.synchronize()
    ref, _, _ = oracle_step(b_cpu, window=window, append=False)
    assert_close(out, ref, torch.bfloat16, f"dynamic window={window}")


# Shapes small enough that the dynamic schedule merges the partitions in the
# decode kernel (at most 8 partitions per sequence, at most two items per
# resident warp): the lane-order partials and the merge at every head_dim and at
# group sizes below the 8 MMA columns (lanes holding padding columns store and
# read nothing).  One launch per call shows that no combine kernel ran.
IN_KERNEL_MERGE = [
    # (num_q_heads, num_kv_heads, head_dim, batch, max context)
    (32, 8, 128, 24, 512),    # G = 4
    (24, 8, 128, 24, 512),    # G = 3
    (16, 16, 128, 12, 512),   # G = 1
    (8, 4, 256, 32, 1024),    # G = 2, head_dim 256
    (16, 8, 64, 24, 2048),    # G = 2, head_dim 64
]


@pytest.mark.parametrize("hq,hkv,d,batch,max_len", IN_KERNEL_MERGE)
def test_in_kernel_merge_at_every_head_dim_and_group(hq, hkv, d, batch, max_len):
    w = wl.WORKLOADS["llama3_8b"].replace(num_q_heads=hq, num_kv_heads=hkv, head_dim=d, prefix_share=0.0)
    g = torch.Generator().manual_seed(77)
    lengths = [max_len] + torch.randint(max_len // 2, max_len + 1, (batch - 1,), generator=g).tolist()  # one at the bound
    b_cpu = wl.make_batch(w, lengths=lengths, seed=77)
    b = to_dev(b_cpu)
    need = pa.decode_splitk_workspace_size(batch, hq, d, max_len, 0, hkv)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(2):
        kc, vc = b.k_cache.clone(), b.v_cache.clone()
        out = pa.decode_step(b.q, b.k_new, b.v_new, kc, vc, b.block_tables, b.context_lens, w.scale, w.softcap,
                             w.window, split=True, max_context_len=max_len, partition_tokens=0, workspace=ws)
        assert pa.last_launch_count() == 1  # merged in the decode kernel
        assert pa.last_decode_schedule() == "dynamic_merged"
        torch.cuda.synchronize()
        assert int(ws[:COUNTER_BYTES].view(torch.int32).abs().sum()) == 0
        outs.append(out)
    assert torch.equal(bits(outs[0]), bits(outs[1]))
    ref, kc_ref, vc_ref = oracle_step(b_cpu)
    assert torch.equal(bits(kc), bits(kc_ref)) and torch.equal(bits(vc), bits(vc_ref))
    assert_close(outs[0], ref, torch.bfloat16, f"in-kernel merge G={hq // hkv} D={d}")
    assert pa.device_errors() == 0


@pytest.mark.parametrize("window", [0, 100, 333, 1000])
def test_dynamic_queue_merged_by_the_combine_kernel_with_windows(window):
    """A step too large for the in-kernel merge: the dynamic queue's partials go
    through the combine kernel.  A window makes a sequence's first item start
    inside a partition and leaves the partitions before it without tokens."""
    w = wl.WORKLOADS["llama3_8b"].replace(prefix_share=0.0)
    b_cpu = wl.make_batch(w, batch=16, max_len=3000, seed=91)
    b = to_dev(b_cpu)
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    out = pa.decode_step(b.q, b.k_new, b.v_new, kc, vc, b.block_tables, b.context_lens, w.scale, w.softcap, window,
                         split=True, max_context_len=b.max_context_len, partition_tokens=0)
    assert pa.last_launch_count() == 2  # decode and combine
    assert pa.last_decode_schedule() == "dynamic"
    torch.cuda.synchronize()
    ref, _, _ = oracle_step(b_cpu, window=window)
    assert_close(out, ref, torch.bfloat16, f"dynamic queue + combine, window={window}")
    assert pa.device_errors() == 0
