"""The seeded input generators: determinism, layout and canaries (CPU)."""

import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_473_b200 import workloads as wl


def _live_mask(batch):
    bs = batch.workload.block_size
    return torch.arange(bs).view(1, bs) < batch.live_per_block.view(-1, 1)


@pytest.mark.parametrize("name", list(wl.WORKLOADS))
def test_shapes_and_determinism(name):
    w = wl.WORKLOADS[name]
    small = {"batch": 5, "max_len": 300} if name != "tiny_fp32" else {}
    a = wl.make_batch(w, **small)
    b = wl.make_batch(w, **small)
    for f in ("q", "k_new", "v_new", "slot_mapping", "k_cache", "v_cache", "block_tables", "context_lens"):
        x, y = getattr(a, f), getattr(b, f)
        assert torch.equal(torch.nan_to_num(x.float(), 7.0), torch.nan_to_num(y.float(), 7.0)), f
    B = a.q.shape[0]
    assert a.q.shape == (B, w.num_q_heads, w.head_dim)
    assert a.k_cache.shape[1:] == (w.num_kv_heads, w.block_size, w.head_dim)
    assert a.q.dtype == w.torch_dtype and a.k_cache.dtype == w.torch_dtype
    c = wl.make_batch(w, seed=w.seed + 1, **small)
    assert not torch.equal(a.q, c.q)


def test_tiny_pool_has_exactly_64_blocks():
    b = wl.make_batch(wl.WORKLOADS["tiny_fp32"])
    assert b.num_blocks == 64
    L = b.context_lens
    assert int(L.min()) >= 1 and int(L.max()) <= 100


@pytest.mark.parametrize("prefilled", [False, True])
def test_canary_marks_exactly_the_dead_slots(prefilled):
    w = wl.WORKLOADS["tinyllama_1b"]
    b = wl.make_batch(w, batch=6, max_len=200, prefilled=prefilled)
    live = _live_mask(b)  # [nb, bs]
    kc = b.k_cache.float().permute(0, 2, 1, 3)  # [nb, bs, Hkv, D]
    assert torch.isfinite(kc[live]).all()
    assert torch.isnan(kc[~live]).all()
    # Live rows per sequence equal L (prefilled) or L-1 (the step still appends one).
    bs = w.block_size
    for i in range(6):
        L = int(b.context_lens[i])
        n = L if prefilled else L - 1
        for t in range(L):
            blk = int(b.block_tables[i, t // bs])
            assert bool(live[blk, t % bs]) == (t < n)


def test_slot_mapping_points_at_position_L_minus_1():
    w = wl.WORKLOADS["gemma2_2b"]
    b = wl.make_batch(w, batch=9, max_len=700)
    bs = w.block_size
    for i in range(9):
        L = int(b.context_lens[i])
        s = int(b.slot_mapping[i])
        assert s // bs == int(b.block_tables[i, (L - 1) // bs]) and s % bs == (L - 1) % bs
    # Slots are distinct and tables are padded with -1 past the last block.
    assert len(set(b.slot_mapping.tolist())) == 9
    for i in range(9):
        n = math.ceil(int(b.context_lens[i]) / bs)
        assert (b.block_tables[i, n:] == -1).all() and (b.block_tables[i, :n] >= 0).all()


def test_prefix_sharing_recipe():
    w = wl.WORKLOADS["llama3_8b"]
    b = wl.make_batch(w, batch=40, max_len=3000)
    shared = set(b.shared_blocks.tolist())
    assert len(shared) == 64
    sharers = [i for i in range(40) if int(b.block_tables[i, 0]) in shared]
    assert len(sharers) == 12  # 30% of 40
    bs = w.block_size
    for i in sharers:
        L = int(b.context_lens[i])
        k = min(64, (L - 1) // bs)
        assert b.block_tables[i, :k].tolist() == b.shared_blocks[:k].tolist()
        assert int(b.block_tables[i, (L - 1) // bs]) not in shared
    # Every other block id appears at most once across tables.
    ids = [int(x) for x in b.block_tables.flatten() if int(x) >= 0 and int(x) not in shared]
    assert len(ids) == len(set(ids))
    assert wl.kv_bytes(b, unique=True) < wl.kv_bytes(b)


def test_length_recipes():
    g = torch.Generator().manual_seed(0)
    L = wl.sample_lengths(wl.WORKLOADS["llama3_8b"], g, 20000)
    assert int(L.min()) >= 256 and int(L.max()) <= 8192
    # log-uniform: the median sits near the geometric mean of the bounds.
    assert abs(float(L.double().median()) / math.sqrt(256 * 8192) - 1) < 0.05
    L = wl.sample_lengths(wl.WORKLOADS["gemma2_2b"], g, 20000)
    assert int(L.min()) >= 129 and int(L.max()) <= 1024
    assert abs(float(L.double().mean()) - 576.5) < 5


def test_append_then_decode_matches_prefilled_oracle():
    """The oracle step (append, then decode) on a generated batch equals the
    decode of a batch whose pool already held the token."""
    w = wl.WORKLOADS["tiny_fp32"]
    b = wl.make_batch(w)
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    oracle.write_kv(b.k_new, b.v_new, b.slot_mapping, kc, vc)
    out = oracle.decode(b.q, kc, vc, b.block_tables, b.context_lens, w.scale)
    assert np.all(np.isfinite(out))
    # Reading any dead slot would have produced NaN; the appended rows are live now.
    L = b.context_lens
    bs = w.block_size
    for i in range(L.numel()):
        t = int(L[i]) - 1
        blk = int(b.block_tables[i, t // bs])
        assert torch.equal(kc[blk, :, t % bs], b.k_new[i])
