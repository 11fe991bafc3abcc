"""Pins for the CPU oracle: checks against things other than itself.

Each test ties the oracle to a library routine on contiguous data, a closed
form, an invariant, or the examples drawn on the pages (fixtures under
tests/golden/).  No GPU is used.
"""

import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from tests.paging_helpers import scatter_to_pool, sdpa_decode, sdpa_multi

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_seqs(gen, lens, hkv, d, dtype=torch.float32):
    ks = [torch.randn((L, hkv, d), generator=gen).to(dtype) for L in lens]
    vs = [torch.randn((L, hkv, d), generator=gen).to(dtype) for L in lens]
    return ks, vs


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("hq,hkv,d,bs", [(4, 4, 4, 4), (8, 2, 64, 16), (6, 3, 64, 8), (8, 1, 16, 4)])
def test_agrees_with_torch_sdpa_on_contiguous_kv(dtype, hq, hkv, d, bs):
    gen = torch.Generator().manual_seed(11 + hq + d)
    lens = [1, 7, 40, 23]
    ks, vs = _rand_seqs(gen, lens, hkv, d, dtype)
    q = torch.randn((len(lens), hq, d), generator=gen).to(dtype)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, bs, gen, dtype=dtype)
    scale = 1.0 / math.sqrt(d)
    got = oracle.decode(q, kc, vc, tables, cl, scale)
    ref = sdpa_decode(q, ks, vs, float(np.float32(scale))).numpy()
    assert np.max(np.abs(got - ref)) <= 1e-12


@pytest.mark.parametrize("window", [1, 5, 22, 23, 24, 100])
def test_window_agrees_with_sdpa_on_the_last_w_positions(window):
    gen = torch.Generator().manual_seed(5)
    lens = [23, 3, 40]
    ks, vs = _rand_seqs(gen, lens, 2, 16)
    q = torch.randn((3, 4, 16), generator=gen)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 4, gen)
    got = oracle.decode(q, kc, vc, tables, cl, 0.25, window=window)
    ref = sdpa_decode(q, ks, vs, 0.25, window=window).numpy()
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_block_permutation_invariance_is_bit_exact():
    gen = torch.Generator().manual_seed(7)
    lens = [37, 64, 5, 90]
    ks, vs = _rand_seqs(gen, lens, 2, 32, torch.bfloat16)
    q = torch.randn((4, 8, 32), generator=gen).to(torch.bfloat16)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 16, gen, dtype=torch.bfloat16)
    base = oracle.decode(q, kc, vc, tables, cl, 0.17, softcap=3.0, window=50)
    nb = kc.shape[0]
    for seed in range(3):
        perm = torch.randperm(nb, generator=torch.Generator().manual_seed(100 + seed))  # new position of block i
        kc2 = torch.empty_like(kc)
        vc2 = torch.empty_like(vc)
        kc2[perm] = kc
        vc2[perm] = vc
        t2 = tables.clone()
        m = t2 >= 0
        t2[m] = perm[t2[m].long()].to(torch.int32)
        got = oracle.decode(q, kc2, vc2, t2, cl, 0.17, softcap=3.0, window=50)
        assert np.array_equal(got, base)


def test_context_of_length_one_returns_v_exactly():
    gen = torch.Generator().manual_seed(3)
    ks, vs = _rand_seqs(gen, [1, 1], 2, 64, torch.bfloat16)
    q = torch.randn((2, 8, 64), generator=gen).to(torch.bfloat16) * 50
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 16, gen, dtype=torch.bfloat16)
    got = oracle.decode(q, kc, vc, tables, cl, 0.125, softcap=7.0)
    for b in range(2):
        for h in range(8):
            assert np.array_equal(got[b, h], vs[b][0, h // 4].double().numpy())


@pytest.mark.parametrize("window", [0, 6])
def test_identical_keys_give_the_mean_of_v(window):
    gen = torch.Generator().manual_seed(9)
    L = 20
    key = torch.randn((1, 2, 16), generator=gen)
    ks = [key.expand(L, 2, 16).clone()]
    vs = [torch.randn((L, 2, 16), generator=gen)]
    q = torch.randn((1, 4, 16), generator=gen)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 8, gen)
    got = oracle.decode(q, kc, vc, tables, cl, 0.25, softcap=2.0, window=window)
    s0 = L - window if window else 0
    for h in range(4):
        mean = vs[0][s0:, h // 2].double().mean(0).numpy()
        assert np.max(np.abs(got[0, h] - mean)) <= 1e-12


def test_infinite_or_zero_softcap_equals_plain_attention_bit_exact():
    gen = torch.Generator().manual_seed(4)
    ks, vs = _rand_seqs(gen, [30, 9], 2, 16)
    q = torch.randn((2, 4, 16), generator=gen) * 4
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 4, gen)
    plain = oracle.decode(q, kc, vc, tables, cl, 0.25)
    assert np.array_equal(oracle.decode(q, kc, vc, tables, cl, 0.25, softcap=float("inf")), plain)
    assert np.array_equal(oracle.decode(q, kc, vc, tables, cl, 0.25, softcap=0.0), plain)
    near = oracle.decode(q, kc, vc, tables, cl, 0.25, softcap=1e6)
    assert np.max(np.abs(near - plain)) <= 1e-6
    assert np.max(np.abs(near - plain)) > 0


def _two_token_case(softcap):
    # D = 4, scale = 1/2, q = [2,0,0,0], k1 = [1,0,0,0], k2 = [-1,0,0,0]
    # -> raw scores +1 and -1 (all values exact in fp32).
    q = torch.tensor([[[2.0, 0, 0, 0]]])
    ks = [torch.tensor([[[1.0, 0, 0, 0]], [[-1.0, 0, 0, 0]]])]
    vs = [torch.tensor([[[1.0, 2.0, -3.0, 0.5]], [[-2.0, 4.0, 1.0, 8.0]]])]
    gen = torch.Generator().manual_seed(0)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 4, gen)
    got = oracle.decode(q, kc, vc, tables, cl, 0.5, softcap=softcap)[0, 0]
    return got, vs[0][0, 0].double().numpy(), vs[0][1, 0].double().numpy()


def test_two_token_closed_form():
    got, v1, v2 = _two_token_case(0.0)
    w1 = 1.0 / (1.0 + math.exp(-2.0))  # e^1 / (e^1 + e^-1)
    assert np.max(np.abs(got - (w1 * v1 + (1 - w1) * v2))) <= 1e-15


def test_two_token_closed_form_with_softcap():
    got, v1, v2 = _two_token_case(2.0)
    x = 2.0 * math.tanh(0.5)  # capped scores are +x and -x
    w1 = 1.0 / (1.0 + math.exp(-2 * x))
    assert np.max(np.abs(got - (w1 * v1 + (1 - w1) * v2))) <= 1e-15


def test_softcap_saturates_at_plus_minus_c():
    # Raw scores +-1000 with c = 5 saturate to +-5 (tanh(200) == 1 in fp64).
    q = torch.tensor([[[2000.0, 0, 0, 0]]])
    ks = [torch.tensor([[[1.0, 0, 0, 0]], [[-1.0, 0, 0, 0]], [[-1.0, 0, 0, 0]]])]
    vs = [torch.tensor([[[1.0, 0, 0, 0]], [[0.0, 1.0, 0, 0]], [[0.0, 0, 1.0, 0]]])]
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 2, torch.Generator().manual_seed(1))
    got = oracle.decode(q, kc, vc, tables, cl, 0.5, softcap=5.0)[0, 0]
    e = math.exp(-10.0)
    want = np.array([1.0, e, e, 0.0]) / (1.0 + 2 * e)
    assert np.max(np.abs(got - want)) <= 1e-15


def test_window_one_returns_last_v_and_wide_window_is_no_window():
    gen = torch.Generator().manual_seed(12)
    ks, vs = _rand_seqs(gen, [17, 4], 1, 8)
    q = torch.randn((2, 2, 8), generator=gen)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 4, gen)
    got = oracle.decode(q, kc, vc, tables, cl, 0.3, window=1)
    for b, L in enumerate([17, 4]):
        for h in range(2):
            assert np.array_equal(got[b, h], vs[b][L - 1, 0].double().numpy())
    plain = oracle.decode(q, kc, vc, tables, cl, 0.3)
    for W in (17, 18, 1000):
        assert np.array_equal(oracle.decode(q, kc, vc, tables, cl, 0.3, window=W), plain)


def test_zero_length_context_gives_zero_row():
    gen = torch.Generator().manual_seed(2)
    ks, vs = _rand_seqs(gen, [0, 5], 1, 8)
    q = torch.randn((2, 1, 8), generator=gen)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 4, gen)
    got = oracle.decode(q, kc, vc, tables, cl, 0.3)
    assert np.array_equal(got[0, 0], np.zeros(8))
    assert np.all(np.isfinite(got[1]))


def test_gqa_grouping_follows_the_xray_example():
    """32 query heads over 8 kv heads: head h reads kv head h // 4 only."""
    fx = json.load(open(os.path.join(GOLDEN, "xray_gqa_shapes.json")))
    hq, hkv, n, d = fx["num_q_heads"], fx["num_kv_heads"], fx["seq_len"], fx["head_dim"]
    assert hq // hkv == fx["group"]
    gen = torch.Generator().manual_seed(21)
    ks, vs = _rand_seqs(gen, [n], hkv, d)
    q = torch.randn((1, hq, d), generator=gen)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 4, gen)
    scale = 1.0 / math.sqrt(128)
    base = oracle.decode(q, kc, vc, tables, cl, scale)
    # Dense scores Q K^T / sqrt(128) for the last query position via SDPA.
    ref = sdpa_decode(q, ks, vs, float(np.float32(scale))).numpy()
    assert np.max(np.abs(base - ref)) <= 1e-12
    # Perturb kv head 3: only query heads 12..15 move.
    ks2 = [ks[0].clone()]
    vs2 = [vs[0].clone()]
    ks2[0][:, 3] += 1.0
    vs2[0][:, 3] -= 2.0
    kc2, vc2, t2, cl2 = scatter_to_pool(ks2, vs2, 4, torch.Generator().manual_seed(22))
    moved = oracle.decode(q, kc2, vc2, t2, cl2, scale)
    changed = [h for h in range(hq) if not np.allclose(moved[0, h], base[0, h], atol=1e-12, rtol=0)]
    assert changed == [12, 13, 14, 15]


def test_block_table_example_from_the_pages(oracle_lib):
    fx = json.load(open(os.path.join(GOLDEN, "nano_vllm_block_table.json")))
    nb, bs = fx["num_blocks"], fx["block_size"]
    tab = fx["tables"]
    hkv, d = 2, 8
    gen = torch.Generator().manual_seed(31)
    lens = [len(tab["A"]) * bs, len(tab["B"]) * bs]
    ks, vs = _rand_seqs(gen, lens, hkv, d)
    kc = torch.full((nb, hkv, bs, d), float("nan"))
    vc = torch.full((nb, hkv, bs, d), float("nan"))
    # Append every token of both sequences through the oracle, one step at a time.
    for b, name in enumerate(["A", "B"]):
        for t in range(lens[b]):
            slot = torch.tensor([tab[name][t // bs] * bs + t % bs])
            oracle.write_kv(ks[b][t : t + 1], vs[b][t : t + 1], slot, kc, vc)
    for blk in fx["free_blocks"]:
        assert torch.isnan(kc[blk]).all() and torch.isnan(vc[blk]).all()
    tables = torch.full((2, 3), -1, dtype=torch.int32)
    tables[0, :2] = torch.tensor(tab["A"])
    tables[1, :3] = torch.tensor(tab["B"])
    q = torch.randn((2, 4, d), generator=gen)
    got = oracle.decode(q, kc, vc, tables, torch.tensor(lens, dtype=torch.int32), 0.35)
    ref = sdpa_decode(q, ks, vs, float(np.float32(0.35))).numpy()
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_incremental_decode_equals_causal_attention():
    """A decode step appends one token and attends over the cache; step i's
    output equals row i of causal attention over the whole sequence (nano-vllm
    README, "Key Concepts Explained: KV Cache")."""
    gen = torch.Generator().manual_seed(41)
    n, hq, hkv, d, bs = 13, 4, 2, 16, 4
    kseq = torch.randn((n, hkv, d), generator=gen)
    vseq = torch.randn((n, hkv, d), generator=gen)
    qseq = torch.randn((n, hq, d), generator=gen)
    nb = 6
    blocks = [4, 0, 5, 2]
    kc = torch.full((nb, hkv, bs, d), float("nan"))
    vc = torch.full((nb, hkv, bs, d), float("nan"))
    tables = torch.tensor([blocks], dtype=torch.int32)
    causal = F.scaled_dot_product_attention(
        qseq.double().permute(1, 0, 2).unsqueeze(0),
        kseq.double().permute(1, 0, 2).unsqueeze(0),
        vseq.double().permute(1, 0, 2).unsqueeze(0),
        is_causal=True,
        scale=0.25,
        enable_gqa=True,
    )[0].permute(1, 0, 2)  # [n, hq, d]
    for i in range(n):
        slot = torch.tensor([blocks[i // bs] * bs + i % bs])
        oracle.write_kv(kseq[i : i + 1], vseq[i : i + 1], slot, kc, vc)
        got = oracle.decode(qseq[i : i + 1], kc, vc, tables, torch.tensor([i + 1], dtype=torch.int32), 0.25)
        assert np.max(np.abs(got[0] - causal[i].numpy())) <= 1e-12


def test_write_kv_touches_only_target_slots_and_skips_padding():
    gen = torch.Generator().manual_seed(51)
    nb, hkv, bs, d = 5, 2, 4, 8
    kc = torch.full((nb, hkv, bs, d), float("nan"), dtype=torch.bfloat16)
    vc = torch.full((nb, hkv, bs, d), float("nan"), dtype=torch.bfloat16)
    k = torch.randn((3, hkv, d), generator=gen).to(torch.bfloat16)
    v = torch.randn((3, hkv, d), generator=gen).to(torch.bfloat16)
    slots = torch.tensor([7, -1, 18])
    oracle.write_kv(k, v, slots, kc, vc)
    assert torch.equal(kc[1, :, 3], k[0]) and torch.equal(vc[1, :, 3], v[0])
    assert torch.equal(kc[4, :, 2], k[2]) and torch.equal(vc[4, :, 2], v[2])
    written = torch.zeros((nb, bs), dtype=torch.bool)
    written[1, 3] = written[4, 2] = True
    assert torch.isnan(kc.permute(0, 2, 1, 3)[~written].float()).all()
    assert torch.isnan(vc.permute(0, 2, 1, 3)[~written].float()).all()
    with pytest.raises(ValueError):
        oracle.write_kv(k, v, torch.tensor([0, 1, nb * bs]), kc, vc)


def test_bad_block_id_is_reported():
    gen = torch.Generator().manual_seed(61)
    ks, vs = _rand_seqs(gen, [6], 1, 8)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 4, gen)
    tables[0, 1] = kc.shape[0]
    with pytest.raises(ValueError):
        oracle.decode(torch.randn((1, 1, 8)), kc, vc, tables, cl, 0.3)


def test_sampled_rows_match_full_output():
    gen = torch.Generator().manual_seed(71)
    ks, vs = _rand_seqs(gen, [9, 30, 2], 2, 16)
    q = torch.randn((3, 8, 16), generator=gen)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 4, gen)
    full = oracle.decode(q, kc, vc, tables, cl, 0.25, softcap=4.0, window=10)
    rows = [(2, 7), (0, 0), (1, 5)]
    got = oracle.decode(q, kc, vc, tables, cl, 0.25, softcap=4.0, window=10, rows=rows)
    for i, (b, h) in enumerate(rows):
        assert np.array_equal(got[i], full[b, h])


# ---- multi-query rows (several new tokens per sequence, causal) ---------------------


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T", [1, 2, 5, 8])
@pytest.mark.parametrize("window", [0, 3, 17])
@pytest.mark.parametrize("hq,hkv,d,bs", [(8, 2, 64, 16), (6, 3, 16, 4)])
def test_multi_agrees_with_torch_under_a_causal_mask(dtype, T, window, hq, hkv, d, bs):
    gen = torch.Generator().manual_seed(100 + T + window + d)
    lens = [T, 9 + T, 40, 23]
    ks, vs = _rand_seqs(gen, lens, hkv, d, dtype)
    q = torch.randn((len(lens), T, hq, d), generator=gen).to(dtype)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, bs, gen, dtype=dtype)
    scale = 1.0 / math.sqrt(d)
    got = oracle.decode_multi(q, kc, vc, tables, cl, scale, window=window)
    ref = sdpa_multi(q, ks, vs, float(np.float32(scale)), window=window).numpy()
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_multi_with_one_query_token_equals_decode_bit_exact():
    gen = torch.Generator().manual_seed(61)
    lens = [1, 17, 64, 33]
    ks, vs = _rand_seqs(gen, lens, 2, 32, torch.bfloat16)
    q = torch.randn((4, 8, 32), generator=gen).to(torch.bfloat16)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 8, gen, dtype=torch.bfloat16)
    for cap, win in [(0.0, 0), (50.0, 0), (0.0, 5)]:
        a = oracle.decode(q, kc, vc, tables, cl, 0.2, cap, win)
        b = oracle.decode_multi(q.unsqueeze(1), kc, vc, tables, cl, 0.2, cap, win)[:, 0]
        assert np.array_equal(a, b)


def test_multi_row_j_is_decode_over_its_own_prefix_with_softcap():
    """Query token j of T is a decode step whose context ends at its own
    position (the incremental reading of the KV cache) -- checked with the
    softcap on, against the pinned decode."""
    gen = torch.Generator().manual_seed(62)
    T, lens = 5, [5, 12, 30]
    ks, vs = _rand_seqs(gen, lens, 4, 16)
    q = torch.randn((3, T, 8, 16), generator=gen)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 4, gen)
    got = oracle.decode_multi(q, kc, vc, tables, cl, 0.5, softcap=3.0, window=7)
    for j in range(T):
        cl_j = (cl - (T - 1 - j)).to(torch.int32)
        ref = oracle.decode(q[:, j], kc, vc, tables, cl_j, 0.5, softcap=3.0, window=7)
        assert np.max(np.abs(got[:, j] - ref)) <= 1e-12


def test_multi_rows_do_not_see_later_positions():
    gen = torch.Generator().manual_seed(63)
    T, lens = 4, [11, 20]
    ks, vs = _rand_seqs(gen, lens, 2, 16)
    q = torch.randn((2, T, 4, 16), generator=gen)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 4, gen)
    base = oracle.decode_multi(q, kc, vc, tables, cl, 0.25)
    for j in range(T):
        ks2 = [k.clone() for k in ks]
        vs2 = [v.clone() for v in vs]
        for b, L in enumerate(lens):  # overwrite every position after query j's
            ks2[b][L - T + j + 1:] = 7.0
            vs2[b][L - T + j + 1:] = -3.0
        kc2, vc2 = kc.clone(), vc.clone()
        for b, L in enumerate(lens):
            for t in range(L - T + j + 1, L):
                blk = int(tables[b, t // 4])
                kc2[blk, :, t % 4] = ks2[b][t]
                vc2[blk, :, t % 4] = vs2[b][t]
        got = oracle.decode_multi(q, kc2, vc2, tables, cl, 0.25)
        assert np.array_equal(got[:, : j + 1], base[:, : j + 1])
        if j + 1 < T:
            assert not np.array_equal(got[:, j + 1:], base[:, j + 1:])


def test_multi_queries_before_the_start_give_zero_rows_and_rows_match():
    gen = torch.Generator().manual_seed(64)
    T, lens = 6, [3, 10]  # sequence 0 holds fewer positions than query tokens
    ks, vs = _rand_seqs(gen, lens, 2, 16)
    q = torch.randn((2, T, 4, 16), generator=gen)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 4, gen)
    full = oracle.decode_multi(q, kc, vc, tables, cl, 0.25)
    assert np.all(full[0, : T - 3] == 0.0) and np.all(np.isfinite(full))
    rows = [(0, 5, 1), (1, 0, 3), (1, 5, 0), (0, 0, 2)]
    part = oracle.decode_multi(q, kc, vc, tables, cl, 0.25, rows=rows)
    for r, (b, j, h) in enumerate(rows):
        assert np.array_equal(part[r], full[b, j, h])


# ---- prefill (append a prompt, attend it causally) --------------------------------


@pytest.mark.parametrize("hq,hkv,bs", [(8, 2, 4), (4, 4, 16), (6, 1, 8)])
def test_prefill_from_scratch_equals_causal_attention(hq, hkv, bs):
    """Prompts written into an empty paged cache and attended in one call are
    causal self-attention over each prompt (torch fp64, is_causal)."""
    gen = torch.Generator().manual_seed(71 + hq + bs)
    d, lens = 16, [1, 7, 20, 13]
    B = len(lens)
    ks, vs = _rand_seqs(gen, lens, hkv, d)
    qs = [torch.randn((L, hq, d), generator=gen) for L in lens]
    kc, vc, tables, cl = scatter_to_pool(ks, vs, bs, gen)
    kc.fill_(float("nan"))  # the cache starts empty: prefill must write every row itself
    vc.fill_(float("nan"))
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    slots = []
    for b, L in enumerate(lens):
        slots += [int(tables[b, t // bs]) * bs + t % bs for t in range(L)]
    got = oracle.prefill(torch.cat(qs), torch.cat(ks), torch.cat(vs), torch.tensor(slots, dtype=torch.int64), cu, kc,
                         vc, tables, cl, 0.25)
    for b, L in enumerate(lens):
        ref = F.scaled_dot_product_attention(qs[b].double().permute(1, 0, 2).unsqueeze(0),
                                             ks[b].double().permute(1, 0, 2).unsqueeze(0),
                                             vs[b].double().permute(1, 0, 2).unsqueeze(0), is_causal=True,
                                             scale=0.25, enable_gqa=True)[0].permute(1, 0, 2)
        assert np.max(np.abs(got[int(cu[b]):int(cu[b + 1])] - ref.numpy())) <= 1e-12


def test_chunked_prefill_equals_one_shot_prefill():
    """Two chunks (the second attending the first from the cache) give the
    rows of a single prefill of the whole prompt."""
    gen = torch.Generator().manual_seed(73)
    hq, hkv, d, bs, L, c1 = 4, 2, 16, 4, 19, 8
    ks, vs = _rand_seqs(gen, [L], hkv, d)
    q = torch.randn((L, hq, d), generator=gen)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, bs, gen)
    slots = torch.tensor([int(tables[0, t // bs]) * bs + t % bs for t in range(L)], dtype=torch.int64)
    one = oracle.prefill(q, ks[0], vs[0], slots, torch.tensor([0, L], dtype=torch.int32), kc.clone(), vc.clone(),
                         tables, cl, 0.3)
    kc2, vc2 = kc.clone(), vc.clone()
    first = oracle.prefill(q[:c1], ks[0][:c1], vs[0][:c1], slots[:c1], torch.tensor([0, c1], dtype=torch.int32),
                           kc2, vc2, tables, torch.tensor([c1], dtype=torch.int32), 0.3)
    second = oracle.prefill(q[c1:], ks[0][c1:], vs[0][c1:], slots[c1:], torch.tensor([0, L - c1], dtype=torch.int32),
                            kc2, vc2, tables, cl, 0.3)
    assert np.array_equal(np.concatenate([first, second]), one)


def _partial_log2(q, k, v, scale, softcap):
    """One partition's (m, l, o) in the log2 domain, fp64: s = scaled (and
    capped) scores times log2(e); m = max s, l = sum 2^(s-m), o = sum 2^(s-m) v."""
    s = (k @ q) * scale
    if softcap > 0 and math.isfinite(softcap):
        s = softcap * np.tanh(s / softcap)
    s = s * math.log2(math.e)
    if s.size == 0:
        return -math.inf, 0.0, np.zeros(v.shape[1])
    m = s.max()
    w = np.exp2(s - m)
    return m, w.sum(), w @ v


def _merge(parts):
    """Log-sum-exp merge: M = max m_p, out = sum 2^(m_p - M) o_p / sum 2^(m_p - M) l_p
    (empty partitions, m = -inf, weigh nothing)."""
    M = max(m for m, _, _ in parts)
    num = sum((0.0 if m == -math.inf else 2.0 ** (m - M)) * o for m, _, o in parts)
    den = sum((0.0 if m == -math.inf else 2.0 ** (m - M)) * l for m, l, _ in parts)
    return num / den


@pytest.mark.parametrize("P", [16, 64, 256])
@pytest.mark.parametrize("softcap,window", [(0.0, 0), (30.0, 0), (0.0, 50)])
def test_split_k_merge_rule_reproduces_the_unsplit_definition(P, softcap, window):
    """The split-K partials and their log-sum-exp merge (what the combine kernel
    and the in-kernel merges compute) equal the oracle's unsplit attention,
    for partitions that split the window start and the end, empty
    partitions included.  The cascade's prefix / own-range split is the same
    identity with two partitions."""
    gen = torch.Generator().manual_seed(41)
    lens = [1, 37, 300]
    hq, hkv, d = 4, 2, 16
    ks, vs = _rand_seqs(gen, lens, hkv, d)
    q = torch.randn((len(lens), hq, d), generator=gen)
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 16, gen)
    scale = float(np.float32(1 / math.sqrt(d)))  # the oracle takes the fp32 scale, widened
    ref = oracle.decode(q, kc, vc, tables, cl, scale, softcap=softcap, window=window)
    for b, L in enumerate(lens):
        s0 = L - window if window and L > window else 0
        for h in range(hq):
            g = h // (hq // hkv)
            k = ks[b][:, g].double().numpy()
            v = vs[b][:, g].double().numpy()
            qv = q[b, h].double().numpy()
            bounds = [s0] + list(range((s0 // P + 1) * P, L, P)) + [L]
            parts = [_partial_log2(qv, k[lo:hi], v[lo:hi], scale, softcap) for lo, hi in zip(bounds, bounds[1:])]
            parts.append(_partial_log2(qv, k[:0], v[:0], scale, softcap))  # an empty partition
            assert np.max(np.abs(_merge(parts) - ref[b, h])) <= 1e-12
            if L > 1:  # cascade: prefix [s0, c) and own range [c, L)
                c = s0 + (L - s0) // 2
                two = [_partial_log2(qv, k[s0:c], v[s0:c], scale, softcap),
                       _partial_log2(qv, k[c:L], v[c:L], scale, softcap)]
                assert np.max(np.abs(_merge(two) - ref[b, h])) <= 1e-12


@pytest.mark.parametrize("tile", [64, 128])
def test_lazy_rescaled_online_softmax_is_exact(tile):
    """The prefill softmax's lazy rescaling: the reference maximum moves only
    when a tile's maximum exceeds it by more than 8 (log2 units), so every
    weight stays <= 2^8, and since the sum and the output share the
    reference the result is the exact softmax (fp64 simulation of the tile
    loop against the oracle's two-pass definition)."""
    gen = torch.Generator().manual_seed(77)
    L, hq, hkv, d = 700, 4, 1, 32
    ks, vs = _rand_seqs(gen, [L], hkv, d)
    # growing scores along the sequence, so the reference has to move several times
    ks[0] = ks[0] * torch.linspace(0.2, 3.0, L).view(L, 1, 1)
    q = torch.randn((1, hq, d), generator=gen) * 2
    kc, vc, tables, cl = scatter_to_pool(ks, vs, 16, gen)
    scale = float(np.float32(1 / math.sqrt(d)))  # the oracle takes the fp32 scale, widened
    ref = oracle.decode(q, kc, vc, tables, cl, scale)
    k = ks[0][:, 0].double().numpy()
    v = vs[0][:, 0].double().numpy()
    for h in range(hq):
        s = (k @ q[0, h].double().numpy()) * scale * math.log2(math.e)
        m, l, o, moves = -math.inf, 0.0, np.zeros(d), 0
        for t0 in range(0, L, tile):
            st = s[t0 : t0 + tile]
            mt = st.max()
            mn = mt if (m == -math.inf or mt > m + 8) else m
            moves += mn != m
            alpha = 2.0 ** (m - mn) if m != -math.inf else 0.0
            w = np.exp2(st - mn)
            assert w.max() <= 2.0 ** 8
            l = l * alpha + w.sum()
            o = o * alpha + w @ v[t0 : t0 + tile]
            m = mn
        assert moves >= 2
        assert np.max(np.abs(o / l - ref[0, h])) <= 1e-12
