"""Test-side helpers: build a paged pool from contiguous per-sequence K/V.

The tests know the contiguous truth and scatter it into randomly chosen blocks
themselves, so that a gather bug in the oracle or in the CUDA path shows up as
a disagreement with dense attention computed by torch on the contiguous data.
"""

from __future__ import annotations

import math

import torch
import torch.nn.functional as F


def scatter_to_pool(seqs_k, seqs_v, block_size, gen, extra_blocks=3, dtype=torch.float32, fill=float("nan")):
    """seqs_k[b]: [L_b, Hkv, D].  Returns (k_cache, v_cache, block_tables, context_lens)."""
    B = len(seqs_k)
    Hkv, D = seqs_k[0].shape[1], seqs_k[0].shape[2]
    need = [max(1, math.ceil(k.shape[0] / block_size)) if k.shape[0] else 0 for k in seqs_k]
    nb = sum(need) + extra_blocks
    perm = torch.randperm(nb, generator=gen)
    maxb = max(1, max(need))
    tables = torch.full((B, maxb), -1, dtype=torch.int32)
    kc = torch.full((nb, Hkv, block_size, D), fill, dtype=dtype)
    vc = torch.full((nb, Hkv, block_size, D), fill, dtype=dtype)
    pos = 0
    for b in range(B):
        L = seqs_k[b].shape[0]
        for i in range(need[b]):
            blk = int(perm[pos])
            pos += 1
            tables[b, i] = blk
            lo, hi = i * block_size, min(L, (i + 1) * block_size)
            if hi > lo:
                kc[blk, :, : hi - lo, :] = seqs_k[b][lo:hi].permute(1, 0, 2).to(dtype)
                vc[blk, :, : hi - lo, :] = seqs_v[b][lo:hi].permute(1, 0, 2).to(dtype)
    lens = torch.tensor([k.shape[0] for k in seqs_k], dtype=torch.int32)
    return kc, vc, tables, lens


def sdpa_decode(q, seqs_k, seqs_v, scale, window=0):
    """torch fp64 scaled_dot_product_attention of each sequence's last query
    against its contiguous K/V (GQA through ``enable_gqa``)."""
    B, Hq, D = q.shape
    out = torch.zeros((B, Hq, D), dtype=torch.float64)
    for b in range(B):
        L = seqs_k[b].shape[0]
        s0 = max(0, L - window) if window > 0 else 0
        if L - s0 <= 0:
            continue
        k = seqs_k[b][s0:L].to(torch.float64).permute(1, 0, 2).unsqueeze(0)  # [1, Hkv, L, D]
        v = seqs_v[b][s0:L].to(torch.float64).permute(1, 0, 2).unsqueeze(0)
        qq = q[b].to(torch.float64).unsqueeze(0).unsqueeze(2)  # [1, Hq, 1, D]
        o = F.scaled_dot_product_attention(qq, k, v, scale=scale, enable_gqa=True)
        out[b] = o[0, :, 0, :]
    return out


def sdpa_multi(q, seqs_k, seqs_v, scale, window=0):
    """torch fp64 attention of each sequence's last T queries (``q``: [B, T, Hq, D])
    against its contiguous K/V, with an explicit boolean mask: query j at
    position p = L - T + j sees positions t with t <= p and p - t < window
    (window > 0)."""
    B, T, Hq, D = q.shape
    out = torch.zeros((B, T, Hq, D), dtype=torch.float64)
    for b in range(B):
        L = seqs_k[b].shape[0]
        pos = torch.arange(L - T, L).unsqueeze(1)  # [T, 1]
        t = torch.arange(L).unsqueeze(0)  # [1, L]
        mask = t <= pos
        if window > 0:
            mask &= (pos - t) < window
        k = seqs_k[b].to(torch.float64).permute(1, 0, 2).unsqueeze(0)  # [1, Hkv, L, D]
        v = seqs_v[b].to(torch.float64).permute(1, 0, 2).unsqueeze(0)
        qq = q[b].to(torch.float64).permute(1, 0, 2).unsqueeze(0)  # [1, Hq, T, D]
        o = F.scaled_dot_product_attention(qq, k, v, attn_mask=mask, scale=scale, enable_gqa=True)
        out[b] = o[0].permute(1, 0, 2)
    return out
