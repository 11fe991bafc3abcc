"""Seeded synthetic decode batches for the paged KV cache.

This module only draws inputs: context lengths, a shuffled pool of physical
blocks with per-sequence block tables, the query / new key / new value rows
and the cache contents.  It holds none of the attention arithmetic, so the
CUDA path and the CPU oracle can both take their inputs from it.

Cache layout ("HND"): ``k_cache`` and ``v_cache`` are
``[num_blocks, num_kv_heads, block_size, head_dim]`` row-major, so that one
(physical block, kv head) pair is one contiguous run of
``block_size * head_dim`` elements.  A sequence's logical block ``i`` lives in
physical block ``block_tables[b, i]``; entries past the sequence's last block
are ``-1``.  This mirrors the block table drawn in the nano-vllm (ovshake)
README, "Key Concepts Explained: PagedAttention" (blocks of one shared pool
handed to sequences on demand, in any order).

Every slot that holds no live token is filled with a NaN canary, so a kernel
that reads a slot it should not ends with NaN in its output.

Convention for one decode step (vLLM style, the pages leave it open):
``context_lens[b]`` counts every cached token *including* the one appended this
step, the new token sits at position ``L - 1`` and its slot is
``block_tables[b][(L-1) // block_size] * block_size + (L-1) % block_size``.
"""

from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass
from typing import Optional

import torch

__all__ = ["Workload", "Batch", "WORKLOADS", "make_batch", "sample_lengths"]


@dataclass(frozen=True)
class Workload:
    """Shape and length recipe of one synthetic decode batch."""

    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str  # "f32" or "bf16"
    lengths: tuple  # ("uniform", lo, hi) | ("sum_uniform", lo1, hi1, lo2, hi2) | ("log_uniform", lo, hi)
    softcap: float = 0.0
    window: int = 0
    prefix_share: float = 0.0  # fraction of sequences that share the prefix blocks
    prefix_blocks: int = 0  # number of shared physical prefix blocks
    num_blocks: Optional[int] = None  # fixed pool size (else used blocks + slack)
    partition_tokens: int = 0  # split-K partition size the workload is run with (0: none)
    seed: int = 1000

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five decode shapes.  Seeds are 1000 + index.
WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_fp32", 4, 8, 2, 64, 16, "f32", ("uniform", 1, 100), num_blocks=64, seed=1000),
        Workload("tinyllama_1b", 64, 32, 4, 64, 16, "bf16", ("uniform", 128, 2048), seed=1001),
        Workload(
            "gemma2_2b", 256, 8, 4, 256, 128, "bf16", ("sum_uniform", 1, 512, 128, 512), softcap=50.0, window=0, seed=1002
        ),
        Workload(
            "llama3_8b", 128, 32, 8, 128, 16, "bf16", ("log_uniform", 256, 8192), prefix_share=0.3, prefix_blocks=64, seed=1003
        ),
        Workload(
            "long_splitk", 8, 32, 8, 128, 16, "bf16", ("uniform", 16384, 131072), partition_tokens=512, seed=1004
        ),
    ]
}


@dataclass
class Batch:
    """One decode step's inputs.  Tensors live on ``device``."""

    workload: Workload
    q: torch.Tensor  # [B, Hq, D]
    k_new: torch.Tensor  # [B, Hkv, D]  key of the token appended this step
    v_new: torch.Tensor  # [B, Hkv, D]
    slot_mapping: torch.Tensor  # [B] int64
    k_cache: torch.Tensor  # [num_blocks, Hkv, bs, D]
    v_cache: torch.Tensor
    block_tables: torch.Tensor  # [B, max_blocks_per_seq] int32, -1 padded
    context_lens: torch.Tensor  # [B] int32 (includes the appended token)
    live_per_block: torch.Tensor  # [num_blocks] int32, live rows at the start of each block (CPU)
    shared_blocks: torch.Tensor  # [prefix_blocks] int64 physical ids of shared blocks (CPU)
    prefilled: bool  # True: the slot of position L-1 already holds k_new / v_new's draw

    @property
    def num_blocks(self) -> int:
        return self.k_cache.shape[0]

    @property
    def max_blocks_per_seq(self) -> int:
        return self.block_tables.shape[1]

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max().item()) if self.context_lens.numel() else 0


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def sample_lengths(w: Workload, gen: torch.Generator, batch: int, max_len: Optional[int] = None) -> torch.Tensor:
    """Context lengths (int64, CPU) following the workload's recipe."""
    kind = w.lengths[0]
    if kind == "uniform":
        lo, hi = w.lengths[1], w.lengths[2]
        L = torch.randint(lo, hi + 1, (batch,), generator=gen)
    elif kind == "sum_uniform":
        a = torch.randint(w.lengths[1], w.lengths[2] + 1, (batch,), generator=gen)
        c = torch.randint(w.lengths[3], w.lengths[4] + 1, (batch,), generator=gen)
        L = a + c
    elif kind == "log_uniform":
        lo, hi = math.log(w.lengths[1]), math.log(w.lengths[2])
        u = torch.rand((batch,), generator=gen, dtype=torch.float64)
        L = torch.floor(torch.exp(lo + (hi - lo) * u)).to(torch.int64)
        L = L.clamp(w.lengths[1], w.lengths[2])
    elif kind == "fixed":
        L = torch.tensor(list(w.lengths[1]), dtype=torch.int64)
        assert L.numel() == batch
    else:
        raise ValueError(f"unknown length recipe {kind!r}")
    if max_len is not None:
        L = L.clamp(max=max_len)
    return L


def _randn(shape, gen_dev: torch.Generator, device, dtype, chunk_rows: int = 1 << 14) -> torch.Tensor:
    """N(0,1) drawn in fp32 and rounded (RNE) to ``dtype``, in chunks along dim 0."""
    out = torch.empty(shape, dtype=dtype, device=device)
    n0 = shape[0]
    for s in range(0, n0, chunk_rows):
        e = min(n0, s + chunk_rows)
        out[s:e] = torch.randn((e - s,) + tuple(shape[1:]), generator=gen_dev, device=device, dtype=torch.float32).to(dtype)
    return out


def make_batch(
    w: Workload,
    *,
    seed: Optional[int] = None,
    device: str | torch.device = "cpu",
    batch: Optional[int] = None,
    max_len: Optional[int] = None,
    lengths: Optional[list] = None,
    prefilled: bool = False,
    slack: float = 0.05,
    q_scale: float = 1.0,
) -> Batch:
    """Draw one decode batch.

    ``prefilled=False``: positions ``[0, L-1)`` of each sequence are live in the
    pool and the step's new row (``k_new``/``v_new``) still has to be appended at
    position ``L-1``.  ``prefilled=True``: positions ``[0, L)`` are live (the pool
    already holds the step's token), for decode-only checks.
    """
    seed = w.seed if seed is None else seed
    B = w.batch if batch is None else batch
    bs, Hkv, D, Hq = w.block_size, w.num_kv_heads, w.head_dim, w.num_q_heads
    g = _gen(seed)

    if lengths is not None:
        L = torch.tensor(list(lengths), dtype=torch.int64)
        B = L.numel()
    else:
        L = sample_lengths(w, g, B, max_len)

    # Blocks each sequence needs to hold L tokens (the appended one included).
    need = (L + bs - 1) // bs
    # Prefix sharing: chosen sequences map their first n_sh logical blocks to the
    # shared physical blocks.  Only full blocks strictly before the block that
    # receives this step's token are shared, so the append never writes a
    # shared block.
    n_sh = torch.zeros(B, dtype=torch.int64)
    if w.prefix_share > 0 and w.prefix_blocks > 0 and B > 0:
        n_sharers = int(round(w.prefix_share * B))
        sharers = torch.randperm(B, generator=g)[:n_sharers]
        n_sh[sharers] = torch.minimum(torch.full_like(L[sharers], w.prefix_blocks), (L[sharers] - 1).clamp(min=0) // bs)
    n_shared_pool = w.prefix_blocks if int(n_sh.sum()) > 0 else 0
    private = need - n_sh
    used = n_shared_pool + int(private.sum())
    if w.num_blocks is not None:
        num_blocks = w.num_blocks
        if used > num_blocks:
            raise ValueError(f"{w.name}: {used} blocks needed, pool has {num_blocks}")
    else:
        num_blocks = max(1, used + int(math.ceil(slack * used)))

    perm = torch.randperm(num_blocks, generator=g)
    shared_ids = perm[:n_shared_pool].clone()
    max_blocks = max(1, int(need.max().item()) if B > 0 else 1)
    tables = torch.full((B, max_blocks), -1, dtype=torch.int32)
    live = torch.zeros(num_blocks, dtype=torch.int32)
    live[shared_ids] = bs
    pos = n_shared_pool
    n_live_tok = L if prefilled else (L - 1).clamp(min=0)
    for b in range(B):
        k = int(n_sh[b])
        if k:
            tables[b, :k] = shared_ids[:k].to(torch.int32)
        m = int(private[b])
        ids = perm[pos : pos + m]
        pos += m
        tables[b, k : k + m] = ids.to(torch.int32)
        for i in range(m):
            li = k + i
            live[ids[i]] = int(max(0, min(bs, int(n_live_tok[b]) - li * bs)))

    slots = torch.full((B,), -1, dtype=torch.int64)
    for b in range(B):
        if L[b] > 0:
            t = int(L[b]) - 1
            slots[b] = int(tables[b, t // bs]) * bs + t % bs

    dev = torch.device(device)
    gd = torch.Generator(device=dev)
    gd.manual_seed(seed * 7919 + 17)
    dt = w.torch_dtype
    q = _randn((B, Hq, D), gd, dev, dt)
    if q_scale != 1.0:
        q = (q.float() * q_scale).to(dt)
    k_new = _randn((B, Hkv, D), gd, dev, dt)
    v_new = _randn((B, Hkv, D), gd, dev, dt)
    k_cache = _randn((num_blocks, Hkv, bs, D), gd, dev, dt, chunk_rows=max(1, (1 << 24) // (Hkv * bs * D)))
    v_cache = _randn((num_blocks, Hkv, bs, D), gd, dev, dt, chunk_rows=max(1, (1 << 24) // (Hkv * bs * D)))
    dead = (torch.arange(bs).view(1, bs) >= live.view(-1, 1)).to(dev)  # [num_blocks, bs]
    dead = dead.view(num_blocks, 1, bs, 1)
    nan = torch.tensor(float("nan"), dtype=dt, device=dev)
    k_cache = torch.where(dead, nan, k_cache)
    v_cache = torch.where(dead, nan, v_cache)

    return Batch(
        workload=w,
        q=q,
        k_new=k_new,
        v_new=v_new,
        slot_mapping=slots.to(dev),
        k_cache=k_cache.contiguous(),
        v_cache=v_cache.contiguous(),
        block_tables=tables.to(dev),
        context_lens=L.to(torch.int32).to(dev),
        live_per_block=live,
        shared_blocks=shared_ids,
        prefilled=prefilled,
    )


def make_multi_queries(batch: Batch, q_len: int, seed: Optional[int] = None, device=None) -> dict:
    """Multi-query inputs for ``batch``: ``q`` ``[B, T, Hq, D]`` for the last
    ``T = q_len`` positions of every sequence, the new rows ``k_new``/``v_new``
    ``[B*T, Hkv, D]`` and their slots ``[B*T]`` (int64; position L-T+j of
    sequence b at row b*T + j, -1 where that position is < 0), all N(0,1)
    drawn in fp32 and rounded to the workload's dtype."""
    w = batch.workload
    B, T = batch.context_lens.numel(), int(q_len)
    dev = torch.device(device) if device is not None else batch.q.device
    gd = torch.Generator(device=dev)
    gd.manual_seed((w.seed if seed is None else seed) * 104729 + 31 * T + 5)
    dt = w.torch_dtype
    q = _randn((B, T, w.num_q_heads, w.head_dim), gd, dev, dt)
    k_new = _randn((B * T, w.num_kv_heads, w.head_dim), gd, dev, dt)
    v_new = _randn((B * T, w.num_kv_heads, w.head_dim), gd, dev, dt)
    L = batch.context_lens.to("cpu").to(torch.int64)
    tables = batch.block_tables.to("cpu")
    bs = w.block_size
    slots = torch.full((B * T,), -1, dtype=torch.int64)
    for b in range(B):
        for j in range(T):
            t = int(L[b]) - T + j
            if t >= 0:
                slots[b * T + j] = int(tables[b, t // bs]) * bs + t % bs
    return {"q": q, "k_new": k_new, "v_new": v_new, "slot_mapping": slots.to(dev)}


def make_prefill_inputs(batch: Batch, q_lens, seed: Optional[int] = None, device=None) -> dict:
    """Prefill inputs for ``batch``: sequence b's last ``q_lens[b]`` positions
    are new.  Returns ``q`` ``[total, Hq, D]``, ``k_new``/``v_new`` ``[total,
    Hkv, D]``, their slots ``[total]`` (int64), ``cu_q_lens`` ``[B+1]`` (int32)
    and ``max_q_len``, N(0,1) drawn in fp32 and rounded to the workload's dtype."""
    w = batch.workload
    ql = [int(x) for x in q_lens]
    B = batch.context_lens.numel()
    assert len(ql) == B
    total = sum(ql)
    dev = torch.device(device) if device is not None else batch.q.device
    gd = torch.Generator(device=dev)
    gd.manual_seed((w.seed if seed is None else seed) * 15485863 + total)
    dt = w.torch_dtype
    q = _randn((max(total, 1), w.num_q_heads, w.head_dim), gd, dev, dt)[:total]
    k_new = _randn((max(total, 1), w.num_kv_heads, w.head_dim), gd, dev, dt)[:total]
    v_new = _randn((max(total, 1), w.num_kv_heads, w.head_dim), gd, dev, dt)[:total]
    L = batch.context_lens.to("cpu").to(torch.int64)
    tables = batch.block_tables.to("cpu")
    bs = w.block_size
    slots = torch.full((total,), -1, dtype=torch.int64)
    cu = [0]
    for b in range(B):
        for j in range(ql[b]):
            t = int(L[b]) - ql[b] + j
            if t >= 0:
                slots[cu[-1] + j] = int(tables[b, t // bs]) * bs + t % bs
        cu.append(cu[-1] + ql[b])
    return {"q": q.contiguous(), "k_new": k_new.contiguous(), "v_new": v_new.contiguous(),
            "slot_mapping": slots.to(dev), "cu_q_lens": torch.tensor(cu, dtype=torch.int32, device=dev),
            "max_q_len": max(ql) if ql else 0}


def order_for_cascade(batch: Batch):
    """Reorder a prefix-sharing batch for the cascade decode: the sequences
    whose tables start with all of the shared blocks come first.  Returns
    ``(batch, n_sharers, prefix_len)``; prefix_len = shared blocks * block_size
    rounded down to a multiple of 64 (0 when nothing is shared)."""
    w = batch.workload
    shared = batch.shared_blocks.tolist()
    k = len(shared)
    bs = w.block_size
    prefix_len = (k * bs) // 64 * 64
    if k == 0 or prefix_len == 0:
        return batch, 0, 0
    nblk = prefix_len // bs
    tables = batch.block_tables.to("cpu")
    ref = torch.tensor(shared[:nblk], dtype=torch.int32)
    is_sharer = [bool(torch.equal(tables[b, :nblk], ref)) for b in range(tables.shape[0])]
    order = [b for b in range(len(is_sharer)) if is_sharer[b]] + [b for b in range(len(is_sharer)) if not is_sharer[b]]
    idx = torch.tensor(order, dtype=torch.long)
    dev = batch.q.device
    kw = {f: getattr(batch, f) for f in ("workload", "k_cache", "v_cache", "live_per_block", "shared_blocks",
                                          "prefilled")}
    kw.update(q=batch.q[idx.to(dev)], k_new=batch.k_new[idx.to(dev)], v_new=batch.v_new[idx.to(dev)],
              slot_mapping=batch.slot_mapping[idx.to(batch.slot_mapping.device)],
              block_tables=batch.block_tables[idx.to(batch.block_tables.device)],
              context_lens=batch.context_lens[idx.to(batch.context_lens.device)])
    return Batch(**kw), sum(is_sharer), prefix_len


def kv_bytes(batch: Batch, unique: bool = False, window: Optional[int] = None) -> int:
    """KV bytes one decode pass must read: sum over sequences of
    ``L_eff * Hkv * 2 * D * elem_bytes`` (``L_eff`` = attended positions).
    With ``unique=True`` a shared prefix block is counted once."""
    w = batch.workload
    W = w.window if window is None else window
    L = batch.context_lens.to("cpu").to(torch.int64)
    s0 = (L - W).clamp(min=0) if W > 0 else torch.zeros_like(L)
    per_tok = w.num_kv_heads * 2 * w.head_dim * w.elem_bytes
    logical = int((L - s0).sum()) * per_tok
    if not unique or batch.shared_blocks.numel() == 0:
        return logical
    bs = w.block_size
    tables = batch.block_tables.to("cpu")
    shared = set(int(x) for x in batch.shared_blocks)
    seen = set()
    total = 0
    for b in range(L.numel()):
        lo, hi = int(s0[b]), int(L[b])
        if hi <= lo:
            continue
        for i in range(lo // bs, (hi + bs - 1) // bs):
            blk = int(tables[b, i])
            ntok = min(hi, (i + 1) * bs) - max(lo, i * bs)
            if blk in shared:
                if blk in seen:
                    continue
                seen.add(blk)
            total += ntok
    return total * per_tok
