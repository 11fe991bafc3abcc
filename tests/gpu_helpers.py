"""Helpers shared by the GPU parity tests: run a step through the C ABI and
compare it with the CPU oracle run on the same seeded inputs."""

from __future__ import annotations

import numpy as np
import torch

import oracle
import paged_kv_cache_473_b200 as pa

TOL = {torch.bfloat16: (2e-2, 2e-3), torch.float32: (1e-4, 1e-5)}


def to_dev(batch, device="cuda"):
    """Copy every tensor of a CPU batch to the GPU (the batch object is shared)."""
    import dataclasses

    kw = {}
    for f in dataclasses.fields(batch):
        x = getattr(batch, f.name)
        if isinstance(x, torch.Tensor) and f.name not in ("live_per_block", "shared_blocks"):
            x = x.to(device)
        kw[f.name] = x
    return type(batch)(**kw)


def gpu_step(b, *, kernel="auto", split=False, partition=0, softcap=None, window=None, append=True, max_ctx=None):
    """Append (optional) + decode on the GPU; returns (out, k_cache, v_cache) on the GPU."""
    w = b.workload
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    if append:
        pa.write_kv(b.k_new, b.v_new, b.slot_mapping, kc, vc)
    cap = w.softcap if softcap is None else softcap
    win = w.window if window is None else window
    if split:
        mx = max_ctx if max_ctx is not None else max(1, b.max_context_len)
        out = pa.decode_splitk(b.q, kc, vc, b.block_tables, b.context_lens, w.scale, cap, win,
                               max_context_len=mx, partition_tokens=partition, kernel=kernel)
    else:
        out = pa.decode(b.q, kc, vc, b.block_tables, b.context_lens, w.scale, cap, win, kernel=kernel)
    torch.cuda.synchronize()
    return out, kc, vc


def oracle_step(b_cpu, *, softcap=None, window=None, append=True, rows=None):
    """Append (optional) + decode with the CPU oracle; fp64 numpy result."""
    w = b_cpu.workload
    kc, vc = b_cpu.k_cache.clone(), b_cpu.v_cache.clone()
    if append:
        oracle.write_kv(b_cpu.k_new, b_cpu.v_new, b_cpu.slot_mapping, kc, vc)
    cap = w.softcap if softcap is None else softcap
    win = w.window if window is None else window
    out = oracle.decode(b_cpu.q, kc, vc, b_cpu.block_tables, b_cpu.context_lens, w.scale, cap, win, rows=rows)
    return out, kc, vc


def errors(got: torch.Tensor, ref: np.ndarray):
    g = got.detach().float().cpu().double().numpy()
    d = np.abs(g - ref)
    return float(np.max(d)) if d.size else 0.0, float(np.mean(d)) if d.size else 0.0


def assert_close(got: torch.Tensor, ref: np.ndarray, dtype, what=""):
    mx, mean = errors(got, ref)
    tmax, tmean = TOL[dtype]
    assert np.all(np.isfinite(got.float().cpu().numpy())), f"{what}: non-finite output"
    assert mx <= tmax and mean <= tmean, f"{what}: max-abs {mx:.3g} (tol {tmax}), mean-abs {mean:.3g} (tol {tmean})"
    return mx, mean


def bits(t: torch.Tensor) -> torch.Tensor:
    """Bit pattern view (NaN canaries compare equal)."""
    t = t.detach().cpu().contiguous()
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)
