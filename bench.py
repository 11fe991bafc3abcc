"""Paged decode benchmark: one step = KV append + paged decode attention for one
synthetic batch, through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints one JSON line (rank 0).  ``value`` is decode tokens/s over all ranks
(one new token per sequence per step), timed on the device with CUDA events
over exactly K steps replayed from a CUDA graph, inputs resident in HBM.  L2
is defeated by rotating over several copies of the KV pool whose total is a
multiple of the L2 size.  ``roofline`` reports the decode launch's achieved
HBM bandwidth on the algorithmic KV bytes; ``e2e`` repeats the measurement
through the public Python API with the step's inputs copied from pinned host
memory and the output copied back inside the timed region; ``cpu_baseline``
times the fp64 CPU oracle on a bounded sample of the same workload.

Multi-GPU (torchrun): every rank runs its own independent batch (different
seed); there is no data-path collective.  Time = max over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from paged_kv_cache_473_b200 import workloads as wl  # noqa: E402

METRIC = "paged decode tokens/s and achieved HBM GB/s (% of B200 peak) per batch shape"
HEADLINE = "tinyllama_1b"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# Decode launches are bracketed by timing events on every EVENT_EVERY-th step
# only: an event node between graph kernels stops the graph from overlapping the
# next launch, which on the 65 MB TinyLlama step alone costs ~8 us per step.
EVENT_EVERY = 10
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
# The decode shapes whose line carries its own roofline, end-to-end figure and
# CPU baselines beside the headline (the shapes the >= 70 % target names, and
# the largest one).
DATA = "synthetic (seeded; q/k/v ~ N(0,1), shuffled physical blocks, NaN canaries in dead slots)"
TARGET_SHAPES = ("gemma2_2b", "llama3_8b", "long_splitk")
L2_NOTE = ("L2 defeated: the timed steps rotate over copies of the KV pool totalling at least 4x the L2 size "
           "(one copy when the pool alone is that large)")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=HEADLINE, choices=list(wl.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--kernel", default="auto", choices=["auto", "cuda_core", "mma"])
    ap.add_argument("--no-split", action="store_true", help="one CTA per (sequence, kv head), no split-K")
    ap.add_argument("--unfused", action="store_true", help="separate append kernel (pa_write_kv) before the decode")
    ap.add_argument("--partition", type=int, default=-1, help="split-K partition tokens (0 auto; -1 workload's)")
    ap.add_argument("--shapes", default="auto", help="comma list of extra workloads to time, 'none', or 'auto'")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="bound on the CPU-oracle sample")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--op", default="decode", choices=["decode", "multi", "cascade", "prefill"],
                    help="the timed op: the decode step (default), multi-query rows, the cascade decode of the "
                         "prefix-sharing shape, or a paged prefill of whole prompts")
    ap.add_argument("--q-len", type=int, default=4, help="--op multi: query tokens per sequence")
    ap.add_argument("--prompts", type=int, default=16, help="--op prefill: prompts per step")
    ap.add_argument("--prompt-len", type=int, default=1024, help="--op prefill: tokens per prompt")
    return ap.parse_args()


# ---- distributed plumbing -----------------------------------------------------------


def dist_init(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def rank_seed(w: wl.Workload, rank: int) -> int:
    """Each rank draws an independent batch of the same shape."""
    return w.seed + 7919 * rank


# ---- clocks -------------------------------------------------------------------------

_REASON_BITS = {
    0x1: "gpu_idle",
    0x2: "applications_clocks_setting",
    0x4: "sw_power_cap",
    0x8: "hw_slowdown",
    0x10: "sync_boost",
    0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown",
    0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001
            self._nv = None

    def _run(self):
        nv = self._nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(get_r(self._h))
            except Exception:  # noqa: BLE001
                break
            time.sleep(0.0005)

    def __enter__(self):
        if self._nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        s = sorted(self.samples)
        reasons = [n for bit, n in _REASON_BITS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": s[len(s) // 2], "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(s)}


# ---- helpers --------------------------------------------------------------------------


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:  # noqa: BLE001
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak() -> float:
    """Dense bf16 tensor peak (TFLOP/s) for a kernel timed on its own: the
    measured burst figure, else the pool's earlier measurement."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:  # noqa: BLE001
        return FALLBACK_BF16_TFLOPS


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_473_b200", "csrc")
    for n in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(n.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel_key: str):
    """dram bytes per launch from a committed ncu summary, if taken on the current sources."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            d = json.load(f)
        e = d[workload][kernel_key]
        if e.get("source_hash") != kernel_source_hash():
            return None
        return int(e["dram_bytes_per_launch"])
    except Exception:  # noqa: BLE001
        return None


def pool_copies(pool_bytes: int, l2_bytes: int) -> int:
    """Rotate over enough pool copies that one pass over them is >= 4x L2."""
    return max(1, min(16, math.ceil(4 * l2_bytes / max(1, pool_bytes))))


# ---- our implementation ------------------------------------------------------------------


class Runner:
    """One workload on this GPU: rotating KV pools, persistent output/workspace.

    A step appends the batch's new key/value rows at position L-1 of every
    sequence and runs the paged decode: fused in one call (pa_decode_step), or
    as pa_write_kv followed by pa_decode / pa_decode_splitk (``fused=False``).
    """

    def __init__(self, w: wl.Workload, rank: int, kernel: str, split: bool, partition: int, fused: bool = True):
        import paged_kv_cache_473_b200 as pa

        self.pa = pa
        self.w = w
        self.kernel = kernel
        self.split = split
        self.fused = fused
        self.batch = wl.make_batch(w, seed=rank_seed(w, rank), device="cuda")
        b = self.batch
        self.B = b.q.shape[0]
        l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
        pool_bytes = 2 * b.k_cache.numel() * b.k_cache.element_size()
        self.R = pool_copies(pool_bytes, l2)
        self.pools = [(b.k_cache, b.v_cache)] + [(b.k_cache.clone(), b.v_cache.clone()) for _ in range(self.R - 1)]
        self.pool_bytes_total = pool_bytes * self.R
        self.max_ctx = max(1, b.max_context_len)
        # 0: the library's schedule (balanced stream schedule on the tensor-core path)
        self.partition = w.partition_tokens if partition < 0 else partition
        nbytes = pa.decode_splitk_workspace_size(self.B, w.num_q_heads, w.head_dim, self.max_ctx, self.partition,
                                                 w.num_kv_heads)
        self.ws = torch.zeros(max(16, nbytes), dtype=torch.uint8, device="cuda")  # zero before first use
        self.out = torch.empty_like(b.q)
        self.kv_bytes = wl.kv_bytes(b)
        self.kv_bytes_unique = wl.kv_bytes(b, unique=True)
        self.launches_per_step = 0
        self.schedule = "none"  # the library's schedule for the decode (pa_last_decode_schedule)

    def inputs(self):
        b = self.batch
        return dict(q=b.q, k_new=b.k_new, v_new=b.v_new, slot_mapping=b.slot_mapping, block_tables=b.block_tables,
                    context_lens=b.context_lens)

    def append(self, r, x):
        kc, vc = self.pools[r]
        self.pa.write_kv(x["k_new"], x["v_new"], x["slot_mapping"], kc, vc)
        return self.pa.last_launch_count()

    def decode(self, r, x):
        w = self.w
        kc, vc = self.pools[r]
        if self.fused:
            self.pa.decode_step(x["q"], x["k_new"], x["v_new"], kc, vc, x["block_tables"], x["context_lens"], w.scale,
                                w.softcap, w.window, split=self.split, max_context_len=self.max_ctx,
                                partition_tokens=self.partition, out=self.out, workspace=self.ws, kernel=self.kernel)
        elif self.split:
            self.pa.decode_splitk(x["q"], kc, vc, x["block_tables"], x["context_lens"], w.scale, w.softcap, w.window,
                                  max_context_len=self.max_ctx, partition_tokens=self.partition, out=self.out,
                                  workspace=self.ws, kernel=self.kernel)
        else:
            self.pa.decode(x["q"], kc, vc, x["block_tables"], x["context_lens"], w.scale, w.softcap, w.window,
                           out=self.out, kernel=self.kernel)
        return self.pa.last_launch_count()

    def step(self, r, x=None, ev=None):
        """One step on pool r.  ``ev``: (start, end) events around the decode launch(es)."""
        x = self.inputs() if x is None else x
        n = 0 if self.fused else self.append(r, x)
        if ev is not None:
            ev[0].record()
        n += self.decode(r, x)
        self.schedule = self.pa.last_decode_schedule()
        if ev is not None:
            ev[1].record()
        self.launches_per_step = n

    def timed_graph(self, K: int):
        """Capture K steps (pool i % R), with external timing events around the
        decode of every EVENT_EVERY-th step."""
        ev = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
              for _ in range(0, K, EVENT_EVERY)]
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for i in range(K):
                    self.step(i % self.R, ev=ev[i // EVENT_EVERY] if i % EVENT_EVERY == 0 else None)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        return g, ev


class MultiRunner(Runner):
    """Multi-query rows on one workload: T query tokens per sequence whose K/V
    rows are already in the cache (positions L-T .. L-1), attending causally
    (pa_decode_multi, library-chosen split).  A step is only that call."""

    def __init__(self, w: wl.Workload, rank: int, q_len: int):
        super().__init__(w, rank, "auto", True, 0, fused=True)
        b = self.batch
        for kc, vc in self.pools:  # make position L-1 live too: every query position is in the cache
            self.pa.write_kv(b.k_new, b.v_new, b.slot_mapping, kc, vc)
        self.T = q_len
        self.q = wl.make_multi_queries(b, q_len)["q"]
        self.out = torch.empty_like(self.q)
        nbytes = self.pa.decode_multi_workspace_size(self.B, q_len, w.num_q_heads, w.head_dim, self.max_ctx, 0,
                                                     w.num_kv_heads)
        self.ws = torch.zeros(max(16, nbytes), dtype=torch.uint8, device="cuda")
        torch.cuda.synchronize()

    def decode(self, r, x):
        w, b = self.w, self.batch
        kc, vc = self.pools[r]
        self.pa.decode_multi(self.q, kc, vc, b.block_tables, b.context_lens, w.scale, w.softcap, w.window,
                             split=True, max_context_len=self.max_ctx, partition_tokens=0, out=self.out,
                             workspace=self.ws)
        return self.pa.last_launch_count()

    def step(self, r, x=None, ev=None):
        if ev is not None:
            ev[0].record()
        n = self.decode(r, None)
        if ev is not None:
            ev[1].record()
        self.launches_per_step = n


class PrefillRunner(Runner):
    """Paged prefill of whole prompts (pa_prefill: append + causal attention)
    with a workload's heads: ``n_prompts`` prompts of ``prompt_len`` tokens.
    A step is only that call."""

    def __init__(self, w: wl.Workload, rank: int, n_prompts: int, prompt_len: int):
        w = w.replace(prefix_share=0.0, batch=n_prompts, lengths=("fixed", (prompt_len,) * n_prompts))
        super().__init__(w, rank, "auto", False, -1, fused=True)
        b = self.batch
        self.x = wl.make_prefill_inputs(b, [prompt_len] * n_prompts)
        self.T = prompt_len
        self.out = torch.empty_like(self.x["q"])
        # causal attention flops: QK^T and PV, 2 flops per multiply-add, T(T+1)/2 pairs per prompt and head
        self.flops = n_prompts * 4 * w.num_q_heads * w.head_dim * prompt_len * (prompt_len + 1) // 2
        torch.cuda.synchronize()

    def decode(self, r, x):
        w, b, x = self.w, self.batch, self.x
        kc, vc = self.pools[r]
        self.pa.prefill(x["q"], x["k_new"], x["v_new"], x["slot_mapping"], x["cu_q_lens"], kc, vc, b.block_tables,
                        b.context_lens, w.scale, w.softcap, w.window, max_q_len=x["max_q_len"], out=self.out)
        return self.pa.last_launch_count()

    def step(self, r, x=None, ev=None):
        if ev is not None:
            ev[0].record()
        n = self.decode(r, None)
        if ev is not None:
            ev[1].record()
        self.launches_per_step = n


class CascadeRunner(Runner):
    """The prefix-sharing workload through pa_decode_cascade: the sequences
    that hold the whole shared prefix go first and read it once per kv head.
    A step is only that call (the KV already holds every position)."""

    def __init__(self, w: wl.Workload, rank: int):
        super().__init__(w, rank, "auto", True, 0, fused=True)
        b = self.batch
        for kc, vc in self.pools:  # position L-1 live too, as in the decode step after its append
            self.pa.write_kv(b.k_new, b.v_new, b.slot_mapping, kc, vc)
        self.batch, self.n_sharers, self.prefix_len = wl.order_for_cascade(b)
        nbytes = self.pa.decode_cascade_workspace_size(self.B, w.num_q_heads, w.head_dim, self.max_ctx,
                                                       self.prefix_len, 0, w.num_kv_heads)
        self.ws = torch.zeros(max(16, nbytes), dtype=torch.uint8, device="cuda")
        torch.cuda.synchronize()

    def decode(self, r, x):
        w, b = self.w, self.batch
        kc, vc = self.pools[r]
        self.pa.decode_cascade(b.q, kc, vc, b.block_tables, b.context_lens, w.scale, w.softcap, w.window,
                               n_sharers=self.n_sharers, prefix_len=self.prefix_len, max_context_len=self.max_ctx,
                               out=self.out, workspace=self.ws)
        return self.pa.last_launch_count()

    def step(self, r, x=None, ev=None):
        if ev is not None:
            ev[0].record()
        n = self.decode(r, None)
        if ev is not None:
            ev[1].record()
        self.launches_per_step = n


class DecodeOnlyRunner(Runner):
    """The decode without the append (pa_decode_splitk, library's schedule):
    the cache already holds position L-1 of every sequence, written once up
    front, so a step is only the attention."""

    def __init__(self, w: wl.Workload, rank: int):
        # fused=True: every launch of a step belongs to the timed op, as in the step
        super().__init__(w, rank, "auto", True, 0, fused=True)
        b = self.batch
        for kc, vc in self.pools:
            self.pa.write_kv(b.k_new, b.v_new, b.slot_mapping, kc, vc)
        torch.cuda.synchronize()

    def decode(self, r, x):
        w, b = self.w, self.batch
        kc, vc = self.pools[r]
        self.pa.decode_splitk(b.q, kc, vc, b.block_tables, b.context_lens, w.scale, w.softcap, w.window,
                              max_context_len=self.max_ctx, partition_tokens=0, out=self.out, workspace=self.ws)
        return self.pa.last_launch_count()

    def step(self, r, x=None, ev=None):
        if ev is not None:
            ev[0].record()
        n = self.decode(r, None)
        if ev is not None:
            ev[1].record()
        self.launches_per_step = n


def run_timed(runner: Runner, K: int, W: int, world: int, device_index: int):
    """Warm up W steps, then time exactly K graph-replayed steps."""
    for i in range(W):
        runner.step(i % runner.R)
    torch.cuda.synchronize()
    g, ev = runner.timed_graph(K)
    # Warm the graph once (the replay itself is not counted).
    g.replay()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(device_index) as clk:
        start.record()
        g.replay()
        end.record()
        torch.cuda.synchronize()
    barrier(world)
    total_ms = start.elapsed_time(end)
    dec_ms = [a.elapsed_time(b) for a, b in ev]
    del g
    return total_ms, sum(dec_ms) / len(dec_ms), clk.summary()


class _Rt:
    """The few CUDA runtime calls the end-to-end leg issues per step, through
    ctypes on the runtime library torch has loaded (the same runtime instance,
    so torch's streams are valid handles)."""

    def __init__(self):
        import ctypes

        lib = ctypes.CDLL("libcudart.so.12")
        vp, sz, ui = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint
        lib.cudaMemcpyAsync.argtypes = [vp, vp, sz, ctypes.c_int, vp]
        lib.cudaEventRecord.argtypes = [vp, vp]
        lib.cudaStreamWaitEvent.argtypes = [vp, vp, ui]
        lib.cudaEventCreateWithFlags.argtypes = [ctypes.POINTER(vp), ui]
        lib.cudaEventDestroy.argtypes = [vp]
        self.lib, self.ct = lib, ctypes

    def event(self):
        h = self.ct.c_void_p()
        assert self.lib.cudaEventCreateWithFlags(self.ct.byref(h), 2) == 0  # cudaEventDisableTiming
        return h.value


def run_e2e(runner: Runner, K: int, world: int):
    """End-to-end steps through the C ABI with host buffers, pipelined as a
    serving loop runs them.  Every step copies its inputs (packed in one pinned
    buffer) host -> device on a copy stream (cudaMemcpyAsync), calls
    pa_decode_step on the compute stream once they have landed, and copies its
    output device -> host on a third stream.  Inputs and outputs are
    double-buffered, so step i+1's input copy and step i-1's output copy
    overlap step i's kernel; every step's two copies lie inside the timed
    region (events on the compute stream, which waits for the last output copy).
    The arguments of each buffer's call are marshalled once, before timing.
    Returns (ms, h2d bytes per step, d2h bytes per step, host ms per step spent
    issuing the calls)."""
    import ctypes

    from paged_kv_cache_473_b200 import _binding as bnd

    b, w = runner.batch, runner.w
    names = ("q", "k_new", "v_new", "block_tables", "context_lens")
    srcs = [getattr(b, n).contiguous() for n in names]
    offs, total = [], 0
    for t in srcs:  # 256-byte aligned slots in one byte buffer
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    host = torch.empty(total, dtype=torch.uint8).pin_memory()
    for t, o in zip(srcs, offs):
        host[o : o + t.numel() * t.element_size()].copy_(t.cpu().view(-1).view(torch.uint8))
    bufs = [torch.empty(total, dtype=torch.uint8, device="cuda") for _ in range(2)]
    outs = [torch.empty_like(runner.out) for _ in range(2)]
    out_hosts = [torch.empty(b.q.shape, dtype=b.q.dtype).pin_memory() for _ in range(2)]
    h2d = total
    d2h = out_hosts[0].numel() * out_hosts[0].element_size()
    rt = _Rt()
    compute = torch.cuda.current_stream()
    copy_in, copy_out = torch.cuda.Stream(), torch.cuda.Stream()
    s_comp, s_in, s_out = compute.cuda_stream, copy_in.cuda_stream, copy_out.cuda_stream
    landed, done, read = [rt.event(), rt.event()], [rt.event(), rt.event()], [rt.event(), rt.event()]
    nb, hkv, bs, d = runner.pools[0][0].shape
    hq = b.q.shape[1]
    step = bnd._lib().pa_decode_step
    kern = bnd.KERNELS[runner.kernel]
    ptoks = runner.partition if runner.split else -1
    wsb = runner.ws.numel() * runner.ws.element_size()
    calls = {}  # (buffer j, pool r) -> marshalled arguments
    for j in range(2):
        base = bufs[j].data_ptr()
        for r in range(runner.R):
            kc, vc = runner.pools[r]
            calls[j, r] = (ctypes.c_void_p(base + offs[0]), ctypes.c_void_p(base + offs[1]),
                           ctypes.c_void_p(base + offs[2]), ctypes.c_void_p(kc.data_ptr()),
                           ctypes.c_void_p(vc.data_ptr()), ctypes.c_void_p(base + offs[3]),
                           ctypes.c_void_p(base + offs[4]), runner.B, hq, hkv, d, bs, b.block_tables.shape[1], nb,
                           ctypes.c_float(w.scale), ctypes.c_float(w.softcap), w.window,
                           ctypes.c_void_p(outs[j].data_ptr()), bnd._dtype_code(b.q), ptoks, runner.max_ctx,
                           ctypes.c_void_p(runner.ws.data_ptr()), wsb, kern, ctypes.c_void_p(s_comp))
    hptr, optrs, dptrs = host.data_ptr(), [o.data_ptr() for o in out_hosts], [o.data_ptr() for o in outs]
    bptrs = [x.data_ptr() for x in bufs]
    lib = rt.lib
    used = [False, False]

    def one(i):
        j = i % 2
        if used[j]:
            lib.cudaStreamWaitEvent(s_in, done[j], 0)  # step i-2 has finished reading buffer j
        lib.cudaMemcpyAsync(bptrs[j], hptr, h2d, 1, s_in)  # host -> device
        lib.cudaEventRecord(landed[j], s_in)
        lib.cudaStreamWaitEvent(s_comp, landed[j], 0)
        if used[j]:
            lib.cudaStreamWaitEvent(s_comp, read[j], 0)  # step i-2's output has been copied out
        st = step(*calls[j, i % runner.R])
        if st != 0:
            raise bnd.PagedAttnError(st, "pa_decode_step")
        lib.cudaEventRecord(done[j], s_comp)
        lib.cudaStreamWaitEvent(s_out, done[j], 0)
        lib.cudaMemcpyAsync(optrs[j], dptrs[j], d2h, 2, s_out)  # device -> host
        lib.cudaEventRecord(read[j], s_out)
        used[j] = True

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record(compute)
    copy_in.wait_event(start)
    copy_out.wait_event(start)
    t0 = time.perf_counter()
    for i in range(K):
        one(i)
    host_ms = (time.perf_counter() - t0) * 1e3 / K
    compute.wait_stream(copy_out)
    compute.wait_stream(copy_in)
    end.record(compute)
    torch.cuda.synchronize()
    barrier(world)
    for e in landed + done + read:
        lib.cudaEventDestroy(e)
    # Every step has the same inputs: what came back to the host is bit for bit
    # the output of the device-timed steps.
    if not torch.equal(out_hosts[(K - 1) % 2].view(torch.int16), runner.out.cpu().view(torch.int16)):
        raise RuntimeError("end-to-end output differs from the device-timed step's")
    return start.elapsed_time(end), h2d, d2h, host_ms


class OracleSample:
    """The CPU oracle as it stands, timed on a bounded sample of one workload
    (the batch is copied to host memory once, outside any timing), on
    ``threads`` host threads (default: every core this process may run on)."""

    def __init__(self, w: wl.Workload, batch: wl.Batch, threads: int = 0):
        import oracle

        self.oracle = oracle
        self.w = w
        self.cpu = dict(q=batch.q.cpu(), k_new=batch.k_new.cpu(), v_new=batch.v_new.cpu(),
                        slots=batch.slot_mapping.cpu(), kc=batch.k_cache.cpu(), vc=batch.v_cache.cpu(),
                        tables=batch.block_tables.cpu(), lens=batch.context_lens.cpu())
        oracle.build()
        c = self.cpu
        self.B, self.hq = c["q"].shape[0], c["q"].shape[1]
        self.set_threads(threads)

    def set_threads(self, threads: int = 0):
        """Run on ``threads`` host threads (0: every core this process may run
        on), and re-estimate one sequence's cost at that count."""
        self.n_threads = threads if threads > 0 else len(os.sched_getaffinity(0))
        self.oracle.set_num_threads(self.n_threads)
        self.threads = self.oracle.num_threads()
        c = self.cpu
        t0 = time.perf_counter()
        self._decode([(0, h) for h in range(self.hq)])
        el = time.perf_counter() - t0
        self.per_seq = max(1e-6, el * float(c["lens"].double().mean()) / max(1, int(c["lens"][0])))

    def _decode(self, rows):
        c, w = self.cpu, self.w
        return self.oracle.decode(c["q"], c["kc"], c["vc"], c["tables"], c["lens"], w.scale, w.softcap, w.window,
                                  rows=rows)

    def run(self, seconds: float):
        """Whole steps (append + decode of every sequence) until ``seconds`` of
        work have run, or one step over the first n sequences when a whole step
        would take longer than that."""
        self.oracle.set_num_threads(self.n_threads)
        c = self.cpu
        B, hq = self.B, self.hq
        n_seq = B if self.per_seq * B <= seconds else max(1, int(seconds / self.per_seq))
        rows = None if n_seq == B else [(i, h) for i in range(n_seq) for h in range(hq)]
        steps = tokens = 0
        t0 = time.perf_counter()
        while True:
            self.oracle.write_kv(c["k_new"][:n_seq], c["v_new"][:n_seq], c["slots"][:n_seq], c["kc"], c["vc"])
            self._decode(rows)
            steps += 1
            tokens += n_seq
            el = time.perf_counter() - t0
            if el >= seconds or n_seq < B:
                break
        sample = (f"{steps} whole step(s): append + decode of all {B} sequences, fp64" if n_seq == B else
                  f"append + decode of the first {n_seq} of {B} sequences (all {hq} query heads), fp64")
        return {"value": tokens / el, "unit": "tokens/s", "cores": self.threads, "kind": "oracle", "sample": sample,
                "seconds": round(el, 3)}


def cpu_baselines(w: wl.Workload, batch: wl.Batch, seconds: float) -> dict:
    """The oracle on every host core and on one core, each on a bounded sample."""
    out = {}
    sampler = OracleSample(w, batch)
    for key, threads, secs in (("cpu_baseline", 0, seconds), ("cpu_baseline_1core", 1, seconds / 2)):
        sampler.set_threads(threads)
        info = sampler.run(secs)
        info["value"] = round(info["value"], 2)
        out[key] = info
    sampler.set_threads(0)
    return out


def workload_config(w: wl.Workload, batch: wl.Batch) -> dict:
    """The workload a line measures, as both arms (the library and the CPU
    oracle) describe it: the same dict on both lines."""
    return {
        "workload": w.name,
        "batch": int(batch.q.shape[0]),
        "num_q_heads": w.num_q_heads,
        "num_kv_heads": w.num_kv_heads,
        "head_dim": w.head_dim,
        "block_size": w.block_size,
        "lengths": list(w.lengths),
        "mean_context": round(float(batch.context_lens.double().mean()), 1),
        "softcap": w.softcap,
        "window": w.window,
        "prefix_share": w.prefix_share,
        "l2": L2_NOTE,
        "seed": "workload seed + 7919 * rank",
    }


SCHEDULE_NAMES = {
    "dynamic_merged": "work queue: warps claim (sequence, kv head, partition) items, merged in the decode kernel",
    "dynamic": "work queue: warps claim (sequence, kv head, partition) items, then the combine kernel",
    "grid": "one CTA per (partition, kv head, sequence), then the combine kernel",
    "single": "one CTA per (sequence, kv head)",
}


def describe_path(runner: Runner, kernel: str, l2_detail: str) -> dict:
    """How the library arm ran the workload (kept out of ``config``, which
    names only the workload)."""
    path = ("pa_decode_step" if runner.fused else "pa_write_kv + " + ("pa_decode_splitk" if runner.split else
                                                                      "pa_decode"))
    path += ((" (split-K, library schedule)" if runner.partition == 0 else
              f" (split-K, partition {runner.partition})") if runner.split else " (one CTA per sequence, kv head)")
    return {"call": path, "schedule": SCHEDULE_NAMES.get(runner.schedule, runner.schedule), "kernel": kernel,
            "l2": l2_detail}


def op_duration(runner: "Runner", total_ms: float, K: int, dec_ms: float):
    """Average duration of the decode op's launches.  In the fused step every
    launch of the timed region belongs to the op (append + decode + merge), so
    it is the timed region over K, with the gaps between graph launches
    included; otherwise the CUDA events sampled around the decode calls."""
    if runner.fused:
        return total_ms / K, (f"whole timed region / {K}: each step is only the fused op's "
                              f"{runner.launches_per_step} launch(es), back to back in a CUDA graph")
    return dec_ms, f"CUDA events around the decode call of every {EVENT_EVERY}th step of the timed graph"


def roofline_block(runner: Runner, op_ms: float, op_timing: str, dec_ms: float, peak: float, peak_kind: str,
                   traffic_key: str) -> dict:
    """HBM roofline of the decode op: algorithmic bytes are the UNIQUE KV bytes
    the step must read (a prefix block shared by several sequences counts
    once); the logical bytes (every sequence's own view) over the same time are
    reported beside them as the effective rate."""
    uniq, logical = runner.kv_bytes_unique, runner.kv_bytes
    achieved = uniq / (op_ms * 1e-3) / 1e9
    return {
        "bound": "hbm",
        "kernel": ("fused append + " if runner.fused else "") + (
            "split-K decode + LSE merge" if runner.split else "decode"),
        "achieved": round(achieved, 1),
        "peak": peak,
        "peak_kind": peak_kind,
        "unit": "GB/s",
        "frac": round(achieved / peak, 4),
        "traffic": recorded_traffic(runner.w.name, traffic_key),
        "traffic_scope": "dram bytes read + written by all launches of one step (ncu), per step",
        "algorithmic_bytes_per_launch": uniq,
        "logical_bytes_per_launch": logical,
        "effective_gbs_logical": round(logical / (op_ms * 1e-3) / 1e9, 1),
        "launch_ms": round(op_ms, 5),
        "launch_timing": op_timing,
        "launch_ms_event_sampled": round(dec_ms, 5),
    }


def traffic_key(runner: Runner) -> str:
    """Key of a step's record in profiles/traffic.json."""
    key = ("step" if runner.fused else "decode") + ("_splitk" if runner.split else "")
    return key + ("_dynamic" if runner.split and runner.partition == 0 and runner.w.partition_tokens else "")


def decode_line(w: wl.Workload, rank: int, kernel: str, split: bool, partition: int, fused: bool, K: int, W: int,
                world: int, dev_idx: int, peak: float, peak_kind: str, e2e: bool = True, cpu_seconds: float = 0.0):
    """Time the decode step on one workload and return the keys of a bench line
    for it: value (tokens/s over all ranks), ms_per_step, config, path,
    roofline, e2e (host buffers, copies inside the timed region), the CPU
    oracle baselines when ``cpu_seconds`` > 0, and the clocks."""
    runner = Runner(w, rank, kernel, split, partition, fused=fused)
    l2 = torch.cuda.get_device_properties(dev_idx).L2_cache_size
    l2_detail = f"rotating {runner.R} KV pool copies ({runner.pool_bytes_total / 1e6:.0f} MB, L2 {l2 / 1e6:.0f} MB)"
    total_ms, dec_ms, clocks = run_timed(runner, K, W, world, dev_idx)
    total_ms = max_over_ranks(total_ms, world)
    dec_ms = max_over_ranks(dec_ms, world)
    tokens = sum_over_ranks(runner.B * K, world)
    op_ms, op_timing = op_duration(runner, total_ms, K, dec_ms)
    line = {
        "value": round(tokens / (total_ms * 1e-3), 1),
        "unit": "tokens/s",
        "ms_per_step": round(total_ms / K, 5),
        "config": workload_config(w, runner.batch),
        "path": describe_path(runner, kernel, l2_detail),
        "roofline": roofline_block(runner, op_ms, op_timing, dec_ms, peak, peak_kind, traffic_key(runner)),
        "gpu_launches": K * runner.launches_per_step,
        "launches_per_step": runner.launches_per_step,
        "clocks": clocks,
    }
    if e2e and runner.fused:
        e2e_ms, h2d, d2h, host_ms = run_e2e(runner, K, world)
        e2e_ms = max_over_ranks(e2e_ms, world)
        line["e2e"] = {"value": round(tokens / (e2e_ms * 1e-3), 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms / K, 5),
                       "host_issue_ms_per_step": round(host_ms, 5),
                       "how": "pa_decode_step through the C ABI (ctypes, arguments marshalled once), eager; per "
                              "step one pinned H2D copy of the step's inputs and one D2H copy of its output "
                              "(cudaMemcpyAsync) on copy streams, double-buffered so they overlap the "
                              "neighbouring steps' kernels"}
    batch = runner.batch
    del runner
    torch.cuda.empty_cache()
    if cpu_seconds > 0 and world == 1 and rank == 0:
        line.update(cpu_baselines(w, batch, cpu_seconds))
    del batch
    torch.cuda.empty_cache()
    return line


def shape_summary(w: wl.Workload, rank: int, kernel: str, K: int, W: int, world: int, dev_idx: int, peak: float,
                  partition: int = -1):
    """A decode shape timed like the headline, without the end-to-end leg and
    CPU baselines: tokens/s and the HBM fraction on unique bytes."""
    d = decode_line(w, rank, kernel, True, partition, True, K, W, world, dev_idx, peak, "measured", e2e=False)
    r = d["roofline"]
    return {
        "tokens_per_s": d["value"],
        "ms_per_step": d["ms_per_step"],
        "decode_ms": r["launch_ms"],
        "decode_gbs": r["achieved"],
        "decode_frac": r["frac"],
        "effective_gbs_logical": r["effective_gbs_logical"],
        "launches_per_step": d["launches_per_step"],
        "kv_bytes_unique": r["algorithmic_bytes_per_launch"],
        "kv_bytes": r["logical_bytes_per_launch"],
        "traffic": r["traffic"],
        "path": d["path"]["call"],
        "schedule": d["path"]["schedule"],
    }


def multi_summary(w: wl.Workload, q_len: int, rank: int, K: int, W: int, world: int, dev_idx: int, peak: float):
    """Multi-query rows (pa_decode_multi) on a decode workload: tokens/s counts
    the B*T query tokens of a step."""
    runner = MultiRunner(w, rank, q_len)
    total_ms, _, _ = run_timed(runner, K, W, world, dev_idx)
    ms = total_ms / K
    gbs = runner.kv_bytes / (ms * 1e-3) / 1e9
    res = {
        "q_len": q_len,
        "tokens_per_s": round(runner.B * q_len / (ms * 1e-3), 1),
        "ms_per_step": round(ms, 5),
        "decode_gbs": round(gbs, 1),
        "decode_frac": round(gbs / peak, 4),
        "launches_per_step": runner.launches_per_step,
        "flop_per_kv_byte": q_len * w.num_q_heads // w.num_kv_heads * (1 if w.elem_bytes == 2 else 2),
        "kv_bytes": runner.kv_bytes,
    }
    del runner
    torch.cuda.empty_cache()
    return res


MULTI_SHAPES = (("tinyllama_1b", 4), ("llama3_8b", 4), ("gemma2_2b", 8))
PREFILL_SHAPES = (("llama3_8b", 16, 1024), ("tinyllama_1b", 16, 1024))


def prefill_summary(w: wl.Workload, n_prompts: int, prompt_len: int, rank: int, K: int, W: int, world: int,
                    dev_idx: int):
    """Paged prefill of whole prompts: prompt tokens/s and causal-attention
    TFLOP/s against the measured dense bf16 peak (tensor-bound)."""
    runner = PrefillRunner(w, rank, n_prompts, prompt_len)
    total_ms, _, _ = run_timed(runner, K, W, world, dev_idx)
    ms = total_ms / K
    tflops = runner.flops / (ms * 1e-3) / 1e12
    peak = tensor_peak()
    res = {
        "prompts": n_prompts,
        "prompt_len": prompt_len,
        "tokens_per_s": round(n_prompts * prompt_len / (ms * 1e-3), 1),
        "ms_per_step": round(ms, 5),
        "tflops": round(tflops, 1),
        "tensor_peak_tflops": peak,
        "tensor_frac": round(tflops / peak, 4),
        "launches_per_step": runner.launches_per_step,
    }
    del runner
    torch.cuda.empty_cache()
    return res


def cascade_summary(w: wl.Workload, rank: int, K: int, W: int, world: int, dev_idx: int, peak: float):
    """The prefix-sharing workload through the cascade decode: logical and
    unique KV GB/s (each shared block counted once)."""
    runner = CascadeRunner(w, rank)
    total_ms, _, _ = run_timed(runner, K, W, world, dev_idx)
    ms = total_ms / K
    res = {
        "n_sharers": runner.n_sharers,
        "prefix_len": runner.prefix_len,
        "tokens_per_s": round(runner.B / (ms * 1e-3), 1),
        "ms_per_step": round(ms, 5),
        "decode_gbs": round(runner.kv_bytes / (ms * 1e-3) / 1e9, 1),
        "decode_gbs_unique": round(runner.kv_bytes_unique / (ms * 1e-3) / 1e9, 1),
        "decode_frac_unique": round(runner.kv_bytes_unique / (ms * 1e-3) / 1e9 / peak, 4),
        "launches_per_step": runner.launches_per_step,
        "kv_bytes": runner.kv_bytes,
        "kv_bytes_unique": runner.kv_bytes_unique,
    }
    del runner
    torch.cuda.empty_cache()
    return res


def main_ours(args, world, rank, local):
    w = wl.WORKLOADS[args.workload]
    if args.op != "decode":
        return main_op(args, world, rank, local)
    split = not args.no_split
    K, W = args.steps, args.warmup
    peak, peak_kind = measured_peaks()
    one = world == 1 and rank == 0
    head = decode_line(w, rank, args.kernel, split, args.partition, not args.unfused, K, W, world, local, peak,
                       peak_kind, e2e=True, cpu_seconds=0.0 if args.no_cpu else args.cpu_seconds)
    line = {
        "metric": METRIC,
        "value": head["value"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": DATA,
        "config": head["config"],
        "path": head["path"],
        "roofline": head["roofline"],
        "e2e": head.get("e2e"),
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
    }
    for k in ("cpu_baseline", "cpu_baseline_1core"):
        if k in head:
            line[k] = head[k]
    if one and not args.unfused and split:
        # The attention alone (the append already done), timed the same way.
        dr = DecodeOnlyRunner(w, rank)
        d_total, d_dec, _ = run_timed(dr, K, W, 1, local)
        d_ms, _ = op_duration(dr, d_total, K, d_dec)
        line["decode_alone"] = {
            "ms_per_step": round(d_ms, 5),
            "tokens_per_s": round(dr.B / (d_ms * 1e-3), 1),
            "kv_gbs": round(dr.kv_bytes_unique / (d_ms * 1e-3) / 1e9, 1),
            "frac": round(dr.kv_bytes_unique / (d_ms * 1e-3) / 1e9 / peak, 4),
            "launches_per_step": dr.launches_per_step,
        }
        del dr
        torch.cuda.empty_cache()
    if one and args.shapes != "none":
        names = [n for n in wl.WORKLOADS if n not in (w.name, "tiny_fp32")] if args.shapes == "auto" else [
            s for s in args.shapes.split(",") if s]
        extra = {}
        for n in names:
            wn = wl.WORKLOADS[n]
            if n in TARGET_SHAPES:
                # A full line: roofline, end-to-end and CPU baselines of its own.
                extra[n] = decode_line(wn, rank, args.kernel, True, -1, True, 50, 5, world, local, peak, peak_kind,
                                       e2e=True, cpu_seconds=0.0 if args.no_cpu else args.cpu_seconds / 2)
            else:
                extra[n] = shape_summary(wn, rank, args.kernel, 50, 5, world, local, peak)
            if wn.partition_tokens:  # also the dynamic schedule
                extra[n + "@dynamic"] = shape_summary(wn, rank, args.kernel, 50, 5, world, local, peak, 0)
        for n, T in MULTI_SHAPES:
            if args.shapes == "auto" or n in names or n == w.name:
                extra[f"{n}@multi{T}"] = multi_summary(wl.WORKLOADS[n], T, rank, 50, 5, world, local, peak)
        for n in [n for n in wl.WORKLOADS if wl.WORKLOADS[n].prefix_share > 0]:
            if args.shapes == "auto" or n in names or n == w.name:
                extra[f"{n}@cascade"] = cascade_summary(wl.WORKLOADS[n], rank, 50, 5, world, local, peak)
        for n, P_, T in PREFILL_SHAPES:
            if args.shapes == "auto" or n in names or n == w.name:
                extra[f"{n}@prefill{P_}x{T}"] = prefill_summary(wl.WORKLOADS[n], P_, T, rank, 20, 3, world, local)
        line["per_shape"] = extra
    if rank == 0:
        print(json.dumps(line), flush=True)


def main_op(args, world, rank, local):
    """One of the other ops as the timed line (multi-query rows, cascade,
    prefill): the same timing and JSON keys as the decode line; the roofline is
    HBM for the attention ops and the tensor pipe for the prefill.  No
    end-to-end leg or CPU baseline (those belong to the decode step)."""
    w = wl.WORKLOADS[args.workload]
    if args.op == "multi":
        runner = MultiRunner(w, rank, args.q_len)
        per_step, what = runner.B * args.q_len, f"pa_decode_multi, T={args.q_len}"
    elif args.op == "cascade":
        runner = CascadeRunner(w, rank)
        per_step, what = runner.B, f"pa_decode_cascade, {runner.n_sharers} sharers of {runner.prefix_len} positions"
    else:
        runner = PrefillRunner(w, rank, args.prompts, args.prompt_len)
        per_step, what = args.prompts * args.prompt_len, f"pa_prefill, {args.prompts} x {args.prompt_len} tokens"
    K, W = args.steps, args.warmup
    total_ms, dec_ms, clocks = run_timed(runner, K, W, world, local)
    total_ms = max_over_ranks(total_ms, world)
    ms = total_ms / K
    value = sum_over_ranks(per_step * K, world) / (total_ms * 1e-3)
    if args.op == "prefill":
        peak, kind = tensor_peak(), "measured bf16 burst"
        achieved = runner.flops / (ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "peak_kind": kind,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": None,
                "algorithmic_flops_per_launch": runner.flops}
    else:
        peak, kind = measured_peaks()
        nbytes = runner.kv_bytes_unique if args.op == "cascade" else runner.kv_bytes
        achieved = nbytes / (ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "peak_kind": kind, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": None, "algorithmic_bytes_per_launch": nbytes}
    roof.update(kernel=what, launch_ms=round(ms, 5),
                launch_timing=f"whole timed region / {K}: each step is only the op's launches, in a CUDA graph")
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic (seeded; q/k/v ~ N(0,1), shuffled physical blocks)",
        "config": {"workload": w.name, "op": args.op, "batch": runner.B, "seed": "workload seed + 7919 * rank"},
        "roofline": roof, "e2e": None, "gpu_launches": K * runner.launches_per_step, "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def main_reference(args, rank):
    """The CPU oracle as the reference arm, on this run's workload and metric.
    Under torchrun only rank 0 works; the other ranks return at once."""
    if rank != 0:
        return
    w = wl.WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    b = wl.make_batch(w, seed=rank_seed(w, 0), device=dev)
    sampler = OracleSample(w, b)
    config = workload_config(w, b)
    del b
    K, W = args.steps, args.warmup
    budget = max(0.05, 120.0 / max(1, K + W))  # keep the whole run within a few minutes
    for _ in range(W):
        sampler.run(budget)
    t_tokens = t_secs = 0.0
    info = None
    for _ in range(K):
        info = sampler.run(budget)
        t_tokens += info["value"] * info["seconds"]
        t_secs += info["seconds"]
    value = t_tokens / t_secs
    world = int(os.environ.get("WORLD_SIZE", "1"))
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(1e3 * t_secs / K, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": DATA,
        "impl": "reference",
        "config": config,
        "path": {"call": "fp64 CPU oracle (C, OpenMP): append + decode", "kernel": "none", "l2": "n/a"},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": info["cores"], "kind": "oracle",
                         "sample": f"each step: {info['sample']}"},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        main_reference(args, int(os.environ.get("RANK", "0")))
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --impl ours needs a CUDA device")
    world, rank, local = dist_init(args)
    try:
        main_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
