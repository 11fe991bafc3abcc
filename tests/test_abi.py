"""The C ABI on a machine without a GPU: the library loads, exports every
function the header declares, and its host-side checks reject bad arguments
before anything touches the device."""

import ctypes
import os
import re

import pytest

import paged_kv_cache_473_b200 as pa
from paged_kv_cache_473_b200 import _binding as bnd

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "pagedattn.h")

# 16-byte aligned fake device addresses: never dereferenced, because every call
# below fails its host checks first.
A = 0x10000
MIS = 0x10004


def declared_functions():
    import glob
    src = "".join(open(h).read() for h in sorted(glob.glob(os.path.join(os.path.dirname(HEADER), "*.h"))))
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["pa_write_kv", "pa_decode", "pa_decode_splitk", "pa_decode_splitk_workspace_size",
              "pa_decode_splitk_partition", "pa_device_errors", "pa_error_string", "pa_last_launch_count", "pa_last_decode_schedule",
              "pa_decode_step", "pa_decode_splitk_noalloc", "pa_decode_multi", "pa_decode_multi_workspace_size",
              "pa_prefill", "pa_copy_blocks", "pa_bm_create", "pa_bm_append_slots", "pa_bm_block_tables",
              "pa_decode_cascade", "pa_decode_cascade_workspace_size"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(bnd._build.LIB)
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_error_strings():
    for s in range(5):
        assert pa.error_string(s)
    assert pa.error_string(99) == "unknown status"


def _decode(**kw):
    a = dict(q=A, k=A, v=A, bt=A, cl=A, B=2, hq=8, hkv=2, d=128, bs=16, mb=4, nb=8, scale=0.1, cap=0.0, win=0,
             out=A, dt=bnd.PA_BF16, kern=0)
    a.update(kw)
    return bnd.lib.pa_decode(a["q"], a["k"], a["v"], a["bt"], a["cl"], a["B"], a["hq"], a["hkv"], a["d"], a["bs"],
                             a["mb"], a["nb"], a["scale"], a["cap"], a["win"], a["out"], a["dt"], a["kern"], None)


@pytest.mark.parametrize(
    "kw,status",
    [
        (dict(q=None), bnd.PA_ERR_INVALID),
        (dict(out=None), bnd.PA_ERR_INVALID),
        (dict(q=MIS), bnd.PA_ERR_INVALID),
        (dict(k=MIS), bnd.PA_ERR_INVALID),
        (dict(bt=A + 2), bnd.PA_ERR_INVALID),
        (dict(hq=6, hkv=4), bnd.PA_ERR_INVALID),
        (dict(hkv=0), bnd.PA_ERR_INVALID),
        (dict(B=-1), bnd.PA_ERR_INVALID),
        (dict(dt=7), bnd.PA_ERR_INVALID),
        (dict(kern=9), bnd.PA_ERR_INVALID),
        (dict(cap=float("nan")), bnd.PA_ERR_INVALID),
        (dict(d=96), bnd.PA_ERR_UNSUPPORTED),
        (dict(bs=8), bnd.PA_ERR_UNSUPPORTED),
        (dict(bs=48), bnd.PA_ERR_UNSUPPORTED),
        (dict(hq=32, hkv=2), bnd.PA_ERR_UNSUPPORTED),
        (dict(B=70000), bnd.PA_ERR_UNSUPPORTED),
        (dict(nb=1 << 26, hkv=8, hq=8, bs=16), bnd.PA_ERR_UNSUPPORTED),
        (dict(dt=bnd.PA_F32, kern=2), bnd.PA_ERR_UNSUPPORTED),
    ],
)
def test_decode_host_checks(kw, status):
    assert _decode(**kw) == status
    assert pa.last_launch_count() == 0
    assert pa.last_decode_schedule() == "none"  # a refused call ran no schedule


def test_empty_batch_is_a_no_op():
    assert _decode(B=0, q=None, out=None) == bnd.PA_OK
    assert pa.last_launch_count() == 0
    assert pa.last_decode_schedule() == "none"


def test_schedule_names_match_the_header():
    """pa_schedule_t's values as the binding names them."""
    src = open(HEADER).read()
    body = src[src.index("typedef enum {\n  PA_SCHEDULE_NONE"):]
    body = body[:body.index("} pa_schedule_t;")]
    vals = {int(v): n for n, v in re.findall(r"PA_SCHEDULE_(\w+) = (\d+)", body)}
    assert {k: v.lower() for k, v in vals.items()} == bnd.SCHEDULES


def _splitk(**kw):
    a = dict(q=A, k=A, v=A, bt=A, cl=A, B=2, hq=8, hkv=2, d=128, bs=16, mb=4, nb=8, scale=0.1, cap=0.0, win=0,
             out=A, dt=bnd.PA_BF16, P=64, maxL=64, ws=A, wsb=1 << 30, kern=0)
    a.update(kw)
    return bnd.lib.pa_decode_splitk(a["q"], a["k"], a["v"], a["bt"], a["cl"], a["B"], a["hq"], a["hkv"], a["d"],
                                    a["bs"], a["mb"], a["nb"], a["scale"], a["cap"], a["win"], a["out"], a["dt"],
                                    a["P"], a["maxL"], a["ws"], a["wsb"], a["kern"], None)


@pytest.mark.parametrize(
    "kw,status",
    [
        (dict(P=100), bnd.PA_ERR_INVALID),
        (dict(P=-64), bnd.PA_ERR_INVALID),
        (dict(maxL=0), bnd.PA_ERR_INVALID),
        (dict(ws=None), bnd.PA_ERR_WORKSPACE),
        (dict(ws=MIS), bnd.PA_ERR_WORKSPACE),
        (dict(wsb=100), bnd.PA_ERR_WORKSPACE),
        (dict(P=64, maxL=64 * 8193), bnd.PA_ERR_UNSUPPORTED),
        (dict(d=32), bnd.PA_ERR_UNSUPPORTED),
    ],
)
def test_splitk_host_checks(kw, status):
    assert _splitk(**kw) == status


def test_workspace_size_formula():
    B, hq, d, maxL, P = 8, 32, 128, 131072, 512
    parts = -(-maxL // P)
    rows = B * hq * parts
    al = lambda x: (x + 255) // 256 * 256  # noqa: E731
    counters = (2 + 65534) * 4  # fixed counter region at the start of every split-K workspace
    assert counters == 256 * 1024
    assert pa.decode_splitk_workspace_size(B, hq, d, maxL, P, 8) == counters + al(rows * d * 4) + al(rows * 2 * 4)
    assert pa.decode_splitk_workspace_size(0, hq, d, maxL, P, 8) == 0
    # The library's choice (0) covers the dynamic schedule's partials too.
    assert pa.decode_splitk_workspace_size(B, hq, d, maxL, 0, 8) >= counters + al(rows * d * 4) + al(rows * 2 * 4)


def test_auto_partition_heuristic():
    # Explicit sizes pass through; auto picks 512 unless that leaves fewer than
    # 8 * 148 work units, halving down to 64.
    assert pa.decode_splitk_partition(8, 8, 131072, 1024) == 1024
    assert pa.decode_splitk_partition(8, 8, 131072, 0) == 512
    assert pa.decode_splitk_partition(128, 8, 8192, 0) == 512
    assert pa.decode_splitk_partition(64, 4, 2048, 0) == 256
    assert pa.decode_splitk_partition(4, 2, 100, 0) == 64


def test_write_kv_host_checks():
    f = bnd.lib.pa_write_kv
    assert f(None, A, A, 4, A, A, 8, 16, 2, 64, bnd.PA_BF16, None) == bnd.PA_ERR_INVALID
    assert f(A, A, A + 4, 4, A, A, 8, 16, 2, 64, bnd.PA_BF16, None) == bnd.PA_ERR_INVALID
    assert f(A, A, A, -1, A, A, 8, 16, 2, 64, bnd.PA_BF16, None) == bnd.PA_ERR_INVALID
    assert f(A, A, A, 4, A, A, 8, 16, 2, 4, bnd.PA_BF16, None) == bnd.PA_ERR_UNSUPPORTED
    assert f(A, A, A, 0, A, A, 8, 16, 2, 64, bnd.PA_BF16, None) == bnd.PA_OK


def _multi(**kw):
    a = dict(q=A, k=A, v=A, bt=A, cl=A, B=2, T=4, hq=8, hkv=2, d=128, bs=16, mb=4, nb=8, scale=0.1, cap=0.0, win=0,
             out=A, dt=bnd.PA_BF16, P=-1, maxL=64, ws=None, wsb=0)
    a.update(kw)
    return bnd.lib.pa_decode_multi(a["q"], a["k"], a["v"], a["bt"], a["cl"], a["B"], a["T"], a["hq"], a["hkv"],
                                   a["d"], a["bs"], a["mb"], a["nb"], a["scale"], a["cap"], a["win"], a["out"],
                                   a["dt"], a["P"], a["maxL"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize(
    "kw,status",
    [
        (dict(T=0), bnd.PA_ERR_INVALID),
        (dict(q=None), bnd.PA_ERR_INVALID),
        (dict(q=MIS), bnd.PA_ERR_INVALID),
        (dict(dt=bnd.PA_F32), bnd.PA_ERR_UNSUPPORTED),  # tensor-core path only
        (dict(T=17), bnd.PA_ERR_UNSUPPORTED),  # 17 * 4 query columns > 64
        (dict(d=96), bnd.PA_ERR_UNSUPPORTED),
        (dict(P=0), bnd.PA_ERR_WORKSPACE),  # split without a workspace
        (dict(P=100, ws=A, wsb=1 << 30), bnd.PA_ERR_INVALID),  # not a multiple of 64
        (dict(P=0, maxL=0, ws=A, wsb=1 << 30), bnd.PA_ERR_INVALID),
        (dict(B=0), bnd.PA_OK),
        (dict(B=0, P=0), bnd.PA_OK),
    ],
)
def test_multi_host_checks(kw, status):
    assert _multi(**kw) == status
    assert pa.last_launch_count() == 0


def test_multi_workspace_size_formula():
    B, T, hq, d, maxL, P = 8, 4, 32, 128, 8192, 512
    rows = B * T * hq * (-(-maxL // P))
    al = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert pa.decode_multi_workspace_size(B, T, hq, d, maxL, P, 8) == 256 * 1024 + al(rows * d * 4) + al(rows * 8)
    assert pa.decode_multi_workspace_size(B, T, hq, d, maxL, -1, 8) == 0


def _prefill(**kw):
    a = dict(q=A, kn=A, vn=A, sl=A, cu=A, total=64, maxq=32, k=A, v=A, bt=A, cl=A, B=2, hq=8, hkv=2, d=128, bs=16,
             mb=4, nb=8, scale=0.1, cap=0.0, win=0, out=A, dt=bnd.PA_BF16)
    a.update(kw)
    return bnd.lib.pa_prefill(a["q"], a["kn"], a["vn"], a["sl"], a["cu"], a["total"], a["maxq"], a["k"], a["v"],
                              a["bt"], a["cl"], a["B"], a["hq"], a["hkv"], a["d"], a["bs"], a["mb"], a["nb"],
                              a["scale"], a["cap"], a["win"], a["out"], a["dt"], None)


@pytest.mark.parametrize(
    "kw,status",
    [
        (dict(cu=None), bnd.PA_ERR_INVALID),
        (dict(cu=A + 2), bnd.PA_ERR_INVALID),
        (dict(total=-1), bnd.PA_ERR_INVALID),
        (dict(kn=None), bnd.PA_ERR_INVALID),  # k_new without v_new
        (dict(sl=None), bnd.PA_ERR_INVALID),
        (dict(dt=bnd.PA_F32), bnd.PA_ERR_UNSUPPORTED),
        (dict(hq=24, hkv=2), bnd.PA_ERR_UNSUPPORTED),  # group 12 > 8
        (dict(B=0), bnd.PA_OK),
        (dict(total=0), bnd.PA_OK),
        (dict(maxq=0), bnd.PA_OK),
    ],
)
def test_prefill_host_checks(kw, status):
    assert _prefill(**kw) == status
    assert pa.last_launch_count() == 0


@pytest.mark.parametrize(
    "kw,status",
    [
        (dict(n=-1), bnd.PA_ERR_INVALID),
        (dict(k=None), bnd.PA_ERR_INVALID),
        (dict(pairs=A + 2), bnd.PA_ERR_INVALID),
        (dict(dt=7), bnd.PA_ERR_INVALID),
        (dict(d=3, dt=bnd.PA_BF16, hkv=1, bs=1), bnd.PA_ERR_UNSUPPORTED),  # 6-byte blocks
        (dict(n=0), bnd.PA_OK),
    ],
)
def test_copy_blocks_host_checks(kw, status):
    a = dict(k=A, v=A, pairs=A, n=2, nb=8, bs=16, hkv=2, d=128, dt=bnd.PA_BF16)
    a.update(kw)
    assert bnd.lib.pa_copy_blocks(a["k"], a["v"], a["pairs"], a["n"], a["nb"], a["bs"], a["hkv"], a["d"], a["dt"],
                                  None) == status
    assert pa.last_launch_count() == 0


def _cascade(**kw):
    a = dict(B=4, hq=8, hkv=2, d=128, bs=16, mb=128, nb=512, dt=bnd.PA_BF16, nsh=2, plen=1024, P=0, maxL=2048,
             ws=None, wsb=0)
    a.update(kw)
    return bnd.lib.pa_decode_cascade(A, A, A, A, A, a["B"], a["hq"], a["hkv"], a["d"], a["bs"], a["mb"], a["nb"],
                                     0.1, 0.0, 0, A, a["dt"], a["nsh"], a["plen"], a["P"], a["maxL"], a["ws"],
                                     a["wsb"], None)


@pytest.mark.parametrize(
    "kw,status",
    [
        (dict(nsh=5), bnd.PA_ERR_INVALID),  # more sharers than sequences
        (dict(plen=1000), bnd.PA_ERR_INVALID),  # not a multiple of 64
        (dict(plen=4096), bnd.PA_ERR_INVALID),  # beyond max_context_len
        (dict(P=384), bnd.PA_ERR_INVALID),  # does not divide the prefix
        (dict(P=100), bnd.PA_ERR_INVALID),
        (dict(dt=bnd.PA_F32), bnd.PA_ERR_UNSUPPORTED),
        (dict(), bnd.PA_ERR_WORKSPACE),
        (dict(B=0, nsh=0), bnd.PA_OK),
    ],
)
def test_cascade_host_checks(kw, status):
    assert _cascade(**kw) == status


def test_cascade_workspace_covers_its_partition():
    # partition 0: the library's choice halved to divide the prefix; never below the split-K size
    n = pa.decode_cascade_workspace_size(128, 32, 128, 8192, 1024, 0, 8)
    assert n >= pa.decode_splitk_workspace_size(128, 32, 128, 8192, 0, 8)
    assert pa.decode_cascade_workspace_size(128, 32, 128, 8192, 1024, 384, 8) == 0


def test_bounded_wait_check_rejects_bad_limits():
    """pa_check_bounded_wait checks its bound before any launch (no GPU needed)."""
    assert bnd.lib.pa_check_bounded_wait(0, None) == bnd.PA_ERR_INVALID
    assert bnd.lib.pa_check_bounded_wait(2_000_000_000, None) == bnd.PA_ERR_INVALID


def _noalloc(**kw):
    a = dict(q=A, k=A, v=A, bt=A, cl=A, B=4, hq=32, hkv=8, d=128, bs=16, mb=4096, nb=1 << 14, out=A,
             dt=bnd.PA_BF16, P=0, maxL=2048, kern=0)
    a.update(kw)
    return bnd.lib.pa_decode_splitk_noalloc(a["q"], a["k"], a["v"], a["bt"], a["cl"], a["B"], a["hq"], a["hkv"],
                                            a["d"], a["bs"], a["mb"], a["nb"], 0.1, 0.0, 0, a["out"], a["dt"], a["P"],
                                            a["maxL"], a["kern"], None)


def test_noalloc_scratch_size_matches_the_header():
    src = open(HEADER).read()
    m = re.search(r"#define\s+PA_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", src)
    assert m, "PA_NOALLOC_SCRATCH_BYTES not found in the header"
    assert int(m.group(1)) << int(m.group(2)) == bnd.NOALLOC_SCRATCH_BYTES


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="fake pointers: CPU-only check")
def test_noalloc_refuses_exactly_above_its_scratch_and_checks_before_touching_the_device():
    """The refusal threshold is the header's size: the first context bound whose
    split-K workspace exceeds it is refused (PA_ERR_WORKSPACE) before anything
    else; the one below passes every host check and only then asks the runtime
    for the scratch, which on a machine without a GPU fails (PA_ERR_CUDA).  A
    call that fails a host check returns that check's status, so it touched
    neither the device nor the scratch."""
    B, hq, d, hkv = 4, 32, 128, 8
    L = 64
    while pa.decode_splitk_workspace_size(B, hq, d, L * 2, 0, hkv) <= bnd.NOALLOC_SCRATCH_BYTES:
        L *= 2
    lo, hi = L, L * 2  # need(lo) <= limit < need(hi): bisect to the first refused bound
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if pa.decode_splitk_workspace_size(B, hq, d, mid, 0, hkv) <= bnd.NOALLOC_SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid
    mb = (hi + 15) // 16
    assert _noalloc(maxL=hi, mb=mb) == bnd.PA_ERR_WORKSPACE
    assert _noalloc(maxL=lo, mb=mb) == bnd.PA_ERR_CUDA
    assert _noalloc(maxL=lo, mb=mb, q=None) == bnd.PA_ERR_INVALID
    assert _noalloc(maxL=lo, mb=mb, d=96) == bnd.PA_ERR_UNSUPPORTED
    assert _noalloc(maxL=2048, mb=128, P=100) == bnd.PA_ERR_INVALID  # not a multiple of 64


def test_importing_the_package_maps_no_gpu_code():
    """The package opens libpagedattn.so on first use, so a process that only
    draws inputs (the benchmark's CPU-oracle arm) maps none of it."""
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import sys; sys.path.insert(0, %r)\n"
            "import paged_kv_cache_473_b200, paged_kv_cache_473_b200.workloads\n"
            "maps = open('/proc/self/maps').read()\n"
            "print('mapped' if 'libpagedattn' in maps else 'clean')\n" % root)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "clean"
