"""The C ABI on the host: the library loads, exports every declared entry point,
and rejects bad arguments before anything is launched (no GPU needed).

Every call below fails a host-side check, so no CUDA call is made; the pointers
are fake addresses that are never dereferenced.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bkv.h")

bkv = pytest.importorskip("kv_cache_compression_bkv_b200.bkv")
LIB = bkv.LIB

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
A = 0x10000          # a 16-byte aligned fake device address
S = 0                # default stream; never touched by rejected calls


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bkv_\w+)\s*\(", text)))


def test_exports_every_declared_function():
    names = declared_functions()
    assert "bkv_compress_step" in names and len(names) >= 8
    for name in names:
        assert hasattr(LIB, name), name
    assert set(bkv.EXPORTS) >= set(names) - set(), (set(names) - set(bkv.EXPORTS))


def test_debug_library_exports_every_declared_function():
    """libbkv_debug.so (the bounds-checked build) has the same ABI."""
    path = os.path.join(os.path.dirname(bkv.__file__), "libbkv_debug.so")
    if not os.path.exists(path):
        pytest.skip("libbkv_debug.so is not built")
    dbg = ctypes.CDLL(path)
    for name in declared_functions():
        assert hasattr(dbg, name), name


def test_status_strings():
    for code in range(7):
        assert LIB.bkv_status_string(code)
    assert LIB.bkv_status_string(99) == b"unknown status"


def desc(Ly=2, Hq=8, Hkv=2, d=128, cap=1024, dt=bkv.BKV_BF16):
    return bkv.CacheDesc(Ly, Hq, Hkv, d, cap, dt)


def score(d, k=A, L=1000, recent=A, R=8, beacons=A, nb=16, M=16, scale=0.0, scores=A, ws=A,
          ws_bytes=1 << 40, fn="bkv_score"):
    return getattr(LIB, fn)(ctypes.byref(d) if d is not None else None, k, L, recent, R, beacons,
                            nb, M, scale, scores, ws, ws_bytes, S)


def test_workspace_size():
    d = desc()
    n = LIB.bkv_workspace_size(ctypes.byref(d), 1000, 8, 16, 64, 300)
    # at least c, one aggregation partial and the kept indices of every head
    assert n >= 2 * 2 * (1000 * 4 + 300 * 4)
    assert LIB.bkv_workspace_size(ctypes.byref(d), 0, 8, 16, 64, 300) == 0
    assert LIB.bkv_workspace_size(ctypes.byref(desc(Hq=7)), 1000, 8, 16, 64, 300) == 0
    assert LIB.bkv_workspace_size(None, 1000, 8, 16, 64, 300) == 0


@pytest.mark.parametrize("kw,expect", [
    (dict(d=None), INVALID),
    (dict(d=desc(Hq=7)), INVALID),            # q heads not a multiple of kv heads
    (dict(d=desc(cap=0)), INVALID),
    (dict(d=desc(d=60)), INVALID),            # row not a multiple of 16 bytes
    (dict(d=desc(dt=5)), INVALID),
    (dict(L=0), INVALID),
    (dict(L=1025), INVALID),                  # beyond capacity
    (dict(nb=17), INVALID),                   # more beacons than slots
    (dict(R=0, nb=0), INVALID),               # empty observation set
    (dict(k=0), INVALID),
    (dict(k=A + 8), INVALID),                 # misaligned
    (dict(recent=0), INVALID),
    (dict(beacons=0), INVALID),
    (dict(scores=0), INVALID),
    (dict(scale=-1.0), INVALID),
    (dict(scale=float("nan")), INVALID),
    (dict(d=desc(d=64)), UNSUPPORTED),        # bf16 tensor-core path is head_dim 128
    (dict(d=desc(d=256, dt=bkv.BKV_F32)), UNSUPPORTED),
    (dict(ws=0), WORKSPACE),
    (dict(ws_bytes=1024), WORKSPACE),
])
@pytest.mark.parametrize("fn", ["bkv_score", "bkv_score_mean"])
def test_score_rejects(kw, expect, fn):
    args = dict(d=desc(), fn=fn)
    args.update(kw)
    assert score(**args) == expect


def test_select_rejects():
    f = LIB.bkv_select_topk
    assert f(None, 4, 100, 10, A, None, 0, S) == INVALID
    assert f(A, 0, 100, 10, A, None, 0, S) == INVALID
    assert f(A, 4, 0, 10, A, None, 0, S) == INVALID
    assert f(A, 4, 100, 0, A, None, 0, S) == INVALID
    assert f(A, 4, 100, 10, None, None, 0, S) == INVALID
    assert f(A + 4, 4, 100, 10, A, None, 0, S) == INVALID
    # rows of any length need no workspace (the select streams them)
    d = desc()
    assert LIB.bkv_workspace_size(ctypes.byref(d), 1 << 20, 8, 16, 0, 10) > 0


def test_compact_rejects():
    f = LIB.bkv_compact
    src, dst = desc(cap=1024), desc(cap=256)
    big = 1 << 30
    ok_args = [ctypes.byref(src), A, A + big, A + 2 * big, 256, ctypes.byref(dst), A + 3 * big,
               A + 4 * big, S]

    def call(**kw):
        a = list(ok_args)
        names = ["src", "k_src", "v_src", "idx", "n", "dst", "k_dst", "v_dst", "s"]
        for key, val in kw.items():
            a[names.index(key)] = val
        return f(*a)

    assert call(n=257) == INVALID                       # beyond dst capacity
    assert call(n=-1) == INVALID
    assert call(idx=0) == INVALID
    assert call(k_dst=0) == INVALID                     # pair half missing
    assert call(k_dst=A + 64) == INVALID                # overlaps k_src
    assert call(v_dst=A + big + 1024) == INVALID        # overlaps v_src
    assert call(k_dst=A + 3 * big + 8) == INVALID       # misaligned
    assert call(dst=ctypes.byref(desc(cap=256, d=64))) == INVALID
    assert call(dst=ctypes.byref(desc(cap=256, dt=bkv.BKV_F32))) == INVALID


def test_compact_inplace_rejects():
    f = LIB.bkv_compact_inplace
    d = desc(cap=1024)
    big = 1 << 30
    assert f(ctypes.byref(d), A, A + big, A + 2 * big, 1025, S) == INVALID  # beyond capacity
    assert f(ctypes.byref(d), A, A + big, A + 2 * big, -1, S) == INVALID
    assert f(ctypes.byref(d), None, A + big, A + 2 * big, 10, S) == INVALID
    assert f(ctypes.byref(d), A, A + big, None, 10, S) == INVALID
    assert f(ctypes.byref(d), A + 8, A + big, A + 2 * big, 10, S) == INVALID  # misaligned
    assert f(ctypes.byref(d), A, A + big, A + 2 * big + 2, 10, S) == INVALID
    assert f(ctypes.byref(d), A, A + 64, A + 2 * big, 10, S) == INVALID   # K and V overlap
    assert f(None, A, A + big, A + 2 * big, 10, S) == INVALID


def test_update_beacons_rejects():
    f = LIB.bkv_update_beacons
    d = desc()
    n = ctypes.c_int32(-7)
    big = 1 << 30
    base = [ctypes.byref(d), A, 16, 16, A + big, 64, A + 2 * big, ctypes.byref(n), None, 0, S]

    def call(**kw):
        a = list(base)
        names = ["d", "bin", "nb", "M", "win", "W", "bout", "nout", "ws", "wsb", "s"]
        for key, val in kw.items():
            a[names.index(key)] = val
        return f(*a)

    assert call(M=0) == INVALID
    assert call(nb=17) == INVALID
    assert call(nb=0, W=0) == INVALID
    assert call(win=0) == INVALID
    assert call(bout=0) == INVALID
    assert call(bout=A + 64) == INVALID                 # overlaps beacons_in
    assert call(bout=A + big + 128) == INVALID          # overlaps window
    # a bf16 union this large keeps its distances in the workspace
    assert call(W=100000) == WORKSPACE
    # the f32 kernel keeps them in shared memory only
    assert call(d=ctypes.byref(desc(dt=bkv.BKV_F32)), W=100000) == UNSUPPORTED
    assert n.value == -7                                # outputs untouched


def step_args(**kw):
    a = bkv.StepArgs()
    big = 1 << 32
    a.cache = desc(cap=1024)
    a.k, a.v, a.L, a.K = A, A + big, 1000, 300
    a.recent_q, a.R = A + 2 * big, 8
    a.beacons_in, a.n_beacons_in, a.M = A + 3 * big, 16, 16
    a.window, a.W, a.beacons_out = A + 4 * big, 64, A + 5 * big
    a.scale = 0.0
    a.dst_cache = desc(cap=512)
    a.k_dst, a.v_dst = A + 6 * big, A + 7 * big
    a.scores_out, a.idx_out = None, None
    a.workspace, a.workspace_bytes = A + 8 * big, 1 << 31
    a.stream = None
    for key, val in kw.items():
        setattr(a, key, val)
    return a


@pytest.mark.parametrize("kw,expect", [
    (dict(K=0), INVALID),
    (dict(dst_cache=desc(cap=299)), INVALID),      # too small for the kept rows
    (dict(dst_cache=desc(cap=512, d=64)), INVALID),
    (dict(v=None), INVALID),
    (dict(k_dst=None), INVALID),
    (dict(beacons_out=None), INVALID),             # needed when a window is given
    (dict(k_dst=(1 << 32) + A + 64), INVALID),     # overlaps v
    (dict(beacons_out=A + 3 * (1 << 32)), INVALID),  # overlaps beacons_in
    (dict(idx_out=A + 2), INVALID),                # misaligned
    (dict(workspace_bytes=4096), WORKSPACE),
    (dict(workspace=None), WORKSPACE),
    (dict(W=100000, cache=desc(cap=1024, dt=bkv.BKV_F32),
          dst_cache=desc(cap=512, dt=bkv.BKV_F32)), UNSUPPORTED),  # f32 union too large
    (dict(W=100000, workspace_bytes=1 << 20), WORKSPACE),  # bf16: needs workspace slices
    (dict(aggregate=2), INVALID),                  # neither max nor mean
    (dict(aggregate=-1), INVALID),
])
def test_compress_step_rejects(kw, expect):
    a = step_args(**kw)
    nb, nl = ctypes.c_int32(-5), ctypes.c_int64(-5)
    assert LIB.bkv_compress_step(ctypes.byref(a), ctypes.byref(nb), ctypes.byref(nl)) == expect
    assert nb.value == -5 and nl.value == -5


def test_compress_step_null():
    assert LIB.bkv_compress_step(None, None, None) == INVALID


def test_step_args_layout_matches_the_header(tmp_path):
    """The binding's StepArgs has the C struct's size and field offsets (gcc
    compiles a probe against include/bkv.h on the host)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    fields = [f[0] for f in bkv.StepArgs._fields_]
    src = tmp_path / "layout.c"
    body = "".join(f'  printf("%zu\\n", offsetof(bkv_step_args, {f}));\n' for f in fields)
    src.write_text("#include <stddef.h>\n#include <stdio.h>\n#include \"bkv.h\"\n"
                   "int main(void) {\n  printf(\"%zu\\n\", sizeof(bkv_step_args));\n"
                   + body + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True,
                                          check=True).stdout.split()]
    assert got[0] == ctypes.sizeof(bkv.StepArgs)
    assert got[1:] == [getattr(bkv.StepArgs, f).offset for f in fields]


INJECT_SCRIPT = r"""
import ctypes, sys
import numpy as np
sys.path.insert(0, {root!r})
from kv_cache_compression_bkv_b200 import bkv
LIB = bkv.LIB
CUDA = 4
# host buffers stand in for device ones: with the injected failure no launch
# (and no access) happens, on a machine with or without a GPU
cap, keep, d = 64, 16, 128
src = np.arange(2 * 2 * cap * d, dtype=np.uint16).reshape(2, 2, cap, d)
dst = np.full((2, 2, keep, d), 7, dtype=np.uint16)
idx = np.tile(np.arange(keep, dtype=np.int32) * 2, (4, 1))
g = bkv.CacheDesc(2, 4, 2, d, cap, bkv.BKV_BF16)
gd = bkv.CacheDesc(2, 4, 2, d, keep, bkv.BKV_BF16)
p = lambda a: ctypes.c_void_p(a.ctypes.data)
before = dst.copy()
st = LIB.bkv_compact(ctypes.byref(g), p(src), None, p(idx), keep, ctypes.byref(gd), p(dst), None, None)
assert st == CUDA, st
assert np.array_equal(dst, before)
scores = np.full((4, cap), 3.0, dtype=np.float32)
out_idx = np.full((4, keep), -5, dtype=np.int32)
st = LIB.bkv_select_topk(p(scores), 4, cap, keep, p(out_idx), None, 0, None)
assert st == CUDA, st
assert (out_idx == -5).all()
outcome = np.full(1, 9, dtype=np.int32)
assert LIB.bkv_selftest_wait_timeout(1000000, p(outcome), None) == CUDA
assert outcome[0] == 9
print("injected launch failures reported")
"""


def test_injected_launch_failure_is_reported_and_outputs_untouched(tmp_path):
    """BKV_INJECT_LAUNCH_FAILURE makes every kernel launch fail before it is
    enqueued: the entry points return BKV_ERR_CUDA and leave their outputs as
    they were (run in a fresh process, since the flag is read once)."""
    import subprocess
    import sys
    script = tmp_path / "inject.py"
    script.write_text(INJECT_SCRIPT.format(root=ROOT))
    env = dict(os.environ, BKV_INJECT_LAUNCH_FAILURE="1")
    r = subprocess.run([sys.executable, str(script)], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "injected launch failures reported" in r.stdout


def test_selftest_rejects_bad_arguments():
    assert LIB.bkv_selftest_wait_timeout(10, A, S) == INVALID          # limit too short
    assert LIB.bkv_selftest_wait_timeout(10**9, A, S) == INVALID       # limit too long
    assert LIB.bkv_selftest_wait_timeout(10**6, 0, S) == INVALID       # no outcome
    assert LIB.bkv_selftest_wait_timeout(10**6, A + 2, S) == INVALID   # misaligned


def test_compress_step_rejects_bad_rings():
    """A decode-side query ring replaces recent_q and window; its sizes are
    checked before anything is launched."""
    def args(**kw):
        a = bkv.StepArgs()
        a.cache = desc()
        a.k = a.v = A
        a.L, a.K = 1000, 100
        a.R, a.M, a.W = 8, 16, 64
        a.beacons_in, a.n_beacons_in = A + 0x100000, 16
        a.beacons_out = A + 0x200000
        a.dst_cache = desc(cap=100)
        a.k_dst, a.v_dst = A + 0x400000, A + 0x800000
        a.workspace, a.workspace_bytes = A + 0x1000000, 1 << 40
        a.query_ring, a.ring_cap, a.ring_pos = A + 0x2000000, 128, 500
        for k, v in kw.items():
            setattr(a, k, v)
        return a

    def call(a):
        return LIB.bkv_compress_step(ctypes.byref(a), None, None)

    assert call(args(recent_q=A)) == INVALID            # the ring replaces recent_q
    assert call(args(window=A)) == INVALID              # ... and the window
    assert call(args(ring_cap=0)) == INVALID
    assert call(args(ring_cap=32)) == INVALID           # W > ring_cap
    assert call(args(ring_pos=40)) == INVALID           # fewer queries written than W
    assert call(args(query_ring=A + 0x2000008)) == INVALID  # misaligned
    # the updated beacons must not overlap the ring
    assert call(args(beacons_out=A + 0x2000000 + 256)) == INVALID
