"""Float64 CPU oracle for the BeaconKV compression step -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or executes anything here, and this
package imports nothing from the product package.

The arithmetic lives in ``bkv_oracle.c`` (plain loops, double precision); this
module compiles it with gcc on first use and marshals numpy arrays to it.  The
only logic written here is the assembly of the observation set of one KV head
(Fig. 5(b) of "BeaconKV: Key-Value Cache Compression Guided by Beacon Queries
for Efficient Large Reasoning Model Inference": beacon queries and recent
queries, for every query head of the GQA group) and the order in which the
steps are composed.

Inputs arrive as numpy arrays of any float dtype; they are converted to
float64, which is exact for bfloat16 and float32 values.

Pins (tests/oracle_pins.py): the C functions by closed forms, library
routines and brute force; the composition here (observation_set, score_head,
newest_rows, ring_rows, update_beacons_head, compress_head) by the
hand-derived whole step of tests/golden/closed_forms.json, brute-force greedy
FPS over the [beacons; window] union, and a history written into a ring one
row at a time.  tests/test_oracle_mutants.py plants plausible mistakes in
both and checks that each fails a pin.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libbkv_oracle.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)
_U8 = ctypes.POINTER(ctypes.c_uint8)
_i64 = ctypes.c_int64


def build(force: bool = False, extra_flags: tuple[str, ...] = (), out: str | None = None) -> str:
    """Compile bkv_oracle.c into a shared library and return its path."""
    out = out or _LIB_PATH
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
               *extra_flags, _SRC, "-o", out, "-lm"]
        subprocess.run(cmd, check=True)
    return out


def _bind(path: str):
    lib = ctypes.CDLL(path)
    lib.oracle_logits.argtypes = [_i64, _i64, _i64, _D, _D, ctypes.c_double, _D]
    lib.oracle_logits.restype = None
    lib.oracle_row_normalizer.argtypes = [_i64, _i64, _D, _D]
    lib.oracle_row_normalizer.restype = None
    lib.oracle_max_aggregate.argtypes = [_i64, _i64, _D, _D, _D]
    lib.oracle_max_aggregate.restype = None
    lib.oracle_mean_aggregate.argtypes = [_i64, _i64, _D, _D, _D]
    lib.oracle_mean_aggregate.restype = None
    lib.oracle_select_topk.argtypes = [_i64, _D, _i64, _I32]
    lib.oracle_select_topk.restype = _i64
    lib.oracle_compact.argtypes = [_i64, _U8, _I32, _i64, _U8]
    lib.oracle_compact.restype = None
    lib.oracle_fps.argtypes = [_i64, _i64, _D, _i64, _I32]
    lib.oracle_fps.restype = _i64
    lib.oracle_fps_replay.argtypes = [_i64, _i64, _D, _i64, _I32, ctypes.c_double, _D]
    lib.oracle_fps_replay.restype = _i64
    return lib


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def load_variant(path: str):
    """Bind an alternative build of the oracle (used by the mutation tests)."""
    return _bind(path)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray, ty):
    return a.ctypes.data_as(ty)


# --------------------------------------------------------------------------
# Step functions (one KV head each)
# --------------------------------------------------------------------------
def logits(q, k, scale: float, L=None, _lib=None):
    """x[o, j] = scale * q_o . k_j  for every observation row o and key j."""
    lb = _lib or lib()
    q, k = _f64(q), _f64(k)
    n_obs, d = q.shape
    L = k.shape[0] if L is None else L
    x = np.empty((n_obs, L), dtype=np.float64)
    lb.oracle_logits(n_obs, L, d, _ptr(q, _D), _ptr(k, _D), float(scale), _ptr(x, _D))
    return x


def row_normalizer(x, _lib=None):
    """c_o = log sum_j exp(x_oj), computed with the row max subtracted first."""
    lb = _lib or lib()
    x = _f64(x)
    n_obs, L = x.shape
    c = np.empty(n_obs, dtype=np.float64)
    lb.oracle_row_normalizer(n_obs, L, _ptr(x, _D), _ptr(c, _D))
    return c


def max_aggregate(x, c, _lib=None):
    """s_j = max_o exp(x_oj - c_o)."""
    lb = _lib or lib()
    x, c = _f64(x), _f64(c)
    n_obs, L = x.shape
    s = np.empty(L, dtype=np.float64)
    lb.oracle_max_aggregate(n_obs, L, _ptr(x, _D), _ptr(c, _D), _ptr(s, _D))
    return s


def mean_aggregate(x, c, _lib=None):
    """s_j = mean_o exp(x_oj - c_o)  (Table 2's Mean ablation)."""
    lb = _lib or lib()
    x, c = _f64(x), _f64(c)
    n_obs, L = x.shape
    s = np.empty(L, dtype=np.float64)
    lb.oracle_mean_aggregate(n_obs, L, _ptr(x, _D), _ptr(c, _D), _ptr(s, _D))
    return s


def select_topk(s, K: int, _lib=None):
    """Positions of the min(K, L) largest scores (ties: lower position), ascending."""
    lb = _lib or lib()
    s = _f64(s)
    L = s.shape[0]
    keep = max(0, min(K, L))
    idx = np.empty(max(keep, 1), dtype=np.int32)
    n = lb.oracle_select_topk(L, _ptr(s, _D), int(K), _ptr(idx, _I32))
    if n < 0:
        raise MemoryError("oracle_select_topk")
    return idx[:keep]


def compact(src_rows, idx, _lib=None):
    """Row gather as a byte copy: dst[i] = src[idx[i]] (any dtype, 2-D)."""
    lb = _lib or lib()
    src = np.ascontiguousarray(src_rows)
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    row_bytes = src.shape[1] * src.itemsize
    dst = np.empty((idx.shape[0],) + src.shape[1:], dtype=src.dtype)
    lb.oracle_compact(row_bytes, src.view(np.uint8).ctypes.data_as(_U8),
                      _ptr(idx, _I32), idx.shape[0], dst.view(np.uint8).ctypes.data_as(_U8))
    return dst


def fps(U, M: int, _lib=None):
    """Continual FPS selection (indices into U, in pick order) in cosine distance."""
    lb = _lib or lib()
    U = _f64(U)
    n, d = U.shape
    m = max(0, min(M, n))
    sel = np.empty(max(m, 1), dtype=np.int32)
    got = lb.oracle_fps(n, d, _ptr(U, _D), int(M), _ptr(sel, _I32))
    if got < 0:
        raise MemoryError("oracle_fps")
    return sel[:m]


def fps_replay(U, picks, tol: float, _lib=None):
    """Replay FPS on another implementation's picks; (first bad step or -1, max gap)."""
    lb = _lib or lib()
    U = _f64(U)
    picks = np.ascontiguousarray(np.asarray(picks, dtype=np.int32))
    n, d = U.shape
    gap = ctypes.c_double(0.0)
    bad = lb.oracle_fps_replay(n, d, _ptr(U, _D), picks.shape[0], _ptr(picks, _I32),
                               float(tol), ctypes.byref(gap))
    return int(bad), float(gap.value)


# --------------------------------------------------------------------------
# Composition for one (layer, KV head)
# --------------------------------------------------------------------------
def observation_set(recent, beacons, n_beacons: int):
    """Rows of the observation set of one KV head (Fig. 5(b)).

    recent: [G, R, d] -- the R most recent decode queries of each query head of
    the group; beacons: [G, M, d] of which the first ``n_beacons`` are valid.
    The rows are ordered (g, recent then beacons); the order does not change a
    max over rows.
    """
    recent = _f64(recent)
    beacons = _f64(beacons)
    G = recent.shape[0]
    parts = []
    for g in range(G):
        parts.append(recent[g])
        parts.append(beacons[g, :n_beacons])
    return np.concatenate(parts, axis=0)


def default_scale(d: int) -> float:
    return 1.0 / np.sqrt(float(d))


def newest_rows(rows, n: int):
    """The n newest rows of a query history listed oldest first ([..., T, d]).

    The recent queries of Fig. 5(a)/(b) are the R newest decode queries; with
    the window of Fig. 7 listed oldest first they are its last R rows.
    """
    rows = np.asarray(rows)
    T = rows.shape[-2]
    return rows[..., T - n:T, :]


def ring_rows(ring, head: int, n: int):
    """The n newest rows, oldest first, of a ring buffer [..., cap, d] whose
    next write goes to slot ``head`` (so the newest row sits at head - 1)."""
    ring = np.asarray(ring)
    cap = ring.shape[-2]
    idx = [(head - n + i) % cap for i in range(n)]
    return ring[..., idx, :]


def score_head(k, recent, beacons, n_beacons: int, scale: float | None = None,
               aggregate: str = "max", _lib=None):
    """Scores s_j of every cached key of one KV head, and the row normalisers c_o."""
    k = _f64(k)
    scale = default_scale(k.shape[1]) if not scale else scale
    q = observation_set(recent, beacons, n_beacons)
    x = logits(q, k, scale, _lib=_lib)
    c = row_normalizer(x, _lib=_lib)
    if aggregate == "max":
        s = max_aggregate(x, c, _lib=_lib)
    elif aggregate == "mean":
        s = mean_aggregate(x, c, _lib=_lib)
    else:
        raise ValueError(aggregate)
    return s, c


def update_beacons_head(beacons, n_beacons: int, window, M: int, _lib=None):
    """Continual FPS for one query head: new beacons from beacons[:n] and the window.

    Returns (new_beacons [m, d] raw vectors in pick order, picks into the union).
    """
    b = np.asarray(beacons)[:n_beacons]
    w = np.asarray(window)
    U = np.concatenate([b, w], axis=0) if w.size else b
    sel = fps(U, M, _lib=_lib)
    return U[sel], sel


def compress_head(k_rows, v_rows, recent, beacons, n_beacons: int, window, M: int,
                  K: int, scale: float | None = None, aggregate: str = "max", _lib=None):
    """The whole step for one (layer, KV head).

    Order (a reading: the pages only show the beacons being used for scoring):
    Continual FPS over beacons and window for each query head of the group,
    then scoring with the updated beacons, top-K and compaction.
    k_rows, v_rows: [L, d] (any dtype; compaction copies their bytes).
    recent: [G, R, d]; beacons: [G, M, d] (first n_beacons valid);
    window: [G, W, d] or None.  aggregate: "max" (the method) or "mean"
    (Table 2's ablation).
    """
    G = np.asarray(recent).shape[0]
    if window is not None and np.asarray(window).shape[1] > 0:
        new_b, picks = [], []
        for g in range(G):
            nb, sel = update_beacons_head(beacons[g], n_beacons, window[g], M, _lib=_lib)
            new_b.append(nb)
            picks.append(sel)
        beacons_used = np.stack(new_b)
        n_used = beacons_used.shape[1]
    else:
        beacons_used, n_used, picks = np.asarray(beacons), n_beacons, None
    s, c = score_head(k_rows, recent, beacons_used, n_used, scale, aggregate=aggregate,
                      _lib=_lib)
    idx = select_topk(s, K, _lib=_lib)
    return {
        "beacons": beacons_used, "n_beacons": n_used, "picks": picks,
        "scores": s, "c": c, "idx": idx,
        "k": compact(np.asarray(k_rows), idx, _lib=_lib),
        "v": compact(np.asarray(v_rows), idx, _lib=_lib),
    }
