"""Python binding of libbkv.so: the C ABI of include/bkv.h, one function per
entry point and with the same names.

Argument marshalling only: each function turns torch tensors into device
pointers and sizes, passes the current CUDA stream, and raises BkvError for a
non-zero status.  Every step of the compression runs in the library's CUDA
kernels; there is no fallback of any kind, and importing this module fails
loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# BKV_LIBRARY=debug loads the bounds-checked build (libbkv_debug.so), whose
# kernels report a data-dependent index out of range in the device status word
LIB_PATH = os.path.join(_HERE, "libbkv_debug.so" if os.environ.get("BKV_LIBRARY") == "debug"
                        else "libbkv.so")

BKV_F32, BKV_BF16 = 0, 1
AGGREGATE = {"max": 0, "mean": 1}   # bkv_aggregate
STATUS = {0: "BKV_OK", 1: "BKV_ERR_INVALID_ARG", 2: "BKV_ERR_UNSUPPORTED",
          3: "BKV_ERR_WORKSPACE", 4: "BKV_ERR_CUDA", 5: "BKV_ERR_TIMEOUT",
          6: "BKV_ERR_DEVICE_ASSERT"}
EXPORTS = ("bkv_workspace_size", "bkv_score", "bkv_select_topk", "bkv_compact",
           "bkv_update_beacons", "bkv_compress_step", "bkv_read_device_status",
           "bkv_status_string", "bkv_score_noalloc", "bkv_score_mean", "bkv_compact_inplace",
           "bkv_selftest_wait_timeout")
SCORE_NOALLOC_SCRATCH_BYTES = 32 << 20


class BkvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({_status_text(status)})")


class CacheDesc(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("capacity", ctypes.c_int64), ("dtype", ctypes.c_int32)]


class StepArgs(ctypes.Structure):
    _fields_ = [("cache", CacheDesc), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("L", ctypes.c_int64), ("K", ctypes.c_int64),
                ("recent_q", ctypes.c_void_p), ("R", ctypes.c_int32),
                ("beacons_in", ctypes.c_void_p), ("n_beacons_in", ctypes.c_int32),
                ("M", ctypes.c_int32), ("window", ctypes.c_void_p), ("W", ctypes.c_int32),
                ("beacons_out", ctypes.c_void_p), ("scale", ctypes.c_float),
                ("dst_cache", CacheDesc), ("k_dst", ctypes.c_void_p), ("v_dst", ctypes.c_void_p),
                ("scores_out", ctypes.c_void_p), ("idx_out", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("stream", ctypes.c_void_p),
                ("phase_events", ctypes.POINTER(ctypes.c_void_p)),
                ("aggregate", ctypes.c_int32),
                ("query_ring", ctypes.c_void_p), ("ring_cap", ctypes.c_int64),
                ("ring_pos", ctypes.c_int64), ("aux_stream", ctypes.c_void_p)]

STEP_EVENTS = 6


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with __graft_entry__.build() "
                          "(python -m kv_cache_compression_bkv_b200.build)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ, F = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                          ctypes.c_float)
    D = ctypes.POINTER(CacheDesc)
    sig = {
        "bkv_workspace_size": ([D, I64, I32, I32, I32, I64], SZ),
        "bkv_score": ([D, P, I64, P, I32, P, I32, I32, F, P, P, SZ, P], ctypes.c_int),
        "bkv_select_topk": ([P, I32, I64, I64, P, P, SZ, P], ctypes.c_int),
        "bkv_compact": ([D, P, P, P, I64, D, P, P, P], ctypes.c_int),
        "bkv_compact_inplace": ([D, P, P, P, I64, P], ctypes.c_int),
        "bkv_update_beacons": ([D, P, I32, I32, P, I32, P, ctypes.POINTER(I32), P, SZ, P],
                               ctypes.c_int),
        "bkv_compress_step": ([ctypes.POINTER(StepArgs), ctypes.POINTER(I32),
                               ctypes.POINTER(I64)], ctypes.c_int),
        "bkv_read_device_status": ([P, ctypes.POINTER(I32)], ctypes.c_int),
        "bkv_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "bkv_score_noalloc": ([D, P, I64, P, I32, P, I32, I32, F, P, P], ctypes.c_int),
        "bkv_score_mean": ([D, P, I64, P, I32, P, I32, I32, F, P, P, SZ, P], ctypes.c_int),
        "bkv_selftest_wait_timeout": ([I64, P, P], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


LIB = _load()


def _status_text(status: int) -> str:
    return LIB.bkv_status_string(status).decode()


def _check(status: int, where: str) -> None:
    if status != 0:
        raise BkvError(status, where)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return BKV_BF16
    if dt == torch.float32:
        return BKV_F32
    raise TypeError(f"unsupported dtype {dt}")


@dataclass(frozen=True)
class Geometry:
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    capacity: int
    dtype: torch.dtype

    def desc(self) -> CacheDesc:
        return CacheDesc(self.n_layers, self.n_q_heads, self.n_kv_heads, self.head_dim,
                         self.capacity, dtype_code(self.dtype))


def geometry_of(cache: torch.Tensor, n_q_heads: int) -> Geometry:
    """Geometry of a cache tensor [n_layers, n_kv_heads, capacity, head_dim]."""
    Ly, Hkv, cap, d = cache.shape
    return Geometry(Ly, n_q_heads, Hkv, d, cap, cache.dtype)


def bkv_workspace_size(geom: Geometry, L: int, R: int, M: int, W: int, K: int) -> int:
    d = geom.desc()
    return int(LIB.bkv_workspace_size(ctypes.byref(d), L, R, M, W, K))


def bkv_score(geom: Geometry, k, L: int, recent_q, R: int, beacons, n_beacons: int, M: int,
              scale: float, scores, workspace, stream=None) -> None:
    d = geom.desc()
    _check(LIB.bkv_score(ctypes.byref(d), _ptr(k), L, _ptr(recent_q), R, _ptr(beacons), n_beacons,
                         M, scale, _ptr(scores), _ptr(workspace),
                         0 if workspace is None else workspace.numel() * workspace.element_size(),
                         _stream(stream)), "bkv_score")


def bkv_score_mean(geom: Geometry, k, L: int, recent_q, R: int, beacons, n_beacons: int,
                   M: int, scale: float, scores, workspace, stream=None) -> None:
    """bkv_score with mean instead of max aggregation over the observation rows."""
    d = geom.desc()
    _check(LIB.bkv_score_mean(ctypes.byref(d), _ptr(k), L, _ptr(recent_q), R, _ptr(beacons),
                              n_beacons, M, scale, _ptr(scores), _ptr(workspace),
                              0 if workspace is None else workspace.numel() * workspace.element_size(),
                              _stream(stream)), "bkv_score_mean")


def bkv_score_noalloc(geom: Geometry, k, L: int, recent_q, R: int, beacons, n_beacons: int,
                      M: int, scale: float, scores, stream=None) -> None:
    """bkv_score on the library's built-in scratch array, for callers that
    cannot allocate device memory where they score (no workspace argument)."""
    d = geom.desc()
    _check(LIB.bkv_score_noalloc(ctypes.byref(d), _ptr(k), L, _ptr(recent_q), R, _ptr(beacons),
                                 n_beacons, M, scale, _ptr(scores), _stream(stream)),
           "bkv_score_noalloc")


def bkv_select_topk(scores, n_rows: int, L: int, K: int, idx, workspace=None,
                    stream=None) -> None:
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(LIB.bkv_select_topk(_ptr(scores), n_rows, L, K, _ptr(idx), _ptr(workspace), nbytes,
                               _stream(stream)), "bkv_select_topk")


def bkv_compact(src: Geometry, k_src, v_src, idx, n_keep: int, dst: Geometry, k_dst, v_dst,
                stream=None) -> None:
    ds, dd = src.desc(), dst.desc()
    _check(LIB.bkv_compact(ctypes.byref(ds), _ptr(k_src), _ptr(v_src), _ptr(idx), n_keep,
                           ctypes.byref(dd), _ptr(k_dst), _ptr(v_dst), _stream(stream)),
           "bkv_compact")


def bkv_compact_inplace(geom: Geometry, k, v, idx, n_keep: int, stream=None) -> None:
    """bkv_compact with the cache as source and destination (idx[r][i] >= i)."""
    d = geom.desc()
    _check(LIB.bkv_compact_inplace(ctypes.byref(d), _ptr(k), _ptr(v), _ptr(idx), n_keep,
                                   _stream(stream)), "bkv_compact_inplace")


def bkv_update_beacons(geom: Geometry, beacons_in, n_beacons_in: int, M: int, window, W: int,
                       beacons_out, workspace=None, stream=None) -> int:
    d = geom.desc()
    n_out = ctypes.c_int32(0)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(LIB.bkv_update_beacons(ctypes.byref(d), _ptr(beacons_in), n_beacons_in, M,
                                  _ptr(window), W, _ptr(beacons_out), ctypes.byref(n_out),
                                  _ptr(workspace), nbytes, _stream(stream)),
           "bkv_update_beacons")
    return n_out.value


def bkv_compress_step(geom: Geometry, k, v, L: int, K: int, recent_q, R: int, beacons_in,
                      n_beacons_in: int, M: int, window, W: int, beacons_out, scale: float,
                      dst: Geometry, k_dst, v_dst, scores_out=None, idx_out=None,
                      workspace=None, stream=None, phase_events=None,
                      aggregate: str = "max", query_ring=None, ring_pos: int = 0,
                      aux_stream=None) -> tuple[int, int]:
    """One whole compression step; returns (beacons valid after, new cache length).

    phase_events: optional list of STEP_EVENTS torch.cuda.Event (timing enabled)
    recorded at the step's phase boundaries.  aggregate: "max" or "mean".
    query_ring: optional decode-side ring [layers, q_heads, cap, d] holding query
    t in slot t % cap, with ring_pos queries written; recent_q and window must
    then be None (the recent rows and the window are the ring's newest R and W).
    aux_stream: optional second torch.cuda.Stream on which each head batch's
    top-K and compaction overlap the next batch's aggregation.
    """
    a = StepArgs()
    a.cache = geom.desc()
    a.k, a.v = _ptr(k), _ptr(v)
    a.L, a.K = L, K
    a.recent_q, a.R = _ptr(recent_q), R
    a.beacons_in, a.n_beacons_in, a.M = _ptr(beacons_in), n_beacons_in, M
    a.window, a.W = _ptr(window), W
    a.beacons_out = _ptr(beacons_out)
    a.scale = scale
    a.dst_cache = dst.desc()
    a.k_dst, a.v_dst = _ptr(k_dst), _ptr(v_dst)
    a.scores_out, a.idx_out = _ptr(scores_out), _ptr(idx_out)
    a.workspace = _ptr(workspace)
    a.workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    a.stream = _stream(stream)
    a.aggregate = AGGREGATE[aggregate]
    if aux_stream is not None:
        a.aux_stream = _stream(aux_stream)
    if query_ring is not None:
        a.query_ring = _ptr(query_ring)
        a.ring_cap = query_ring.shape[2]
        a.ring_pos = ring_pos
    if phase_events is not None:
        if len(phase_events) != STEP_EVENTS:
            raise ValueError(f"phase_events needs {STEP_EVENTS} events")
        arr = (ctypes.c_void_p * STEP_EVENTS)(*[ctypes.c_void_p(e.cuda_event) for e in phase_events])
        a.phase_events = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    nb = ctypes.c_int32(0)
    nl = ctypes.c_int64(0)
    _check(LIB.bkv_compress_step(ctypes.byref(a), ctypes.byref(nb), ctypes.byref(nl)),
           "bkv_compress_step")
    return nb.value, nl.value


def bkv_selftest_wait_timeout(limit_ns: int, outcome, stream=None) -> None:
    """Make one bounded device-side wait give up on purpose (diagnostic)."""
    _check(LIB.bkv_selftest_wait_timeout(limit_ns, _ptr(outcome), _stream(stream)),
           "bkv_selftest_wait_timeout")


def bkv_read_device_status(stream=None) -> tuple[int, int]:
    where = ctypes.c_int32(0)
    st = LIB.bkv_read_device_status(_stream(stream), ctypes.byref(where))
    return int(st), where.value
