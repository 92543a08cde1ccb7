"""Seeded synthetic inputs for the BeaconKV compression step.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no scores, softmax, selection or sampling), so both the
CUDA path and the float64 oracle can take their inputs from it.

The workloads stand in for the reasoning models that "BeaconKV: Key-Value Cache
Compression Guided by Beacon Queries for Efficient Large Reasoning Model
Inference" evaluates (R1-Distill-Qwen-7B, R1-Distill-Llama-8B, Qwen3-4B,
Qwen3-14B; Fig. 8) with the GQA shapes of those models and the trace lengths of
Tables 4 and 6.  No weights or datasets are used: the structure the page
reports (queries that fall into a few cosine-similarity clusters, Fig. 4, and
early "plan" keys that later queries revisit, Figs. 1, 2 and 9) is planted by
construction.

Every (layer, KV head) is generated from its own seed, so a test can rebuild
any single head on the CPU without generating the whole cache.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    L: int                 # valid cache rows per (layer, KV head) at the step
    R: int                 # recent queries per query head
    M: int                 # beacon slots per query head
    K: int                 # budget: rows kept per (layer, KV head)
    W: int                 # window of newest queries fed to Continual FPS (0: none)
    dtype: str             # "f32" or "bf16"
    n_clusters: int        # query clusters per query head
    q_noise: float         # per-component std of the query noise
    n_plan: int            # planted plan keys per (layer, KV head)
    plan_span: int         # plan keys sit at positions [0, plan_span)
    n_outlier_channels: int = 0
    outlier_scale: float = 10.0
    big_key_frac: float = 0.0
    big_key_norm: float = 40.0
    n_beacons_in: int = -1  # valid beacons in the input (-1: all M)
    capacity: int = -1      # allocated rows per head (-1: L)
    q_centroid_scale: float = 8.0
    plan_key_scale: float = 6.0

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def cap(self) -> int:
        return self.L if self.capacity < 0 else self.capacity

    @property
    def beacons_in(self) -> int:
        return self.M if self.n_beacons_in < 0 else self.n_beacons_in

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def n_heads(self) -> int:
        """(layer, KV head) pairs."""
        return self.n_layers * self.n_kv_heads

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads.  Readings where the description is brief: "drift noise
# 0.5" is a per-component std of 0.5; the window fed to Continual FPS holds the
# 4096 queries of one compression interval; the recent queries are the newest R
# queries of that window; the input beacons are earlier queries of the same
# clusters.
WORKLOADS: dict[str, Workload] = {
    "tiny": Workload(
        name="tiny", n_layers=1, n_q_heads=4, n_kv_heads=1, head_dim=64, L=1024,
        R=32, M=16, K=256, W=1024, dtype="f32", n_clusters=4, q_noise=1.0,
        n_plan=32, plan_span=128),
    "r1_qwen7b": Workload(
        name="r1_qwen7b", n_layers=28, n_q_heads=28, n_kv_heads=4, head_dim=128,
        L=8192, R=32, M=64, K=2048, W=4096, dtype="bf16", n_clusters=8,
        q_noise=0.5, n_plan=8192 * 5 // 100, plan_span=8192 * 5 // 100,
        n_outlier_channels=4),
    "llama8b": Workload(
        name="llama8b", n_layers=32, n_q_heads=32, n_kv_heads=8, head_dim=128,
        L=16384, R=64, M=64, K=4096, W=4096, dtype="bf16", n_clusters=12,
        q_noise=0.5, n_plan=16384 * 5 // 100, plan_span=16384 * 5 // 100,
        n_outlier_channels=4),
    # One evicting step of the Qwen3-4B-shaped continual decoding trace: the
    # cache holds two compression intervals (8192 rows) and is cut to 4096.
    "qwen3_4b_step": Workload(
        name="qwen3_4b_step", n_layers=36, n_q_heads=32, n_kv_heads=8,
        head_dim=128, L=8192, R=16, M=64, K=4096, W=4096, dtype="bf16",
        n_clusters=8, q_noise=0.5, n_plan=1024, plan_span=1024,
        n_outlier_channels=4),
    "qwen3_14b": Workload(
        name="qwen3_14b", n_layers=40, n_q_heads=40, n_kv_heads=8, head_dim=128,
        L=32768, R=64, M=128, K=6144, W=4096, dtype="bf16", n_clusters=16,
        q_noise=0.5, n_plan=64, plan_span=2048, n_outlier_channels=4,
        big_key_frac=0.01, big_key_norm=40.0),
}


def _gen(seed: int, layer: int, head: int, stream: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed((seed * 1_000_003 + layer * 10_007 + head * 101 + stream) % (2**63 - 1))
    return g


def _unit_rows(n: int, d: int, g: torch.Generator) -> torch.Tensor:
    x = torch.randn(n, d, generator=g, dtype=torch.float32)
    return x / x.norm(dim=1, keepdim=True)


def centroids(wl: Workload, seed: int, layer: int, q_head: int) -> torch.Tensor:
    """Unit cluster centroids of one query head: [n_clusters, d]."""
    return _unit_rows(wl.n_clusters, wl.head_dim, _gen(seed, layer, q_head, 1))


def queries(wl: Workload, seed: int, layer: int, q_head: int, n: int, stream: int) -> torch.Tensor:
    """n queries of one query head: centroid_scale * c + noise, c drawn uniformly."""
    cen = centroids(wl, seed, layer, q_head)
    g = _gen(seed, layer, q_head, stream)
    which = torch.randint(0, wl.n_clusters, (n,), generator=g)
    noise = torch.randn(n, wl.head_dim, generator=g, dtype=torch.float32)
    return wl.q_centroid_scale * cen[which] + wl.q_noise * noise


def keys_values(wl: Workload, seed: int, layer: int, kv_head: int):
    """Keys and values of one (layer, KV head): two float32 [L, d] tensors."""
    d, L, G = wl.head_dim, wl.L, wl.group
    g = _gen(seed, layer, kv_head, 2)
    k = torch.randn(L, d, generator=g, dtype=torch.float32)
    v = torch.randn(L, d, generator=g, dtype=torch.float32)
    if wl.n_plan > 0:
        span = min(wl.plan_span, L)
        n_plan = min(wl.n_plan, span)
        pos = torch.randperm(span, generator=g)[:n_plan] if n_plan < span else torch.arange(span)
        cen = torch.cat([centroids(wl, seed, layer, kv_head * G + gg) for gg in range(G)])
        which = torch.randint(0, cen.shape[0], (n_plan,), generator=g)
        k[pos] = wl.plan_key_scale * cen[which] + torch.randn(n_plan, d, generator=g)
    if wl.n_outlier_channels > 0:
        ch = torch.randperm(d, generator=g)[:wl.n_outlier_channels]
        k[:, ch] *= wl.outlier_scale
    if wl.big_key_frac > 0:
        n_big = max(1, int(round(wl.big_key_frac * L)))
        pos = torch.randperm(L, generator=g)[:n_big]
        k[pos] = k[pos] / k[pos].norm(dim=1, keepdim=True) * wl.big_key_norm
    return k, v


def head_queries(wl: Workload, seed: int, layer: int, q_head: int):
    """(recent [R, d], beacons [M, d], window [W, d]) of one query head, float32.

    The window lists the newest W queries oldest first; the recent queries are
    its last R rows (or separate draws when there is no window).  Beacon slots
    past ``beacons_in`` hold zeros.
    """
    d = wl.head_dim
    window = queries(wl, seed, layer, q_head, wl.W, 3) if wl.W > 0 else torch.zeros(0, d)
    if wl.W >= wl.R:
        recent = window[wl.W - wl.R:].clone()
    else:
        recent = queries(wl, seed, layer, q_head, wl.R, 4)
    beacons = torch.zeros(wl.M, d)
    nb = wl.beacons_in
    if nb > 0:
        beacons[:nb] = queries(wl, seed, layer, q_head, nb, 5)
    return recent, beacons, window


@dataclass
class StepInputs:
    """Host tensors of one compression step, in the library's layouts.

    k, v:          [layers, kv_heads, capacity, d]
    recent:        [layers, q_heads, R, d]
    beacons:       [layers, q_heads, M, d]   (first n_beacons valid)
    window:        [layers, q_heads, W, d]
    """
    wl: Workload
    seed: int
    k: torch.Tensor
    v: torch.Tensor
    recent: torch.Tensor
    beacons: torch.Tensor
    window: torch.Tensor


def make_step_inputs(wl: Workload, seed: int = 0, pin: bool = False,
                     poison_tail: float | None = 100.0) -> StepInputs:
    """All inputs of one step.  Rows past L (capacity > L) hold ``poison_tail``."""
    dt = wl.torch_dtype
    Ly, Hq, Hkv, d = wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim

    def alloc(*shape):
        t = torch.empty(*shape, dtype=dt)
        return t.pin_memory() if pin else t

    k = alloc(Ly, Hkv, wl.cap, d)
    v = alloc(Ly, Hkv, wl.cap, d)
    recent = alloc(Ly, Hq, wl.R, d)
    beacons = alloc(Ly, Hq, wl.M, d)
    window = alloc(Ly, Hq, wl.W, d)
    for l in range(Ly):
        for h in range(Hkv):
            kk, vv = keys_values(wl, seed, l, h)
            k[l, h, :wl.L] = kk.to(dt)
            v[l, h, :wl.L] = vv.to(dt)
            if wl.cap > wl.L:
                fill = 0.0 if poison_tail is None else poison_tail
                k[l, h, wl.L:] = fill
                v[l, h, wl.L:] = fill
        for qh in range(Hq):
            r, b, w = head_queries(wl, seed, l, qh)
            recent[l, qh] = r.to(dt)
            beacons[l, qh] = b.to(dt)
            if wl.W > 0:
                window[l, qh] = w.to(dt)
    return StepInputs(wl, seed, k, v, recent, beacons, window)


def head_slice(inp: StepInputs, layer: int, kv_head: int):
    """Views of one (layer, KV head): k, v [L, d]; recent, beacons, window [G, *, d]."""
    wl = inp.wl
    G = wl.group
    q0 = kv_head * G
    return (inp.k[layer, kv_head, :wl.L], inp.v[layer, kv_head, :wl.L],
            inp.recent[layer, q0:q0 + G], inp.beacons[layer, q0:q0 + G],
            inp.window[layer, q0:q0 + G])


# --------------------------------------------------------------------------
# Continual decoding trace (Qwen3-4B-shaped): queries from slowly drifting
# clusters, a share of steps re-aiming at fixed early "plan" centroids, and
# plan keys in the first steps.
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class Trace:
    name: str
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    steps: int
    interval: int
    K: int
    R: int
    M: int
    n_clusters: int = 8
    n_plan_centroids: int = 4
    revisit_prob: float = 0.10
    drift_per_step: float = 0.01   # norm of the centroid perturbation per step
    drift_block: int = 64          # the drift is drawn once per block of steps
    plan_steps: int = 1024
    q_noise: float = 0.5
    q_centroid_scale: float = 8.0
    plan_key_scale: float = 6.0
    n_outlier_channels: int = 4
    outlier_scale: float = 10.0
    dtype: str = "bf16"

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def replace(self, **kw) -> "Trace":
        return dataclasses.replace(self, **kw)


TRACES: dict[str, Trace] = {
    "qwen3_4b_trace": Trace(name="qwen3_4b_trace", n_layers=36, n_q_heads=32,
                            n_kv_heads=8, head_dim=128, steps=32768, interval=4096,
                            K=4096, R=16, M=64),
}


def trace_plan_centroids(tr: Trace, seed: int, layer: int, q_head: int) -> torch.Tensor:
    return _unit_rows(tr.n_plan_centroids, tr.head_dim, _gen(seed, layer, q_head, 11))


def trace_queries(tr: Trace, seed: int, layer: int, q_head: int) -> torch.Tensor:
    """All ``steps`` queries of one query head, float32 [steps, d]."""
    d, T = tr.head_dim, tr.steps
    g = _gen(seed, layer, q_head, 12)
    c0 = _unit_rows(tr.n_clusters, d, g)
    n_blocks = (T + tr.drift_block - 1) // tr.drift_block
    step_std = tr.drift_per_step / math.sqrt(d) * math.sqrt(tr.drift_block)
    walk = torch.cumsum(torch.randn(n_blocks, tr.n_clusters, d, generator=g) * step_std, dim=0)
    cen = c0.unsqueeze(0) + walk                      # [blocks, clusters, d]
    cen = cen / cen.norm(dim=2, keepdim=True)
    plan = trace_plan_centroids(tr, seed, layer, q_head)
    which = torch.randint(0, tr.n_clusters, (T,), generator=g)
    revisit = torch.rand(T, generator=g) < tr.revisit_prob
    which_plan = torch.randint(0, tr.n_plan_centroids, (T,), generator=g)
    blk = torch.arange(T) // tr.drift_block
    base = cen[blk, which]
    base[revisit] = plan[which_plan[revisit]]
    noise = torch.randn(T, d, generator=g)
    return tr.q_centroid_scale * base + tr.q_noise * noise


def trace_keys_values(tr: Trace, seed: int, layer: int, kv_head: int):
    """All ``steps`` keys and values of one (layer, KV head), float32 [steps, d]."""
    d, T, G = tr.head_dim, tr.steps, tr.group
    g = _gen(seed, layer, kv_head, 13)
    k = torch.randn(T, d, generator=g)
    v = torch.randn(T, d, generator=g)
    n_plan = min(tr.plan_steps, T)
    plan = torch.cat([trace_plan_centroids(tr, seed, layer, kv_head * G + gg) for gg in range(G)])
    which = torch.randint(0, plan.shape[0], (n_plan,), generator=g)
    k[:n_plan] = tr.plan_key_scale * plan[which] + torch.randn(n_plan, d, generator=g)
    if tr.n_outlier_channels > 0:
        ch = torch.randperm(d, generator=g)[:tr.n_outlier_channels]
        k[:, ch] *= tr.outlier_scale
    return k, v
