"""CUDA path against the float64 oracle, element by element, through the C ABI.

Small cases cover every head of several tiles with ragged tails and the
degenerate shapes; the full-size workloads run the same launch configuration
as bench.py and compare seeded samples of heads.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
from parity_helpers import (check_compaction, check_fps, check_scores, check_topk, f64,
                            picks_from_rows, raw)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch.device("cuda:0")


def _lib():
    from kv_cache_compression_bkv_b200 import bkv
    return bkv


def _synth():
    from kv_cache_compression_bkv_b200 import synth
    return synth


def small(**kw):
    base = dict(name="case", n_layers=1, n_q_heads=4, n_kv_heads=2, head_dim=128, L=1000,
                R=8, M=16, K=300, W=0, dtype="bf16", n_clusters=4, q_noise=0.5, n_plan=16,
                plan_span=64, n_outlier_channels=2, n_beacons_in=12)
    base.update(kw)
    base.setdefault("capacity", base["L"] + 100)  # poisoned rows past L
    return _synth().Workload(**base)


SCORE_CASES = {
    "tiny_f32": lambda: _synth().WORKLOADS["tiny"].replace(W=0),
    "ragged_bf16": lambda: small(n_layers=2),
    "row_blocks": lambda: small(n_q_heads=16, R=24, M=20, n_beacons_in=20, L=777, K=100),
    "two_groups": lambda: small(n_q_heads=16, R=40, M=40, n_beacons_in=40, L=513, K=64),
    # 1152 observation rows: three groups meet in the max aggregation's row of keys
    "three_groups": lambda: small(n_q_heads=16, R=64, M=80, n_beacons_in=80, L=700, K=150),
    "one_key": lambda: small(L=1, K=1, capacity=16),
    "short": lambda: small(L=129, K=5),
    "recent_only": lambda: small(n_beacons_in=0, L=300),
    "beacons_only": lambda: small(R=0, L=300),
    "exact_tiles": lambda: small(n_q_heads=8, n_kv_heads=1, R=32, M=32, n_beacons_in=32,
                                 L=4096, K=1024, capacity=4096),
    "big_norms": lambda: small(big_key_frac=0.05, big_key_norm=40.0, L=2000, K=500),
    "rising_logits": lambda: small(L=1000, K=200),
}


def _rising_logits(inp):
    """Keys whose first channel climbs from 0 to 400 along the cache, with a
    spike of 800 at 80% of it, and queries whose first channel runs from -1
    to 4 over the rows: the logits of the leaning rows climb by ~200 log2
    units (a spike ~400 up), so the row statistics move their reference in
    mid-row, past the 2^64 and 2^128 marks; the rows at -1 see the logits
    fall as far (their exps underflow)."""
    gen = torch.Generator().manual_seed(123)
    L = inp.wl.L
    ramp = torch.linspace(0.0, 400.0, L)
    ramp[int(0.8 * L)] = 800.0
    k = 0.5 * torch.randn(inp.k[:, :, :L].shape, generator=gen)
    k[..., 0] += ramp
    inp.k[:, :, :L] = k.to(inp.k.dtype)
    for t in (inp.recent, inp.beacons):
        q = 0.5 * torch.randn(t.shape, generator=gen)
        q[..., 0] = torch.linspace(-1.0, 4.0, t.shape[2])
        t.copy_(q.to(t.dtype))


INPUT_HOOKS = {"rising_logits": _rising_logits}


def score_inputs(case, wl, seed):
    inp = _synth().make_step_inputs(wl, seed=seed)
    if case in INPUT_HOOKS:
        INPUT_HOOKS[case](inp)
    return inp


@pytest.mark.parametrize("case", sorted(SCORE_CASES))
def test_score_select_compact(case, dev):
    bkv, synth = _lib(), _synth()
    wl = SCORE_CASES[case]()
    inp = score_inputs(case, wl, seed=11)
    g = bkv.geometry_of(inp.k, wl.n_q_heads)
    k, v = inp.k.to(dev), inp.v.to(dev)
    rq, bq = inp.recent.to(dev), inp.beacons.to(dev)
    H = wl.n_heads
    scores = torch.full((wl.n_layers, wl.n_kv_heads, wl.L), -1.0, device=dev)
    ws = torch.empty(bkv.bkv_workspace_size(g, wl.L, wl.R, wl.M, 0, wl.K), dtype=torch.uint8,
                     device=dev)
    bkv.bkv_score(g, k, wl.L, rq if wl.R else None, wl.R, bq if wl.beacons_in else None,
                  wl.beacons_in, wl.M, 0.0, scores, ws)
    keep = min(wl.K, wl.L)
    idx = torch.full((H, keep), -1, dtype=torch.int32, device=dev)
    bkv.bkv_select_topk(scores, H, wl.L, wl.K, idx, ws)
    dst = bkv.Geometry(g.n_layers, g.n_q_heads, g.n_kv_heads, g.head_dim, keep, g.dtype)
    kd = torch.empty(wl.n_layers, wl.n_kv_heads, keep, wl.head_dim, dtype=inp.k.dtype, device=dev)
    vd = torch.empty_like(kd)
    bkv.bkv_compact(g, k, v, idx, keep, dst, kd, vd)
    torch.cuda.synchronize()
    assert bkv.bkv_read_device_status()[0] == 0
    s_all = scores.double().cpu().numpy()
    idx_all = idx.cpu().numpy()
    kd_raw, vd_raw = raw(kd), raw(vd)
    k_raw, v_raw = raw(inp.k), raw(inp.v)
    for l in range(wl.n_layers):
        for h in range(wl.n_kv_heads):
            kk, vv, rr, bb, _ = synth.head_slice(inp, l, h)
            s_ref, _ = oracle.score_head(f64(kk), f64(rr), f64(bb), wl.beacons_in)
            check_scores(s_all[l, h], s_ref, f"{case} scores l{l} h{h}")
            r = l * wl.n_kv_heads + h
            check_topk(idx_all[r], s_ref, wl.K, f"{case} top-K l{l} h{h}")
            check_compaction(kd_raw[l, h], k_raw[l, h], idx_all[r], f"{case} K rows")
            check_compaction(vd_raw[l, h], v_raw[l, h], idx_all[r], f"{case} V rows")


@pytest.mark.parametrize("case", sorted(SCORE_CASES))
def test_score_mean(case, dev):
    """Mean aggregation (Table 2's ablation) against the oracle's mean, then
    top-K on those scores; the mean of softmax rows sums to 1 over the keys."""
    bkv, synth = _lib(), _synth()
    wl = SCORE_CASES[case]()
    inp = score_inputs(case, wl, seed=12)
    g = bkv.geometry_of(inp.k, wl.n_q_heads)
    k = inp.k.to(dev)
    rq, bq = inp.recent.to(dev), inp.beacons.to(dev)
    H = wl.n_heads
    scores = torch.full((wl.n_layers, wl.n_kv_heads, wl.L), -1.0, device=dev)
    ws = torch.empty(bkv.bkv_workspace_size(g, wl.L, wl.R, wl.M, 0, wl.K), dtype=torch.uint8,
                     device=dev)
    bkv.bkv_score_mean(g, k, wl.L, rq if wl.R else None, wl.R, bq if wl.beacons_in else None,
                       wl.beacons_in, wl.M, 0.0, scores, ws)
    keep = min(wl.K, wl.L)
    idx = torch.full((H, keep), -1, dtype=torch.int32, device=dev)
    bkv.bkv_select_topk(scores, H, wl.L, wl.K, idx, ws)
    torch.cuda.synchronize()
    assert bkv.bkv_read_device_status()[0] == 0
    s_all = scores.double().cpu().numpy()
    idx_all = idx.cpu().numpy()
    for l in range(wl.n_layers):
        for h in range(wl.n_kv_heads):
            kk, _, rr, bb, _ = synth.head_slice(inp, l, h)
            s_ref, _ = oracle.score_head(f64(kk), f64(rr), f64(bb), wl.beacons_in,
                                         aggregate="mean")
            check_scores(s_all[l, h], s_ref, f"{case} mean scores l{l} h{h}")
            assert abs(s_all[l, h].sum() - 1.0) < 1e-3, (case, l, h, s_all[l, h].sum())
            check_topk(idx_all[l * wl.n_kv_heads + h], s_ref, wl.K, f"{case} mean top-K l{l} h{h}")


def _threshold_bin_rows(rng, n_bin):
    """Rows whose K-th largest score falls in [1, 1.125) -- one bin of the
    select's first 12-bit digit (sign, exponent, 3 mantissa bits) -- holding
    exactly n_bin keys: 100 keys above it, the rest below."""
    L = 32768
    rows = []
    for _ in range(2):
        x = rng.uniform(0.0, 0.5, L)
        pos = rng.permutation(L)
        x[pos[:100]] = rng.uniform(2.0, 4.0, 100)
        x[pos[100:100 + n_bin]] = rng.uniform(1.0, 1.125, n_bin)
        rows.append(x)
    return np.stack(rows), 3100


SELECT_CASES = {
    "normal": lambda rng: (rng.standard_normal((6, 32768)), 6144),
    "scores_like": lambda rng: (np.exp(rng.standard_normal((8, 32768)) * 2.0 - 12.0), 6144),
    "rows_unaligned": lambda rng: (rng.standard_normal((5, 1001)), 300),
    "ragged_slices": lambda rng: (rng.standard_normal((3, 1004)), 17),
    "all_equal": lambda rng: (np.full((3, 20000), 0.25), 777),
    "one_top_bin": lambda rng: (1.0 + rng.integers(0, 4096, (4, 32768)) * 2.0 ** -20, 5000),
    "few_levels": lambda rng: (rng.integers(0, 7, (4, 32768)).astype(np.float64), 10000),
    "signed_zeros": lambda rng: (rng.choice([-0.0, 0.0, -1.0, 1.0, 0.5], size=(4, 4096)), 1500),
    "infinities": lambda rng: (np.where(rng.random((3, 8192)) < 0.01,
                                        rng.choice([np.inf, -np.inf], size=(3, 8192)),
                                        rng.standard_normal((3, 8192)) * 1e30), 700),
    "bin_at_list_capacity": lambda rng: _threshold_bin_rows(rng, 6144),
    "bin_past_list_capacity": lambda rng: _threshold_bin_rows(rng, 6145),
    "k_one": lambda rng: (rng.standard_normal((2, 5000)), 1),
    "k_all_but_one": lambda rng: (rng.standard_normal((2, 4096)), 4095),
    "long_rows": lambda rng: (np.exp(rng.uniform(-60.0, 0.0, (2, 1 << 20))), 1 << 17),
}


@pytest.mark.parametrize("case", sorted(SELECT_CASES))
def test_select_topk_exact(case, dev):
    """The select on float32 scores is exact: the same positions, in the same
    order, as the oracle's selection on those scores (ties to the lower
    position, -0 equal to +0), over both of the kernel's routes -- a threshold
    bin collected in shared memory, and the streaming radix for rows whose
    threshold bin is too full or whose rows are not 16-byte aligned."""
    bkv = _lib()
    x, K = SELECT_CASES[case](np.random.default_rng(31))
    x32 = np.ascontiguousarray(x, dtype=np.float32)
    n_rows, L = x32.shape
    scores = torch.from_numpy(x32).to(dev)
    idx = torch.full((n_rows, min(K, L)), -1, dtype=torch.int32, device=dev)
    bkv.bkv_select_topk(scores, n_rows, L, K, idx, None)
    torch.cuda.synchronize()
    assert bkv.bkv_read_device_status()[0] == 0
    got = idx.cpu().numpy()
    for r in range(n_rows):
        ref = oracle.select_topk(x32[r].astype(np.float64), K)
        assert np.array_equal(got[r], ref), (case, r, np.flatnonzero(got[r] != ref)[:5])


FPS_CASES = {
    "tiny_f32": lambda: _synth().WORKLOADS["tiny"],
    "bf16_small": lambda: small(W=300, M=24, n_beacons_in=10),
    "no_beacons": lambda: small(W=40, M=16, n_beacons_in=0),
    "window_lt_M": lambda: small(W=5, M=16, n_beacons_in=4),
    "window_only_one": lambda: small(W=1, M=4, n_beacons_in=0, R=1),
    "ragged_tiles": lambda: small(W=333, M=40, n_beacons_in=37),
    "many_rounds": lambda: small(n_q_heads=2, n_kv_heads=1, W=1200, M=128, n_beacons_in=100),
    # unions too large for the shared-memory distance arrays: the tensor-core
    # kernel keeps them in the workspace (one slice per CTA)
    "large_union": lambda: small(n_q_heads=2, n_kv_heads=1, W=9000, M=32, n_beacons_in=32),
    # naive FPS (Fig. 7's baseline): the whole query history, no beacons
    "naive_history": lambda: small(n_q_heads=4, n_kv_heads=1, W=20000, M=48, n_beacons_in=0),
    # 1500 copies of one window row: the candidate select's threshold bin
    # holds them all, past what it ranks directly, so its fallbacks run
    "duplicate_rows": lambda: small(n_q_heads=2, n_kv_heads=1, W=2000, M=64, n_beacons_in=16),
    # a window of nearly parallel rows: every distance below 1e-3
    "near_parallel": lambda: small(n_q_heads=2, n_kv_heads=1, W=600, M=32, n_beacons_in=8),
    # more than 128 beacons, and bf16 rows of 64 dimensions: the CUDA-core kernel
    "many_beacons": lambda: small(n_q_heads=2, n_kv_heads=1, W=400, M=160, n_beacons_in=100),
    "bf16_d64": lambda: small(head_dim=64, W=300, M=24, n_beacons_in=10),
}


def _duplicate_rows(inp):
    inp.window[:, :, 200:1700] = inp.window[:, :, 100:101]


def _near_parallel(inp):
    gen = torch.Generator().manual_seed(77)
    base = torch.randn(inp.window.shape[:2] + (1, inp.window.shape[-1]), generator=gen)
    noise = 0.02 * torch.randn(inp.window.shape, generator=gen)
    inp.window.copy_((base + noise).to(inp.window.dtype))
    nb = inp.beacons.shape[2]
    bnoise = 0.02 * torch.randn(inp.beacons.shape, generator=gen)
    inp.beacons.copy_((base.expand(-1, -1, nb, -1) + bnoise).to(inp.beacons.dtype))


FPS_HOOKS = {"duplicate_rows": _duplicate_rows, "near_parallel": _near_parallel}


@pytest.mark.parametrize("case", sorted(FPS_CASES))
def test_update_beacons(case, dev):
    bkv, synth = _lib(), _synth()
    wl = FPS_CASES[case]()
    inp = synth.make_step_inputs(wl, seed=5)
    if case in FPS_HOOKS:
        FPS_HOOKS[case](inp)
    g = bkv.geometry_of(inp.k, wl.n_q_heads)
    bin_, win = inp.beacons.to(dev), inp.window.to(dev)
    bout = torch.zeros_like(bin_)
    ws = torch.empty(max(1, bkv.bkv_workspace_size(g, 1, 0, wl.M, wl.W, 1)), dtype=torch.uint8,
                     device=dev)
    n = bkv.bkv_update_beacons(g, bin_ if wl.beacons_in else None, wl.beacons_in, wl.M, win,
                               wl.W, bout, ws)
    torch.cuda.synchronize()
    assert bkv.bkv_read_device_status()[0] == 0
    assert n == min(wl.M, wl.beacons_in + wl.W)
    out_raw = raw(bout)
    for l in range(wl.n_layers):
        for qh in range(wl.n_q_heads):
            U = torch.cat([inp.beacons[l, qh, :wl.beacons_in], inp.window[l, qh]])
            picks = picks_from_rows(raw(U), out_raw[l, qh, :n])
            check_fps(f64(U), picks, wl.M, f"{case} l{l} q{qh}")


def _run_step(wl, inp, dev, scores=True, aggregate="max", aux=False):
    bkv = _lib()
    g = bkv.geometry_of(inp.k, wl.n_q_heads)
    keep = min(wl.K, wl.L)
    dst = bkv.Geometry(g.n_layers, g.n_q_heads, g.n_kv_heads, g.head_dim, keep, g.dtype)
    t = {n: getattr(inp, n).to(dev) for n in ("k", "v", "recent", "beacons", "window")}
    out = dict(
        bout=torch.zeros_like(t["beacons"]),
        kd=torch.empty(wl.n_layers, wl.n_kv_heads, keep, wl.head_dim, dtype=inp.k.dtype,
                       device=dev),
        scores=torch.empty(wl.n_layers, wl.n_kv_heads, wl.L, device=dev) if scores else None,
        idx=torch.empty(wl.n_layers, wl.n_kv_heads, keep, dtype=torch.int32, device=dev),
    )
    out["vd"] = torch.empty_like(out["kd"])
    ws = torch.empty(bkv.bkv_workspace_size(g, wl.L, wl.R, wl.M, wl.W, wl.K), dtype=torch.uint8,
                     device=dev)
    nb, nl = bkv.bkv_compress_step(
        g, t["k"], t["v"], wl.L, wl.K, t["recent"] if wl.R else None, wl.R,
        t["beacons"] if wl.beacons_in else None, wl.beacons_in, wl.M,
        t["window"] if wl.W else None, wl.W, out["bout"], 0.0, dst, out["kd"], out["vd"],
        out["scores"], out["idx"], ws, aggregate=aggregate,
        aux_stream=torch.cuda.Stream(device=dev, priority=-1) if aux else None)
    torch.cuda.synchronize()
    assert bkv.bkv_read_device_status()[0] == 0
    assert nl == keep
    assert nb == (min(wl.M, wl.beacons_in + wl.W) if wl.W else wl.beacons_in)
    return out, nb


def _check_step_heads(wl, inp, out, nb, heads, what, aggregate="max"):
    """Oracle comparison of whole-step outputs for the sampled (layer, KV head)s.

    Every head is compared.  When the GPU's FPS picks equal the oracle's, the
    whole oracle step is the reference; when they differ at a legal near-tie
    (each pick within 1e-5 of the farthest distance, checked by replay), the
    GPU's beacons are a valid Continual FPS result, and the oracle scores the
    head with those beacons.  Returns (heads whose picks were exact, the
    largest |s_gpu - s_ref| / (1e-6 + 1e-3 |s_ref|) seen)."""
    synth = _synth()
    G = wl.group
    out_b = out["bout"].double().cpu().numpy()
    out_b_raw = raw(out["bout"])
    s_all = out["scores"].double().cpu().numpy() if out["scores"] is not None else None
    idx_all = out["idx"].cpu().numpy()
    kd_raw, vd_raw = raw(out["kd"]), raw(out["vd"])
    k_raw, v_raw = raw(inp.k), raw(inp.v)

    def one_head(lh):
        l, h = lh
        kk, vv, rr, bb, ww = synth.head_slice(inp, l, h)
        exact = True
        if wl.W:
            for gq in range(G):
                U = torch.cat([bb[gq, :wl.beacons_in], ww[gq]])
                picks = picks_from_rows(raw(U), out_b_raw[l, h * G + gq, :nb])
                exact &= check_fps(f64(U), picks, wl.M, f"{what} FPS l{l} q{h * G + gq}")
        check_compaction(kd_raw[l, h], k_raw[l, h], idx_all[l, h], f"{what} K rows l{l} h{h}")
        check_compaction(vd_raw[l, h], v_raw[l, h], idx_all[l, h], f"{what} V rows l{l} h{h}")
        if exact:
            ref = oracle.compress_head(f64(kk), f64(vv), f64(rr), f64(bb), wl.beacons_in,
                                       f64(ww) if wl.W else None, wl.M, wl.K,
                                       aggregate=aggregate)
            s_ref = ref["scores"]
        else:
            # the GPU's beacons (a valid FPS result at a near-tie) as scored
            s_ref, _ = oracle.score_head(f64(kk), f64(rr), out_b[l, h * G:(h + 1) * G], nb,
                                         aggregate=aggregate)
        err = 0.0
        if s_all is not None:
            err = check_scores(s_all[l, h], s_ref, f"{what} scores l{l} h{h}")
        check_topk(idx_all[l, h], s_ref, wl.K, f"{what} top-K l{l} h{h}")
        return exact, err

    # the oracle runs in C through ctypes, which releases the GIL: one thread per head
    with ThreadPoolExecutor(max_workers=min(len(heads), os.cpu_count() or 1)) as ex:
        results = list(ex.map(one_head, heads))
    return sum(1 for e, _ in results if e), max((w for _, w in results), default=0.0)


STEP_CASES = {
    "tiny_f32": lambda: _synth().WORKLOADS["tiny"],
    "bf16_fps": lambda: small(n_layers=2, W=200, M=16, n_beacons_in=8, L=1500, K=400,
                              capacity=1600),
    "keep_all": lambda: small(L=200, K=512, W=20, capacity=256),
    "no_window": lambda: small(W=0),
}


@pytest.mark.parametrize("case", sorted(STEP_CASES))
def test_compress_step_small(case, dev):
    wl = STEP_CASES[case]()
    inp = _synth().make_step_inputs(wl, seed=3)
    out, nb = _run_step(wl, inp, dev)
    heads = [(l, h) for l in range(wl.n_layers) for h in range(wl.n_kv_heads)]
    n_exact, _ = _check_step_heads(wl, inp, out, nb, heads, case)
    assert n_exact == len(heads), "FPS near-ties on a small case"


@pytest.mark.parametrize("case", sorted(STEP_CASES))
def test_compress_step_mean(case, dev):
    """The whole step with mean aggregation."""
    wl = STEP_CASES[case]()
    inp = _synth().make_step_inputs(wl, seed=4)
    out, nb = _run_step(wl, inp, dev, aggregate="mean")
    heads = [(l, h) for l in range(wl.n_layers) for h in range(wl.n_kv_heads)]
    n_exact, _ = _check_step_heads(wl, inp, out, nb, heads, case + " mean", aggregate="mean")
    assert n_exact == len(heads), "FPS near-ties on a small case"


FULL = ["r1_qwen7b", "llama8b", "qwen3_4b_step", "qwen3_14b"]


@pytest.mark.slow
@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled(name, dev):
    """The benchmark's launch configuration at full size; sampled heads vs the oracle."""
    synth = _synth()
    wl = synth.WORKLOADS[name]
    inp = synth.make_step_inputs(wl, seed=0)
    out, nb = _run_step(wl, inp, dev)
    rng = np.random.default_rng(123)
    heads = sorted({(int(rng.integers(wl.n_layers)), int(rng.integers(wl.n_kv_heads)))
                    for _ in range(7)} | {(0, 0), (wl.n_layers - 1, wl.n_kv_heads - 1)})
    n_exact, worst = _check_step_heads(wl, inp, out, nb, heads, name)
    print(f"{name}: {len(heads)} heads compared ({n_exact} with the oracle's own picks), "
          f"largest score error / tolerance {worst:.3g}")
    # compaction of every head: each kept row is a byte copy of its source row
    idx = out["idx"].long()
    k_dev = inp.k.to(dev)
    gathered = torch.gather(k_dev, 2, idx[..., None].expand(-1, -1, -1, wl.head_dim))
    assert torch.equal(gathered.view(torch.int16), out["kd"].view(torch.int16))
    # kept positions are strictly ascending in every head
    assert bool((idx[..., 1:] > idx[..., :-1]).all())


@pytest.mark.slow
def test_full_size_sampled_mean(dev):
    """Mean aggregation in the 14B launch configuration; sampled heads vs the oracle."""
    synth = _synth()
    wl = synth.WORKLOADS["qwen3_14b"]
    inp = synth.make_step_inputs(wl, seed=5)
    out, nb = _run_step(wl, inp, dev, aggregate="mean")
    rng = np.random.default_rng(321)
    heads = sorted({(int(rng.integers(wl.n_layers)), int(rng.integers(wl.n_kv_heads)))
                    for _ in range(2)} | {(0, 0)})
    n_exact, worst = _check_step_heads(wl, inp, out, nb, heads, "qwen3_14b mean",
                                       aggregate="mean")
    print(f"qwen3_14b mean: {len(heads)} heads compared ({n_exact} with the oracle's own "
          f"picks), largest score error / tolerance {worst:.3g}")
    sums = out["scores"].double().sum(-1)
    assert bool(((sums - 1.0).abs() < 1e-3).all()), sums.flatten()[:8]


def _ascending_positions(rng, cap, n_keep, mode):
    """Kept positions in [0, cap), ascending, with the shapes compaction meets."""
    if mode == "prefix_kept":       # the first rows stay, then a sparse tail
        head = np.arange(n_keep // 3)
        rest = np.sort(rng.choice(np.arange(n_keep // 3, cap), n_keep - head.size, replace=False))
        return np.concatenate([head, rest])
    if mode == "tail":              # only the newest rows survive
        return np.arange(cap - n_keep, cap)
    return np.sort(rng.choice(cap, n_keep, replace=False))


@pytest.mark.parametrize("dtype,d,cap,n_keep,mode", [
    ("bf16", 128, 1000, 300, "random"),
    ("bf16", 128, 4096, 1537, "prefix_kept"),
    ("bf16", 128, 777, 777, "random"),        # every row kept: nothing moves
    ("bf16", 128, 5000, 129, "tail"),
    ("f32", 128, 2000, 1000, "random"),       # 512-byte rows: 32-row chunks
    ("f32", 24, 999, 400, "prefix_kept"),     # 96-byte rows: chunks of 170 rows
    ("bf16", 64, 3000, 1000, "random"),       # 128-byte rows: 256-row chunks
    ("f32", 256, 600, 250, "prefix_kept"),    # 1024-byte rows: 32-row chunks
])
def test_compact_inplace(dtype, d, cap, n_keep, mode, dev):
    """In-place compaction equals the out-of-place gather, byte for byte."""
    bkv = _lib()
    rng = np.random.default_rng(cap + n_keep)
    Ly, Hkv = 2, 3
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    k0 = torch.randn(Ly, Hkv, cap, d, generator=torch.Generator().manual_seed(1)).to(tdt)
    v0 = torch.randn(Ly, Hkv, cap, d, generator=torch.Generator().manual_seed(2)).to(tdt)
    idx = np.stack([_ascending_positions(rng, cap, n_keep, mode) for _ in range(Ly * Hkv)])
    idx_t = torch.from_numpy(idx.astype(np.int32)).to(dev)
    k, v = k0.to(dev), v0.to(dev)
    g = bkv.Geometry(Ly, Hkv, Hkv, d, cap, tdt)
    bkv.bkv_compact_inplace(g, k, v, idx_t, n_keep)
    torch.cuda.synchronize()
    assert bkv.bkv_read_device_status()[0] == 0
    kr, vr = raw(k), raw(v)
    k0r, v0r = raw(k0), raw(v0)
    for r in range(Ly * Hkv):
        l, h = divmod(r, Hkv)
        check_compaction(kr[l, h, :n_keep], k0r[l, h], idx[r], f"in-place K {mode} r{r}")
        check_compaction(vr[l, h, :n_keep], v0r[l, h], idx[r], f"in-place V {mode} r{r}")
        # rows past n_keep are left as they were or hold moved-from data; the
        # kept prefix is all that is defined


def test_compact_inplace_reports_a_backward_index(dev):
    """A position below its slot is skipped and reported, not followed."""
    bkv = _lib()
    cap, n_keep, d = 512, 200, 128
    k = torch.randn(1, 1, cap, d, device=dev).to(torch.bfloat16)
    before = raw(k)
    idx = torch.arange(n_keep, dtype=torch.int32) + 5
    idx[150] = 3                                   # 3 < 150: breaks idx[i] >= i
    g = bkv.Geometry(1, 1, 1, d, cap, torch.bfloat16)
    bkv.bkv_compact_inplace(g, k, None, idx.to(dev), n_keep)
    st, where = bkv.bkv_read_device_status()
    assert st == 6 and where == 501                # BKV_ERR_DEVICE_ASSERT
    after = raw(k)
    good = [i for i in range(n_keep) if i != 150]
    assert np.array_equal(after[0, 0, good], before[0, 0, np.array(good) + 5])


def test_compact_reports_a_position_outside_the_cache(dev):
    """A kept position past the source capacity is skipped and reported, and
    every other row is still copied byte for byte."""
    bkv = _lib()
    cap, n_keep, d = 300, 100, 128
    k = torch.randn(1, 2, cap, d, device=dev).to(torch.bfloat16)
    v = torch.randn(1, 2, cap, d, device=dev).to(torch.bfloat16)
    idx = torch.stack([torch.arange(n_keep, dtype=torch.int32) * 2 + r for r in range(2)])
    idx[1, 40] = cap + 5                            # outside the source cache
    g = bkv.Geometry(1, 2, 2, d, cap, torch.bfloat16)
    gd = bkv.Geometry(1, 2, 2, d, n_keep, torch.bfloat16)
    kd = torch.zeros(1, 2, n_keep, d, dtype=torch.bfloat16, device=dev)
    vd = torch.zeros_like(kd)
    bkv.bkv_compact(g, k, v, idx.to(dev), n_keep, gd, kd, vd)
    st, where = bkv.bkv_read_device_status()
    assert st == 6 and where == 502                # BKV_ERR_DEVICE_ASSERT
    kr, vr, kdr, vdr = raw(k), raw(v), raw(kd), raw(vd)
    for r in range(2):
        good = [i for i in range(n_keep) if (r, i) != (1, 40)]
        src = idx[r, good].long().numpy()
        assert np.array_equal(kdr[0, r, good], kr[0, r, src])
        assert np.array_equal(vdr[0, r, good], vr[0, r, src])
    assert not kdr[0, 1, 40].any() and not vdr[0, 1, 40].any()   # left as it was
    assert bkv.bkv_read_device_status()[0] == 0    # the code was cleared


@pytest.mark.parametrize("case", ["bf16_fps", "no_window", "keep_all"])
def test_compress_step_in_place(case, dev):
    """The step with the source cache as destination gives the out-of-place result."""
    bkv, synth = _lib(), _synth()
    wl = STEP_CASES[case]()
    inp = synth.make_step_inputs(wl, seed=6)
    out, nb = _run_step(wl, inp, dev)
    g = bkv.geometry_of(inp.k, wl.n_q_heads)
    t = {n: getattr(inp, n).to(dev) for n in ("k", "v", "recent", "beacons", "window")}
    keep = min(wl.K, wl.L)
    bout = torch.zeros_like(t["beacons"])
    idx = torch.empty(wl.n_layers, wl.n_kv_heads, keep, dtype=torch.int32, device=dev)
    ws = torch.empty(bkv.bkv_workspace_size(g, wl.L, wl.R, wl.M, wl.W, wl.K), dtype=torch.uint8,
                     device=dev)
    nb2, nl = bkv.bkv_compress_step(
        g, t["k"], t["v"], wl.L, wl.K, t["recent"] if wl.R else None, wl.R,
        t["beacons"] if wl.beacons_in else None, wl.beacons_in, wl.M,
        t["window"] if wl.W else None, wl.W, bout, 0.0, g, t["k"], t["v"], None, idx, ws)
    torch.cuda.synchronize()
    assert bkv.bkv_read_device_status()[0] == 0
    assert (nb2, nl) == (nb, keep)
    assert torch.equal(idx, out["idx"])
    assert np.array_equal(raw(t["k"])[:, :, :keep], raw(out["kd"]))
    assert np.array_equal(raw(t["v"])[:, :, :keep], raw(out["vd"]))


RING_CASES = {
    # ring of 300 slots, 700 queries written: the 200-row window starts at
    # slot 200 and wraps to slot 99; the 8 recent rows are slots 92..99
    "wraps_mid_window": dict(cap=300, pos=700, W=200, R=8),
    # the window ends exactly at the ring's end (no wrap), recent rows too
    "ends_at_ring_end": dict(cap=256, pos=512, W=128, R=16),
    # the whole ring is the window, starting mid-ring; recent rows wrap
    "full_ring": dict(cap=260, pos=1000 + 3, W=260, R=5),
}


@pytest.mark.parametrize("case", sorted(RING_CASES))
def test_compress_step_query_ring(case, dev):
    """The step reading its recent queries and window in place from a
    decode-side query ring (slot of query t = t mod cap) equals the step on
    the same queries unrolled into dense blocks, bit for bit, and matches the
    oracle on the ring's newest rows (oracle.ring_rows)."""
    bkv, synth = _lib(), _synth()
    rc = RING_CASES[case]
    cap, pos, W, R = rc["cap"], rc["pos"], rc["W"], rc["R"]
    wl = small(n_layers=2, W=W, R=R, M=24, n_beacons_in=10, L=900, K=250, capacity=1000)
    inp = synth.make_step_inputs(wl, seed=9)
    gen = torch.Generator().manual_seed(cap + pos)
    # the decode history: pos queries per query head, written into the ring in order
    hist = (8.0 * torch.randn(wl.n_layers, wl.n_q_heads, 1, 128, generator=gen)
            + 0.5 * torch.randn(wl.n_layers, wl.n_q_heads, pos, 128, generator=gen)
            ).to(torch.bfloat16)
    ring = torch.zeros(wl.n_layers, wl.n_q_heads, cap, 128, dtype=torch.bfloat16)
    for t in range(pos):
        ring[:, :, t % cap] = hist[:, :, t]
    window = hist[:, :, pos - W:].contiguous()
    recent = hist[:, :, pos - R:].contiguous()
    np.testing.assert_array_equal(raw(window), oracle.ring_rows(raw(ring), pos % cap, W))
    np.testing.assert_array_equal(raw(recent), oracle.ring_rows(raw(ring), pos % cap, R))
    g = bkv.geometry_of(inp.k, wl.n_q_heads)
    keep = min(wl.K, wl.L)
    dst = bkv.Geometry(g.n_layers, g.n_q_heads, g.n_kv_heads, g.head_dim, keep, g.dtype)
    k, v, bq = inp.k.to(dev), inp.v.to(dev), inp.beacons.to(dev)
    ws = torch.empty(bkv.bkv_workspace_size(g, wl.L, R, wl.M, cap, wl.K), dtype=torch.uint8,
                     device=dev)
    outs = []
    for use_ring in (False, True):
        o = dict(bout=torch.zeros_like(bq),
                 kd=torch.empty(wl.n_layers, wl.n_kv_heads, keep, 128, dtype=torch.bfloat16,
                                device=dev),
                 scores=torch.empty(wl.n_layers, wl.n_kv_heads, wl.L, device=dev),
                 idx=torch.empty(wl.n_layers, wl.n_kv_heads, keep, dtype=torch.int32,
                                 device=dev))
        o["vd"] = torch.empty_like(o["kd"])
        if use_ring:
            nb, nl = bkv.bkv_compress_step(
                g, k, v, wl.L, wl.K, None, R, bq, wl.beacons_in, wl.M, None, W, o["bout"], 0.0,
                dst, o["kd"], o["vd"], o["scores"], o["idx"], ws, query_ring=ring.to(dev),
                ring_pos=pos)
        else:
            nb, nl = bkv.bkv_compress_step(
                g, k, v, wl.L, wl.K, recent.to(dev), R, bq, wl.beacons_in, wl.M,
                window.to(dev), W, o["bout"], 0.0, dst, o["kd"], o["vd"], o["scores"], o["idx"],
                ws)
        torch.cuda.synchronize()
        assert bkv.bkv_read_device_status()[0] == 0
        assert (nb, nl) == (min(wl.M, wl.beacons_in + W), keep)
        outs.append(o)
    for name in ("bout", "kd", "vd", "scores", "idx"):
        assert torch.equal(outs[0][name], outs[1][name]), name
    # the oracle on the ring's newest rows
    G = wl.group
    out_b = raw(outs[1]["bout"])
    s_all = outs[1]["scores"].double().cpu().numpy()
    idx_all = outs[1]["idx"].cpu().numpy()
    for l in range(wl.n_layers):
        for h in range(wl.n_kv_heads):
            kk, vv, _, bb, _ = synth.head_slice(inp, l, h)
            rg = raw(ring[l, h * G:(h + 1) * G])
            win_raw = oracle.ring_rows(rg, pos % cap, W)
            win64 = oracle.ring_rows(f64(ring[l, h * G:(h + 1) * G]), pos % cap, W)
            rec64 = oracle.newest_rows(win64, R) if R <= W else None
            exact = True
            for gq in range(G):
                U_raw = np.concatenate([raw(bb[gq, :wl.beacons_in]), win_raw[gq]])
                U64 = np.concatenate([f64(bb[gq, :wl.beacons_in]), win64[gq]])
                picks = picks_from_rows(U_raw, out_b[l, h * G + gq, :nb])
                exact &= check_fps(U64, picks, wl.M, f"ring {case} FPS l{l} q{h * G + gq}")
            rec64 = oracle.ring_rows(f64(ring[l, h * G:(h + 1) * G]), pos % cap, R)
            s_ref, _ = oracle.score_head(f64(kk), rec64,
                                         outs[1]["bout"][l, h * G:(h + 1) * G].double().cpu().numpy(),
                                         nb)
            check_scores(s_all[l, h], s_ref, f"ring {case} scores l{l} h{h}")
            check_topk(idx_all[l, h], s_ref, wl.K, f"ring {case} top-K l{l} h{h}")


@pytest.mark.parametrize("case,aggregate", [("bf16_fps", "max"), ("bf16_fps", "mean"),
                                            ("no_window", "max")])
def test_compress_step_aux_stream(case, aggregate, dev):
    """With a second stream, each head batch's top-K and compaction overlap the
    next batch's aggregation; the results are those of the one-stream step,
    bit for bit (out of place, then in place)."""
    wl = STEP_CASES[case]().replace(n_layers=3, n_kv_heads=2, n_q_heads=8)
    inp = _synth().make_step_inputs(wl, seed=13)
    one, nb1 = _run_step(wl, inp, dev, aggregate=aggregate)
    two, nb2 = _run_step(wl, inp, dev, aggregate=aggregate, aux=True)
    assert nb1 == nb2
    for name in ("bout", "kd", "vd", "scores", "idx"):
        assert torch.equal(one[name], two[name]), name
    # in place with the aux stream: the cache itself becomes the compacted one
    bkv = _lib()
    g = bkv.geometry_of(inp.k, wl.n_q_heads)
    t = {n: getattr(inp, n).to(dev) for n in ("k", "v", "recent", "beacons", "window")}
    keep = min(wl.K, wl.L)
    idx = torch.empty(wl.n_layers, wl.n_kv_heads, keep, dtype=torch.int32, device=dev)
    ws = torch.empty(bkv.bkv_workspace_size(g, wl.L, wl.R, wl.M, wl.W, wl.K), dtype=torch.uint8,
                     device=dev)
    bkv.bkv_compress_step(
        g, t["k"], t["v"], wl.L, wl.K, t["recent"] if wl.R else None, wl.R,
        t["beacons"] if wl.beacons_in else None, wl.beacons_in, wl.M,
        t["window"] if wl.W else None, wl.W, torch.zeros_like(t["beacons"]), 0.0, g, t["k"],
        t["v"], None, idx, ws, aggregate=aggregate,
        aux_stream=torch.cuda.Stream(device=dev, priority=-1))
    torch.cuda.synchronize()
    assert bkv.bkv_read_device_status()[0] == 0
    assert torch.equal(idx, one["idx"])
    assert np.array_equal(raw(t["k"])[:, :, :keep], raw(one["kd"]))
    assert np.array_equal(raw(t["v"])[:, :, :keep], raw(one["vd"]))
