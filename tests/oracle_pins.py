"""Pins of the float64 oracle to facts outside the oracle itself.

Each ``pin_*`` function takes a bound oracle library (the real one, or a
mutant built by test_oracle_mutants.py) and raises AssertionError when the
oracle disagrees with:
  * hand-derived closed forms (tests/golden/closed_forms.json),
  * independent library routines (numpy matmul, scipy logsumexp / softmax,
    numpy fancy indexing, Python's sorted),
  * invariants of the definitions (softmax rows sum to one, the aggregate is
    an upper bound attained by some row),
  * brute force on tiny inputs (FPS with every min-distance recomputed from
    scratch).
Definitions: "BeaconKV: Key-Value Cache Compression Guided by Beacon Queries
for Efficient Large Reasoning Model Inference", Fig. 5(b)/(c), Table 2 and
Fig. 7.
"""
from __future__ import annotations

import json
import os

import numpy as np
from scipy.special import logsumexp, softmax

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "closed_forms.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def pin_closed_forms(lib):
    for case in _golden()["softmax_cases"]:
        q = np.array(case["q"])
        k = np.array(case["k"])
        x = oracle.logits(q, k, case["scale"], _lib=lib)
        c = oracle.row_normalizer(x, _lib=lib)
        s = oracle.max_aggregate(x, c, _lib=lib)
        np.testing.assert_allclose(c, case["c"], rtol=0, atol=1e-12, err_msg=case["name"])
        np.testing.assert_allclose(s, case["s"], rtol=0, atol=1e-12, err_msg=case["name"])
        sm = oracle.mean_aggregate(x, c, _lib=lib)
        np.testing.assert_allclose(sm, case["s_mean"], rtol=0, atol=1e-12, err_msg=case["name"])
        for K, want in case["topk"].items():
            got = oracle.select_topk(np.array(case["s"]), int(K), _lib=lib)
            assert got.tolist() == want, (case["name"], K, got.tolist(), want)
    for case in _golden()["fps_cases"]:
        sel = oracle.fps(np.array(case["U"]), case["M"], _lib=lib)
        assert sel.tolist() == case["sel"], (case["name"], sel.tolist(), case["sel"])


def pin_logits_matmul(lib):
    rng = np.random.default_rng(1)
    for n_obs, L, d in [(3, 7, 5), (6, 11, 4), (1, 1, 1), (9, 2, 13)]:
        q = rng.standard_normal((n_obs, d))
        k = rng.standard_normal((L, d))
        scale = 0.37
        x = oracle.logits(q, k, scale, _lib=lib)
        np.testing.assert_allclose(x, scale * (q @ k.T), rtol=1e-12, atol=1e-12)


def pin_softmax(lib):
    rng = np.random.default_rng(2)
    for n_obs, L in [(4, 9), (1, 1), (3, 50), (7, 3)]:
        x = rng.standard_normal((n_obs, L)) * 5.0 + rng.standard_normal((n_obs, 1)) * 30
        c = oracle.row_normalizer(x, _lib=lib)
        np.testing.assert_allclose(c, logsumexp(x, axis=1), rtol=0, atol=1e-10)
        # softmax rows sum to one
        np.testing.assert_allclose(np.exp(x - c[:, None]).sum(axis=1), 1.0, rtol=0, atol=1e-12)
        s = oracle.max_aggregate(x, c, _lib=lib)
        p = softmax(x, axis=1)
        # the aggregate bounds every constituent and equals one of them
        assert np.all(s[None, :] >= p * (1 - 1e-13))
        assert np.all(np.isclose(s[None, :], p, rtol=1e-13, atol=0).any(axis=0))
        np.testing.assert_allclose(s, p.max(axis=0), rtol=1e-12, atol=0)
        # one observation row: the aggregate is that row's softmax
        s1 = oracle.max_aggregate(x[:1], c[:1], _lib=lib)
        np.testing.assert_allclose(s1, p[0], rtol=1e-12, atol=0)
        m = oracle.mean_aggregate(x, c, _lib=lib)
        np.testing.assert_allclose(m, p.mean(axis=0), rtol=1e-12, atol=0)
        # a mean of distributions is a distribution, below the max aggregate
        np.testing.assert_allclose(m.sum(), 1.0, rtol=0, atol=1e-12)
        assert np.all(m <= s * (1 + 1e-13))


def pin_score_head_composition(lib):
    """Observation set = every query head's recent and beacon rows (Fig. 5(b))."""
    rng = np.random.default_rng(3)
    G, R, M, nb, L, d = 3, 4, 5, 2, 17, 8
    k = rng.standard_normal((L, d))
    recent = rng.standard_normal((G, R, d))
    beacons = rng.standard_normal((G, M, d))
    beacons[:, nb:] = 1e3  # slots past n_beacons must be ignored
    s, c = oracle.score_head(k, recent, beacons, nb, 0.25, _lib=lib)
    rows = [recent[g, i] for g in range(G) for i in range(R)]
    rows += [beacons[g, i] for g in range(G) for i in range(nb)]
    p = np.stack([softmax(0.25 * (k @ r)) for r in rows])
    np.testing.assert_allclose(s, p.max(axis=0), rtol=1e-12, atol=0)
    assert c.shape == (G * (R + nb),)
    sm, _ = oracle.score_head(k, recent, beacons, nb, 0.25, aggregate="mean", _lib=lib)
    np.testing.assert_allclose(sm, p.mean(axis=0), rtol=1e-12, atol=0)


def _sorted_topk(s, K):
    order = sorted(range(len(s)), key=lambda j: (-s[j], j))
    return sorted(order[:max(0, min(K, len(s)))])


def pin_topk_full_sort(lib):
    rng = np.random.default_rng(4)
    cases = []
    for L in [1, 2, 5, 16, 100, 257]:
        cases.append(rng.standard_normal(L))
        cases.append(rng.integers(0, 4, L).astype(np.float64))  # heavy ties
    for s in cases:
        L = len(s)
        for K in sorted({0, 1, 2, L // 3, L - 1, L, L + 5}):
            got = oracle.select_topk(s, K, _lib=lib)
            assert got.tolist() == _sorted_topk(s.tolist(), K), (L, K)
    s = rng.standard_normal(40)
    assert oracle.select_topk(s, 1, _lib=lib).tolist() == [int(np.argmax(s))]
    assert oracle.select_topk(s, 40, _lib=lib).tolist() == list(range(40))


def pin_compact_bytes(lib):
    rng = np.random.default_rng(5)
    src = rng.integers(0, 2**16, (33, 24), dtype=np.uint16)
    idx = np.sort(rng.choice(33, 11, replace=False)).astype(np.int32)
    np.testing.assert_array_equal(oracle.compact(src, idx, _lib=lib), src[idx])
    srcf = rng.standard_normal((9, 7)).astype(np.float32)
    idx2 = np.array([8, 0, 3], dtype=np.int32)
    assert oracle.compact(srcf, idx2, _lib=lib).tobytes() == srcf[idx2].tobytes()


def _fps_brute(U, M):
    """Greedy FPS with every point's distance to the selected set recomputed."""
    n = U.shape[0]
    nrm = np.linalg.norm(U, axis=1)
    def dist(a, b):
        if nrm[a] == 0 or nrm[b] == 0:
            return 1.0
        return float(np.clip(1.0 - (U[a] / nrm[a]) @ (U[b] / nrm[b]), 0.0, 2.0))
    sel = [0]
    while len(sel) < min(M, n):
        best, bestd = None, None
        for i in range(n):
            if i in sel:
                continue
            di = min(dist(i, s) for s in sel)
            if bestd is None or di > bestd:
                best, bestd = i, di
        sel.append(best)
    return sel[:min(M, n)]


def pin_fps_bruteforce(lib):
    rng = np.random.default_rng(6)
    for trial in range(60):
        n = int(rng.integers(1, 9))
        d = int(rng.integers(2, 6))
        U = rng.standard_normal((n, d))
        if trial % 3 == 0 and n > 2:
            U[n - 1] = U[0] * 3.0   # a duplicate direction of the seed
        M = int(rng.integers(1, 10))
        got = oracle.fps(U, M, _lib=lib).tolist()
        assert got == _fps_brute(U, M), (trial, got)


def pin_fps_special_sets(lib):
    # orthonormal: every distance is 1 -> picks in index order
    E = np.eye(6)
    assert oracle.fps(E, 6, _lib=lib).tolist() == [0, 1, 2, 3, 4, 5]
    # collinear (same direction): every distance 0 -> lowest unselected index
    C = np.outer(np.arange(1, 6, dtype=np.float64), np.array([1.0, 2.0, -1.0]))
    assert oracle.fps(C, 4, _lib=lib).tolist() == [0, 1, 2, 3]
    # a query equal to a beacon is not added while a positive distance remains
    rng = np.random.default_rng(7)
    B = rng.standard_normal((4, 8))
    Wn = np.concatenate([B[2:3], rng.standard_normal((3, 8)), B[0:1] * 2.0])
    U = np.concatenate([B, Wn])
    sel = oracle.fps(U, 7, _lib=lib).tolist()
    assert 4 not in sel and 8 not in sel, sel
    # M larger than the union: everything, each once
    assert sorted(oracle.fps(U, 50, _lib=lib).tolist()) == list(range(U.shape[0]))


def pin_fps_replay(lib):
    rng = np.random.default_rng(8)
    U = rng.standard_normal((30, 5))
    sel = oracle.fps(U, 10, _lib=lib)
    bad, gap = oracle.fps_replay(U, sel, 1e-9, _lib=lib)
    assert bad == -1 and gap <= 1e-12
    wrong = sel.copy()
    wrong[3] = [i for i in range(30) if i not in sel][0]
    bad, _ = oracle.fps_replay(U, wrong, 1e-9, _lib=lib)
    assert bad == 3, bad
    # exact ties: both orders are acceptable
    E = np.eye(4)
    assert oracle.fps_replay(E, [0, 3, 1, 2], 1e-9, _lib=lib)[0] == -1


ALL_PINS = [pin_closed_forms, pin_logits_matmul, pin_softmax, pin_score_head_composition,
            pin_topk_full_sort, pin_compact_bytes, pin_fps_bruteforce, pin_fps_special_sets,
            pin_fps_replay]


# --------------------------------------------------------------------------
# Pins of the composition (oracle/__init__.py): each takes the oracle module
# itself (or a mutated copy of it, see test_oracle_mutants.py).
# --------------------------------------------------------------------------
def pin_step_golden(mod):
    """The hand-derived whole step of tests/golden/closed_forms.json: Continual
    FPS over [stored beacons; window] (Fig. 7), then scores from the recent
    query and the updated beacons (Fig. 5(b)), max aggregation and top-K
    (Fig. 5(c)), compaction (Fig. 5(a))."""
    for case in _golden()["step_cases"]:
        b = np.array(case["beacons"])
        w = np.array(case["window"])
        k = np.array(case["k"])
        v = np.array(case["v"])
        recent = mod.newest_rows(w, case["R"])
        for K, want in case["topk"].items():
            r = mod.compress_head(k, v, recent, b, case["n_beacons"], w, case["M"], int(K),
                                  scale=case["scale"])
            assert [p.tolist() for p in r["picks"]] == case["picks"], (case["name"], r["picks"])
            np.testing.assert_array_equal(r["beacons"], np.array(case["new_beacons"]))
            assert r["n_beacons"] == case["M"]
            np.testing.assert_allclose(r["scores"], case["s"], rtol=0, atol=1e-12,
                                       err_msg=case["name"])
            assert r["idx"].tolist() == want, (case["name"], K, r["idx"].tolist())
            np.testing.assert_array_equal(r["k"], k[want])
            np.testing.assert_array_equal(r["v"], v[want])


def pin_update_beacons_composition(mod):
    """Continual FPS over the stored beacons (slots past n_beacons ignored),
    then the window oldest first, against brute-force greedy on that union."""
    rng = np.random.default_rng(9)
    for trial in range(40):
        d = int(rng.integers(2, 5))
        M = int(rng.integers(1, 6))
        nb = int(rng.integers(0, M + 1))
        W = int(rng.integers(0 if nb else 1, 5))
        beacons = rng.standard_normal((M, d))
        beacons[nb:] = rng.standard_normal((M - nb, d)) * 50.0   # stale slots
        window = rng.standard_normal((W, d))
        if trial % 4 == 0 and W and nb:
            window[W - 1] = beacons[0] * 2.0   # a query in a beacon's direction
        newb, sel = mod.update_beacons_head(beacons, nb, window, M)
        U = np.concatenate([beacons[:nb], window])
        want = _fps_brute(U, M)
        assert sel.tolist() == want, (trial, sel.tolist(), want)
        np.testing.assert_array_equal(newb, U[want])


def pin_ring_rows(mod):
    """The newest n rows of a ring buffer, oldest first, against a history
    written into the ring one row at a time."""
    rng = np.random.default_rng(10)
    for cap, T, n in [(8, 5, 3), (8, 8, 8), (8, 13, 5), (5, 27, 5), (6, 6, 0), (7, 100, 1)]:
        hist = rng.standard_normal((T, 3))
        ring = np.zeros((cap, 3))
        head = 0
        for t in range(T):
            ring[head] = hist[t]
            head = (head + 1) % cap
        got = mod.ring_rows(ring, head, n)
        want = np.stack([hist[t] for t in range(T - n, T)]) if n else np.zeros((0, 3))
        np.testing.assert_array_equal(got, want)
        np.testing.assert_array_equal(mod.newest_rows(hist, n), want)


COMPOSITION_PINS = [pin_step_golden, pin_update_beacons_composition, pin_ring_rows]
