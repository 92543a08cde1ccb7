"""Comparators between the CUDA path and the float64 oracle.

Tolerances (float inputs rounded to bf16/f32 as given, f32 accumulation on the
GPU, float64 in the oracle):
  * scores s_j: |s_gpu - s_ref| <= 1e-6 + 1e-3 |s_ref|;
  * kept positions: exactly min(K, L) distinct, ascending; any position in
    one set and not the other must have an oracle score within that same
    tolerance of the oracle's K-th largest score (a near-tie at the budget
    boundary, where either choice is correct);
  * compaction: byte-exact copies of the rows the GPU chose;
  * FPS: the GPU's picks replayed through the oracle must each be within 1e-5
    (cosine distance) of the oracle's farthest point at that step.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

S_RTOL, S_ATOL = 1e-3, 1e-6
FPS_TOL = 1e-5


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def raw(t: torch.Tensor) -> np.ndarray:
    """Bit pattern of a tensor as unsigned integers of the same width."""
    t = t.detach().cpu().contiguous()
    return t.view({2: torch.int16, 4: torch.int32}[t.element_size()]).numpy()


def check_scores(s_got: np.ndarray, s_ref: np.ndarray, what: str = "scores") -> float:
    err = np.abs(s_got - s_ref)
    bad = err > S_ATOL + S_RTOL * np.abs(s_ref)
    if bad.any():
        j = int(np.argmax(bad))
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; "
                             f"first j={j} got={s_got[j]!r} ref={s_ref[j]!r}")
    return float(np.max(err / (S_ATOL + np.abs(s_ref))))


def check_topk(idx_got: np.ndarray, s_ref: np.ndarray, K: int, what: str = "top-K") -> int:
    """Returns how many positions differ from the oracle's set (all near-ties)."""
    L = s_ref.shape[0]
    keep = min(K, L)
    idx_got = np.asarray(idx_got).astype(np.int64)
    assert idx_got.shape == (keep,), (what, idx_got.shape, keep)
    assert np.all(np.diff(idx_got) > 0), f"{what}: not strictly ascending"
    assert idx_got.min() >= 0 and idx_got.max() < L, f"{what}: out of range"
    ref = oracle.select_topk(s_ref, K)
    diff = set(idx_got.tolist()) ^ set(ref.tolist())
    if diff:
        theta = np.sort(s_ref)[::-1][keep - 1]
        band = S_ATOL + S_RTOL * theta
        far = [j for j in diff if abs(s_ref[j] - theta) > band]
        assert not far, f"{what}: {len(far)} differing positions are not near-ties, e.g. {far[:5]}"
    return len(diff)


def check_compaction(dst_rows: np.ndarray, src_rows: np.ndarray, idx: np.ndarray,
                     what: str = "compaction") -> None:
    assert np.array_equal(dst_rows, src_rows[np.asarray(idx, dtype=np.int64)]), what


def picks_from_rows(U_raw: np.ndarray, out_raw: np.ndarray) -> list[int]:
    """Union indices of the GPU's output beacon rows (matched by bit pattern)."""
    where: dict[bytes, list[int]] = {}
    for i in range(U_raw.shape[0]):
        where.setdefault(U_raw[i].tobytes(), []).append(i)
    used: set[int] = set()
    picks = []
    for r in range(out_raw.shape[0]):
        cands = [i for i in where.get(out_raw[r].tobytes(), []) if i not in used]
        assert cands, f"output beacon {r} is not a row of the union"
        picks.append(cands[0])
        used.add(cands[0])
    return picks


def check_fps(U64: np.ndarray, picks: list[int], M: int, what: str = "FPS") -> bool:
    """True when the picks equal the oracle's exactly; False for accepted near-ties."""
    n = U64.shape[0]
    assert len(picks) == min(M, n), (what, len(picks), min(M, n))
    ref = oracle.fps(U64, M).tolist()
    if picks == ref:
        return True
    bad, gap = oracle.fps_replay(U64, picks, FPS_TOL)
    assert bad == -1, f"{what}: pick {bad} is {gap:.3g} short of the farthest point"
    return False
