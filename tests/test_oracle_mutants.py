"""The pins bite: plausible mistakes planted in a copy of the oracle fail them.

Each mutant is a one-line textual change to a temporary copy of
oracle/bkv_oracle.c (a dropped term, a flipped sign or comparison, a wrong
index, a lost sort), compiled on the CPU, or of the composition in
oracle/__init__.py (the order of the FPS union, the stale beacon slots, the
beacons used for scoring, which end of the history the recent queries come
from), imported from a temporary directory.  The real oracle is untouched.
"""
import importlib.util
import os
import shutil
import subprocess
import sys

import pytest

import oracle
from oracle_pins import ALL_PINS, COMPOSITION_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "bkv_oracle.c")

MUTANTS = {
    "logits_drop_scale": ("x[o * L + j] = scale * acc;", "x[o * L + j] = acc;"),
    "normaliser_drop_max": ("c[o] = m + log(sum);", "c[o] = log(sum);"),
    "normaliser_sign": ("sum += exp(row[j] - m);", "sum += exp(m - row[j]);"),
    "aggregate_min": ("if (p > best) best = p;", "if (p < best || o == 0) best = p;"),
    "aggregate_row_index": ("double p = exp(x[o * L + j] - c[o]);", "double p = exp(x[o * L + j] - c[0]);"),
    "mean_drop_divide": ("s[j] = sum / (double)n_obs;", "s[j] = sum;"),
    "mean_divide_by_keys": ("s[j] = sum / (double)n_obs;", "s[j] = sum / (double)L;"),
    "mean_row_index": ("for (int64_t o = 0; o < n_obs; ++o) sum += exp(x[o * L + j] - c[o]);",
                       "for (int64_t o = 0; o < n_obs; ++o) sum += exp(x[o * L + j] - c[0]);"),
    "topk_tie_high": ("return (x->j < y->j) ? -1 : (x->j > y->j);", "return (x->j > y->j) ? -1 : (x->j < y->j);"),
    "topk_no_ascending_sort": ("qsort(idx, (size_t)keep, sizeof(int32_t), oracle_cmp_int_asc);", ""),
    "topk_ascending_scores": ("if (x->s > y->s) return -1;\n  if (x->s < y->s) return 1;", "if (x->s < y->s) return -1;\n  if (x->s > y->s) return 1;"),
    "compact_wrong_row": ("memcpy(dst + i * row_bytes, src + (int64_t)idx[i] * row_bytes,", "memcpy(dst + i * row_bytes, src + i * row_bytes,"),
    "fps_running_max": ("if (db < dist[i]) dist[i] = db;", "if (db > dist[i]) dist[i] = db;"),
    "fps_tie_high": ("if (best < 0 || dist[i] > dist[best]) best = i;", "if (best < 0 || dist[i] >= dist[best]) best = i;"),
    "fps_distance_to_seed": ("double db = oracle_cosine_distance(d, U + i * d, nrm[i], U + best * d,\n                                         nrm[best]);",
                             "double db = oracle_cosine_distance(d, U + i * d, nrm[i], U,\n                                         nrm[0]);"),
    "fps_no_normalise": ("double dist = 1.0 - dot / (na * nb);", "double dist = 1.0 - dot;"),
    "fps_no_clamp": ("if (dist < 0.0) dist = 0.0;", ""),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_fails_a_pin(name, tmp_path):
    before, after = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(before) == 1, f"mutation site for {name} not unique/present"
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(before, after))
    so = str(tmp_path / "libmutant.so")
    subprocess.run(["gcc", "-O1", "-shared", "-fPIC", str(src), "-o", so, "-lm"], check=True)
    lib = oracle.load_variant(so)
    failed = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"


PY_SRC = os.path.join(os.path.dirname(oracle.__file__), "__init__.py")

PY_MUTANTS = {
    # Fig. 7: the union lists the current beacons first, then the window
    "union_window_first": ("U = np.concatenate([b, w], axis=0) if w.size else b",
                           "U = np.concatenate([w, b], axis=0) if w.size else b"),
    # only the first n_beacons slots hold beacons
    "union_all_slots": ("b = np.asarray(beacons)[:n_beacons]", "b = np.asarray(beacons)"),
    # scoring uses the beacons after the update, not the stored ones
    "score_old_beacons": ("s, c = score_head(k_rows, recent, beacons_used, n_used, scale,",
                          "s, c = score_head(k_rows, recent, beacons, n_beacons, scale,"),
    # the recent queries are the newest rows of the history
    "recent_oldest_rows": ("return rows[..., T - n:T, :]", "return rows[..., 0:n, :]"),
    # the observation set holds every query head's recent rows
    "obs_drops_recent": ("        parts.append(recent[g])\n", ""),
    # a ring's newest row sits just before the write position
    "ring_off_by_one": ("idx = [(head - n + i) % cap for i in range(n)]",
                        "idx = [(head - n + i + 1) % cap for i in range(n)]"),
}


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_composition_mutant_fails_a_pin(name, tmp_path):
    before, after = PY_MUTANTS[name]
    text = open(PY_SRC).read()
    assert text.count(before) == 1, f"mutation site for {name} not unique/present"
    pkg = tmp_path / f"oracle_mut_{name}"
    pkg.mkdir()
    (pkg / "__init__.py").write_text(text.replace(before, after))
    shutil.copy(SRC, pkg / "bkv_oracle.c")
    spec = importlib.util.spec_from_file_location(pkg.name, pkg / "__init__.py",
                                                  submodule_search_locations=[str(pkg)])
    mod = importlib.util.module_from_spec(spec)
    sys.modules[pkg.name] = mod
    try:
        spec.loader.exec_module(mod)
        failed = []
        for pin in COMPOSITION_PINS:
            try:
                pin(mod)
            except AssertionError:
                failed.append(pin.__name__)
    finally:
        sys.modules.pop(pkg.name, None)
    assert failed, f"composition mutant {name} passed every pin"
