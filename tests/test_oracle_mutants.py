"""The pins bite: plausible mistakes planted in a copy of the oracle fail them.

Each mutant is a one-line textual change to a temporary copy of
oracle/bkv_oracle.c (a dropped term, a flipped sign or comparison, a wrong
index, a lost sort), compiled on the CPU.  The real oracle is untouched.
"""
import os
import shutil
import subprocess

import pytest

import oracle
from oracle_pins import ALL_PINS

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
