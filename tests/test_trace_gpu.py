"""The Qwen3-4B-shaped continual decoding trace (32768 steps, compression every
4096 steps to K = 4096 with Continual FPS into M = 64 beacons), first layer,
against an independent float64 oracle trace.

Each compression event is compared while the GPU's state (kept positions and
beacons) equals the oracle's.  A legal near-tie (an FPS pick within 1e-5 of
the farthest distance, or a top-K swap within the score tolerance of the
budget boundary) lets the two traces part; from then on that head's events
are checked structurally only (kept count, ascending positions, byte-exact
compaction of the rows the GPU chose, beacons drawn from the union).
"""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
from parity_helpers import check_fps, check_topk, f64, picks_from_rows, raw

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.mark.parametrize("in_place", [False, True])
def test_qwen3_4b_trace_follows_the_oracle_trace(in_place):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from kv_cache_compression_bkv_b200 import synth
    from kv_cache_compression_bkv_b200.trace import TraceRun

    tr = synth.TRACES["qwen3_4b_trace"]
    run = TraceRun(tr, seed=0, device=torch.device("cuda:0"), layers=1, in_place=in_place)
    G, Hkv, I, K, M, R = tr.group, tr.n_kv_heads, tr.interval, tr.K, tr.M, tr.R
    keys_raw = raw(run.keys[0])          # [Hkv, steps, d]
    vals_raw = raw(run.values[0])
    keys64 = f64(run.keys[0])
    vals64 = f64(run.values[0])
    q64 = f64(run.queries[0])            # [Hq, steps, d]
    q_raw = raw(run.queries[0])
    state = {h: dict(gpu_pos=np.zeros(0, np.int64), ora_pos=np.zeros(0, np.int64),
                     ora_beac=np.zeros((G, 0, tr.head_dim)), diverged=False) for h in range(Hkv)}
    counts = dict(exact=0, near_tie=0, structural=0)

    def union_rows(h, gq, n_b, beacon_raw, t0):
        qh = h * G + gq
        return np.concatenate([beacon_raw[qh, :n_b], q_raw[qh, t0:t0 + I]])

    def on_event(run, ev):
        t1 = ev.step
        t0 = t1 - I
        idx = run.last_idx[0].cpu().numpy().astype(np.int64)         # [Hkv, kept]
        kc = raw(run.cache[run.cur][0][0])
        vc = raw(run.cache[run.cur][1][0])
        bout = raw(run.beacons[run.cur][0])
        bprev = raw(run.beacons[1 - run.cur][0])
        chunk = np.arange(t0, t1)

        def one_head(h):
            st = state[h]
            pre_gpu = np.concatenate([st["gpu_pos"], chunk])
            assert idx[h].shape == (min(K, ev.L),)
            assert np.all(np.diff(idx[h]) > 0)
            new_gpu = pre_gpu[idx[h]]
            # compaction: the kept rows are byte copies of the trace's rows
            assert np.array_equal(kc[h, :len(new_gpu)], keys_raw[h, new_gpu])
            assert np.array_equal(vc[h, :len(new_gpu)], vals_raw[h, new_gpu])
            picks = [picks_from_rows(union_rows(h, gq, ev.n_beacons_in, bprev, t0),
                                     bout[h * G + gq, :ev.n_beacons_out]) for gq in range(G)]
            result = "structural"
            if not st["diverged"]:
                pre_ora = np.concatenate([st["ora_pos"], chunk])
                assert np.array_equal(pre_ora, pre_gpu)
                recent = np.stack([q64[h * G + gq, t1 - R:t1] for gq in range(G)])
                window = np.stack([q64[h * G + gq, t0:t1] for gq in range(G)])
                beac = np.zeros((G, M, tr.head_dim))
                beac[:, :st["ora_beac"].shape[1]] = st["ora_beac"]
                ref = oracle.compress_head(keys64[h, pre_ora], vals64[h, pre_ora], recent, beac,
                                           ev.n_beacons_in, window, M, K)
                exact = True
                for gq in range(G):
                    U = np.concatenate([beac[gq, :ev.n_beacons_in], window[gq]])
                    exact &= check_fps(U, picks[gq], M, f"event {ev.index} head {h} q{gq}")
                if exact:
                    n_diff = check_topk(idx[h], ref["scores"], K, f"event {ev.index} head {h}")
                    exact = n_diff == 0
                result = "exact" if exact else "near_tie"
                st["diverged"] = not exact
                st["ora_pos"] = pre_ora[ref["idx"]]
                st["ora_beac"] = ref["beacons"]
            st["gpu_pos"] = new_gpu
            return result

        with ThreadPoolExecutor(max_workers=Hkv) as ex:
            for r in ex.map(one_head, range(Hkv)):
                counts[r] += 1

    events = run.run(on_event)
    assert len(events) == tr.steps // I
    assert events[0].L == I and events[0].new_len == min(K, I) and events[0].n_beacons_out == M
    assert all(e.L == K + I and e.new_len == K for e in events[1:])
    total = sum(counts.values())
    assert total == Hkv * len(events)
    # most (event, head) pairs are compared exactly against the oracle
    assert counts["exact"] >= total // 2, counts
