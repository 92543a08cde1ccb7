"""The Qwen3-4B-shaped continual decoding trace (32768 steps, compression every
4096 steps to K = 4096 with Continual FPS into M = 64 beacons), first layer,
against the float64 oracle at every compression event.

Every (event, KV head) is compared, given the GPU's state before the event
(the rows its cache holds and its beacons): the GPU's FPS picks against the
oracle's (a legal near-tie -- every pick within 1e-5 of the farthest distance
-- is accepted by replay); the GPU's scores' top-K against the oracle's
scores of the head with the GPU's new beacons (near-ties at the budget
boundary accepted); and the compacted cache byte for byte against the
trace's rows.  Following the GPU's state keeps every event comparable even
after a near-tie has let the two diverge.
"""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
from parity_helpers import check_fps, check_topk, f64, picks_from_rows, raw

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.mark.parametrize("in_place,ring_cap", [(False, None), (True, None), (False, 5000)])
def test_qwen3_4b_trace_follows_the_oracle_trace(in_place, ring_cap):
    """ring_cap: the decode loop appends every query to a 5000-slot ring and
    the step reads the window and recent queries from it in place (the
    4096-query window wraps around the ring's end at most events)."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from kv_cache_compression_bkv_b200 import synth
    from kv_cache_compression_bkv_b200.trace import TraceRun

    tr = synth.TRACES["qwen3_4b_trace"]
    run = TraceRun(tr, seed=0, device=torch.device("cuda:0"), layers=1, in_place=in_place,
                   ring_cap=ring_cap)
    G, Hkv, I, K, M, R = tr.group, tr.n_kv_heads, tr.interval, tr.K, tr.M, tr.R
    keys_raw = raw(run.keys[0])          # [Hkv, steps, d]
    vals_raw = raw(run.values[0])
    keys64 = f64(run.keys[0])
    q64 = f64(run.queries[0])            # [Hq, steps, d]
    q_raw = raw(run.queries[0])
    gpu_pos = {h: np.zeros(0, np.int64) for h in range(Hkv)}   # trace steps the cache holds
    counts = dict(exact=0, near_tie=0)

    def on_event(run, ev):
        t1 = ev.step
        t0 = t1 - I
        idx = run.last_idx[0].cpu().numpy().astype(np.int64)         # [Hkv, kept]
        kc = raw(run.cache[run.cur][0][0])
        vc = raw(run.cache[run.cur][1][0])
        bout = raw(run.beacons[run.cur][0])
        bout64 = run.beacons[run.cur][0].double().cpu().numpy()
        bprev = raw(run.beacons[1 - run.cur][0])
        bprev64 = run.beacons[1 - run.cur][0].double().cpu().numpy()
        chunk = np.arange(t0, t1)

        def one_head(h):
            pre = np.concatenate([gpu_pos[h], chunk])
            assert idx[h].shape == (min(K, ev.L),)
            assert np.all(np.diff(idx[h]) > 0)
            new = pre[idx[h]]
            # compaction: the kept rows are byte copies of the trace's rows
            assert np.array_equal(kc[h, :len(new)], keys_raw[h, new])
            assert np.array_equal(vc[h, :len(new)], vals_raw[h, new])
            exact = True
            for gq in range(G):
                qh = h * G + gq
                U_raw = np.concatenate([bprev[qh, :ev.n_beacons_in], q_raw[qh, t0:t1]])
                U64 = np.concatenate([bprev64[qh, :ev.n_beacons_in], q64[qh, t0:t1]])
                picks = picks_from_rows(U_raw, bout[qh, :ev.n_beacons_out])
                exact &= check_fps(U64, picks, M, f"event {ev.index} head {h} q{gq}")
            # the recent queries are the newest R of the interval; the oracle
            # scores the cache the GPU held with the beacons the GPU chose
            recent = oracle.newest_rows(np.stack([q64[h * G + gq, t0:t1] for gq in range(G)]), R)
            s_ref, _ = oracle.score_head(keys64[h, pre], recent, bout64[h * G:(h + 1) * G],
                                         ev.n_beacons_out)
            check_topk(idx[h], s_ref, K, f"event {ev.index} head {h}")
            gpu_pos[h] = new
            return "exact" if exact else "near_tie"

        with ThreadPoolExecutor(max_workers=Hkv) as ex:
            for r in ex.map(one_head, range(Hkv)):
                counts[r] += 1

    events = run.run(on_event)
    assert len(events) == tr.steps // I
    assert events[0].L == I and events[0].new_len == min(K, I) and events[0].n_beacons_out == M
    assert all(e.L == K + I and e.new_len == K for e in events[1:])
    assert sum(counts.values()) == Hkv * len(events), counts
    print(f"trace ({'in place' if in_place else 'out of place'}"
          f"{', query ring' if ring_cap else ''}): {counts}")


def test_trace_resumes_from_a_checkpoint_bit_exactly(tmp_path):
    """Run the trace to its end; run it again to event 3, checkpoint, resume
    in a fresh run and finish: every later event keeps the same positions and
    the final cache and beacons are the same bytes."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from kv_cache_compression_bkv_b200 import synth
    from kv_cache_compression_bkv_b200.trace import TraceRun

    tr = synth.TRACES["qwen3_4b_trace"]
    dev = torch.device("cuda:0")

    def record(store):
        def on_event(run, ev):
            store[ev.index] = (ev.L, ev.new_len, ev.n_beacons_out, run.last_idx.cpu().clone())
        return on_event

    full = {}
    ref = TraceRun(tr, seed=0, device=dev, layers=1, ring_cap=5000)
    ref.run(record(full))
    first = TraceRun(tr, seed=0, device=dev, layers=1, ring_cap=5000)
    first.run(stop_after=3)
    path = tmp_path / "trace.pt"
    first.checkpoint(path)
    rest = {}
    resumed = TraceRun.resume(path, dev)
    assert resumed.next_event == 4 and len(resumed.events) == 4
    resumed.run(record(rest))
    assert sorted(rest) == [e for e in sorted(full) if e >= 4]
    for e, (L, n, nb, idx) in rest.items():
        fL, fn, fnb, fidx = full[e]
        assert (L, n, nb) == (fL, fn, fnb), e
        assert torch.equal(idx, fidx), e
    for a, b in zip(ref.cache[ref.cur], resumed.cache[resumed.cur]):
        assert torch.equal(a[:, :, :ref.L].view(torch.int16), b[:, :, :resumed.L].view(torch.int16))
    assert torch.equal(ref.beacons[ref.cur][:, :, :ref.n_beacons].view(torch.int16),
                       resumed.beacons[resumed.cur][:, :, :resumed.n_beacons].view(torch.int16))
