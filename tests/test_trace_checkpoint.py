"""Checkpoint and resume of the trace driver (host side): the state written
between two compression events comes back exactly, and a checkpoint of
another format version is refused."""
import dataclasses

import pytest
import torch

from kv_cache_compression_bkv_b200 import synth
from kv_cache_compression_bkv_b200.trace import TraceEvent, TraceRun

TINY = synth.Trace(name="tiny_trace", n_layers=2, n_q_heads=4, n_kv_heads=2, head_dim=16,
                   steps=64, interval=16, K=24, R=4, M=8, n_clusters=2, plan_steps=32,
                   dtype="f32")


def _filled(ring_cap, in_place):
    run = TraceRun(TINY, seed=3, device=torch.device("cpu"), in_place=in_place,
                   ring_cap=ring_cap)
    gen = torch.Generator().manual_seed(9)
    run.cur = 1 if not in_place else 0
    run.L, run.n_beacons, run.next_event = 21, 6, 2
    kc, vc = run.cache[run.cur]
    kc.copy_(torch.randn(kc.shape, generator=gen))
    vc.copy_(torch.randn(vc.shape, generator=gen))
    run.beacons[run.cur].copy_(torch.randn(run.beacons[run.cur].shape, generator=gen))
    if run.ring is not None:
        run.ring.copy_(torch.randn(run.ring.shape, generator=gen))
    run.events = [TraceEvent(0, 16, 16, 16, 0, 8, 0.5), TraceEvent(1, 32, 32, 21, 8, 6, 0.25)]
    return run


@pytest.mark.parametrize("ring_cap,in_place", [(None, False), (20, False), (None, True)])
def test_checkpoint_round_trip(tmp_path, ring_cap, in_place):
    run = _filled(ring_cap, in_place)
    path = tmp_path / "trace.pt"
    run.checkpoint(path)
    back = TraceRun.resume(path, torch.device("cpu"))
    assert dataclasses.asdict(back.tr) == dataclasses.asdict(TINY)
    assert (back.seed, back.Ly, back.in_place, back.ring_cap) == (3, 2, in_place, ring_cap)
    assert (back.L, back.n_beacons, back.next_event) == (21, 6, 2)
    assert back.events == run.events
    kc, vc = run.cache[run.cur]
    bk, bv = back.cache[back.cur]
    assert torch.equal(bk[:, :, :21], kc[:, :, :21])
    assert torch.equal(bv[:, :, :21], vc[:, :, :21])
    assert torch.equal(back.beacons[back.cur][:, :, :6], run.beacons[run.cur][:, :, :6])
    if ring_cap is not None:
        assert torch.equal(back.ring, run.ring)
    # the regenerated trace is the same trace
    assert torch.equal(back.keys, run.keys) and torch.equal(back.queries, run.queries)


def test_checkpoint_of_another_version_is_refused(tmp_path):
    run = _filled(None, False)
    path = tmp_path / "trace.pt"
    run.checkpoint(path)
    state = torch.load(path, weights_only=True)
    state["version"] = 99
    torch.save(state, path)
    with pytest.raises(ValueError, match="version"):
        TraceRun.resume(path, torch.device("cpu"))
