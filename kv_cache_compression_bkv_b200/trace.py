"""A continual decoding trace driven through the C ABI.

The caller's side of BeaconKV's periodic compression: the cache grows by one
row per decode step, and every `interval` steps one bkv_compress_step call
updates the beacons by Continual FPS over the queries of that interval (the
window), scores the cache with the recent and beacon queries, keeps the
budget K and compacts into the other of two cache buffers.  The decode step
itself is not simulated: the keys, values and queries of each interval come
from the seeded trace generator (synth.trace_*) and are appended in one copy.
With in_place the step compacts into the cache it scored (one cache buffer).

With ring_cap set, the decode loop keeps the queries the way a serving loop
would: every decode step appends its query of every (layer, query head) to a
device ring of ring_cap slots (query t in slot t % ring_cap), and the step
reads the recent queries and the window in place from that ring (the window
wraps around the ring's end whenever ring_cap is not a multiple of the
interval); no window or recent-query buffer is assembled.

Checkpoint and resume: between two compression events the whole state of the
run is the current cache rows, the current beacons, the query ring (if any),
the event log and a few counters; `checkpoint(path)` writes them with
torch.save and `TraceRun.resume(path, device)` rebuilds the run (the trace's
keys, values and queries are regenerated from its seed) and continues with
the next event, with results identical to an uninterrupted run.
"""
from __future__ import annotations

from dataclasses import asdict, dataclass, field

import torch

from . import bkv, synth


@dataclass
class TraceEvent:
    index: int          # compression event number (0-based)
    step: int           # decode steps generated so far
    L: int              # cache rows scored
    new_len: int        # rows kept
    n_beacons_in: int
    n_beacons_out: int
    ms: float           # device time of the compress_step call


@dataclass
class TraceRun:
    tr: synth.Trace
    seed: int
    device: torch.device
    layers: int | None = None      # use only the first `layers` layers
    in_place: bool = False         # compact into the cache itself (one cache buffer)
    ring_cap: int | None = None    # keep the queries in a decode-side ring of this many slots
    events: list[TraceEvent] = field(default_factory=list)

    def __post_init__(self):
        tr = self.tr
        self.Ly = self.layers or tr.n_layers
        Ly, Hq, Hkv, d, dt = self.Ly, tr.n_q_heads, tr.n_kv_heads, tr.head_dim, tr.torch_dtype
        self.cap = tr.K + tr.interval
        self.keys = torch.empty(Ly, Hkv, tr.steps, d, dtype=dt)
        self.values = torch.empty(Ly, Hkv, tr.steps, d, dtype=dt)
        self.queries = torch.empty(Ly, Hq, tr.steps, d, dtype=dt)
        for l in range(Ly):
            for h in range(Hkv):
                k, v = synth.trace_keys_values(tr, self.seed, l, h)
                self.keys[l, h] = k.to(dt)
                self.values[l, h] = v.to(dt)
            for q in range(Hq):
                self.queries[l, q] = synth.trace_queries(tr, self.seed, l, q).to(dt)
        dev = self.device
        self.cache = [(torch.zeros(Ly, Hkv, self.cap, d, dtype=dt, device=dev),
                       torch.zeros(Ly, Hkv, self.cap, d, dtype=dt, device=dev))
                      for _ in range(1 if self.in_place else 2)]
        if self.in_place:  # source and destination are the same buffers
            self.cache.append(self.cache[0])
        self.beacons = [torch.zeros(Ly, Hq, tr.M, d, dtype=dt, device=dev) for _ in range(2)]
        if self.ring_cap is not None:
            if self.ring_cap < tr.interval:
                raise ValueError("the ring must hold a whole interval of queries")
            self.ring = torch.zeros(Ly, Hq, self.ring_cap, d, dtype=dt, device=dev)
            self.window = self.recent = None
        else:
            self.ring = None
            self.window = torch.empty(Ly, Hq, tr.interval, d, dtype=dt, device=dev)
            self.recent = torch.empty(Ly, Hq, tr.R, d, dtype=dt, device=dev)
        self.idx_flat = torch.empty(Ly * Hkv * tr.K, dtype=torch.int32, device=dev)
        self.last_idx = None    # kept positions of the last event, [Ly][Hkv][kept]
        self.geom = bkv.Geometry(Ly, Hq, Hkv, d, self.cap, dt)
        self.ws = torch.empty(bkv.bkv_workspace_size(self.geom, self.cap, tr.R, tr.M,
                                                     tr.interval, tr.K),
                              dtype=torch.uint8, device=dev)
        self.cur = 0            # which cache / beacon buffer holds the state
        self.L = 0              # cache rows
        self.n_beacons = 0
        self.next_event = 0     # the event the next run() starts with

    CHECKPOINT_VERSION = 1

    def checkpoint(self, path) -> None:
        """Write the state between two events (call it between run() calls)."""
        kc, vc = self.cache[self.cur]
        state = {
            "version": self.CHECKPOINT_VERSION,
            "trace": asdict(self.tr),
            "seed": self.seed,
            "layers": self.Ly,
            "in_place": self.in_place,
            "ring_cap": self.ring_cap,
            "next_event": self.next_event,
            "L": self.L,
            "n_beacons": self.n_beacons,
            "k": kc[:, :, :self.L].cpu(),
            "v": vc[:, :, :self.L].cpu(),
            "beacons": self.beacons[self.cur][:, :, :self.n_beacons].cpu(),
            "ring": None if self.ring is None else self.ring.cpu(),
            "events": [asdict(e) for e in self.events],
        }
        torch.save(state, path)

    @classmethod
    def resume(cls, path, device: torch.device) -> "TraceRun":
        """A run in the state `checkpoint` wrote, ready to continue."""
        state = torch.load(path, map_location="cpu", weights_only=True)
        if state.get("version") != cls.CHECKPOINT_VERSION:
            raise ValueError(f"unsupported trace checkpoint version {state.get('version')}")
        run = cls(synth.Trace(**state["trace"]), seed=state["seed"], device=device,
                  layers=state["layers"], in_place=state["in_place"],
                  ring_cap=state["ring_cap"])
        L, nb = state["L"], state["n_beacons"]
        kc, vc = run.cache[run.cur]
        kc[:, :, :L].copy_(state["k"])
        vc[:, :, :L].copy_(state["v"])
        run.beacons[run.cur][:, :, :nb].copy_(state["beacons"])
        if run.ring is not None:
            run.ring.copy_(state["ring"])
        run.L, run.n_beacons, run.next_event = L, nb, state["next_event"]
        run.events = [TraceEvent(**e) for e in state["events"]]
        return run

    def run(self, on_event=None, stop_after: int | None = None):
        """Run the trace from the next event to the end (or through event
        stop_after); on_event(run, event) sees the state after each
        compression (the current buffers; run.last_idx = kept positions)."""
        tr = self.tr
        stream = torch.cuda.current_stream(self.device)
        for e, t0 in enumerate(range(0, tr.steps, tr.interval)):
            if e < self.next_event:
                continue
            if stop_after is not None and e > stop_after:
                break
            t1 = t0 + tr.interval
            kc, vc = self.cache[self.cur]
            kc[:, :, self.L:self.L + tr.interval].copy_(self.keys[:, :, t0:t1])
            vc[:, :, self.L:self.L + tr.interval].copy_(self.values[:, :, t0:t1])
            if self.ring is not None:
                # each decode step appends its query to the ring
                q = self.queries[:, :, t0:t1].to(self.device)
                for t in range(t0, t1):
                    self.ring[:, :, t % self.ring_cap].copy_(q[:, :, t - t0])
            else:
                self.window.copy_(self.queries[:, :, t0:t1])
                self.recent.copy_(self.queries[:, :, t1 - tr.R:t1])
            L = self.L + tr.interval
            kd, vd = self.cache[1 - self.cur]
            bin_, bout = self.beacons[self.cur], self.beacons[1 - self.cur]
            keep = min(tr.K, L)
            idx = self.idx_flat[:self.Ly * tr.n_kv_heads * keep].view(self.Ly, tr.n_kv_heads, keep)
            ev0 = torch.cuda.Event(enable_timing=True)
            ev1 = torch.cuda.Event(enable_timing=True)
            ev0.record(stream)
            nb, nl = bkv.bkv_compress_step(
                self.geom, kc, vc, L, tr.K, self.recent, tr.R,
                bin_ if self.n_beacons else None, self.n_beacons, tr.M, self.window,
                tr.interval, bout, 0.0, self.geom, kd, vd, None, idx, self.ws, stream,
                query_ring=self.ring, ring_pos=t1)
            ev1.record(stream)
            torch.cuda.synchronize(self.device)
            event = TraceEvent(e, t1, L, nl, self.n_beacons, nb, ev0.elapsed_time(ev1))
            self.events.append(event)
            self.cur = 1 - self.cur
            self.L, self.n_beacons = nl, nb
            self.last_idx = idx
            self.next_event = e + 1
            if on_event is not None:
                on_event(self, event)
        return self.events
