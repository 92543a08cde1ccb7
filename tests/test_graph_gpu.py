"""The whole compression step captured once in a CUDA graph and replayed: the
step makes no host synchronisation, allocation or query, so a serving loop
can capture it (its five kernels and the FPS head counter's reset) and replay
it every interval.  The replays must give the eager step's bytes, also after
the inputs change in place."""
import pytest
import torch

from parity_helpers import raw

pytestmark = pytest.mark.gpu


def test_compress_step_replays_in_a_cuda_graph():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from kv_cache_compression_bkv_b200 import bkv, synth

    dev = torch.device("cuda:0")
    wl = synth.Workload(name="graph", n_layers=2, n_q_heads=4, n_kv_heads=2, head_dim=128,
                        L=1500, R=8, M=16, K=400, W=200, dtype="bf16", n_clusters=4,
                        q_noise=0.5, n_plan=16, plan_span=64, n_outlier_channels=2,
                        n_beacons_in=8, capacity=1600)
    inp = synth.make_step_inputs(wl, seed=21)
    g = bkv.geometry_of(inp.k, wl.n_q_heads)
    dst = bkv.Geometry(g.n_layers, g.n_q_heads, g.n_kv_heads, g.head_dim, wl.K, g.dtype)
    t = {n: getattr(inp, n).to(dev) for n in ("k", "v", "recent", "beacons", "window")}
    out = dict(bout=torch.zeros_like(t["beacons"]),
               kd=torch.empty(wl.n_layers, wl.n_kv_heads, wl.K, wl.head_dim, dtype=inp.k.dtype,
                              device=dev),
               scores=torch.empty(wl.n_layers, wl.n_kv_heads, wl.L, device=dev),
               idx=torch.empty(wl.n_layers, wl.n_kv_heads, wl.K, dtype=torch.int32, device=dev))
    out["vd"] = torch.empty_like(out["kd"])
    ws = torch.empty(bkv.bkv_workspace_size(g, wl.L, wl.R, wl.M, wl.W, wl.K), dtype=torch.uint8,
                     device=dev)

    def step():
        bkv.bkv_compress_step(g, t["k"], t["v"], wl.L, wl.K, t["recent"], wl.R, t["beacons"],
                              wl.beacons_in, wl.M, t["window"], wl.W, out["bout"], 0.0, dst,
                              out["kd"], out["vd"], out["scores"], out["idx"], ws)

    def snapshot():
        torch.cuda.synchronize()
        return {n: raw(x.cpu()) for n, x in out.items()}

    step()  # eager: also sets the kernels' attributes once
    eager = snapshot()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for x in out.values():
        x.zero_()
    graph.replay()
    replayed = snapshot()
    for n in out:
        assert (replayed[n] == eager[n]).all(), n

    # new inputs in the captured buffers: the replay follows them
    gen = torch.Generator().manual_seed(5)
    for n in ("k", "v", "window"):
        t[n].copy_((torch.randn(t[n].shape, generator=gen)).to(t[n].dtype))
    graph.replay()
    replayed = snapshot()
    step()
    eager = snapshot()
    for n in out:
        assert (replayed[n] == eager[n]).all(), n
    assert bkv.bkv_read_device_status()[0] == 0
    del graph
