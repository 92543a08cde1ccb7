"""Device-side failure paths, made to happen without faulting or hanging the
GPU: a bounded wait that nothing satisfies gives up after its limit, records
BKV_ERR_TIMEOUT with its location tag, the kernel exits normally, and the
next calls run clean."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch.device("cuda:0")


def test_bounded_wait_gives_up_and_reports(dev):
    from kv_cache_compression_bkv_b200 import bkv, synth
    assert bkv.bkv_read_device_status()[0] == 0          # start clean
    outcome = torch.full((1,), 7, dtype=torch.int32, device=dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    bkv.bkv_selftest_wait_timeout(2_000_000, outcome)    # a 2 ms limit
    ev1.record()
    torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1)
    assert 1.5 <= ms < 200.0, ms                         # it waited about its limit, then ended
    assert int(outcome.item()) == 0                      # the wait gave up
    st, where = bkv.bkv_read_device_status()
    assert (st, where) == (5, 901)                       # BKV_ERR_TIMEOUT at the self-test's wait
    assert bkv.bkv_read_device_status()[0] == 0          # reading cleared it
    # the context is fine: a real call runs and reports nothing
    wl = synth.Workload(name="after", n_layers=1, n_q_heads=4, n_kv_heads=1, head_dim=128,
                        L=300, R=8, M=8, K=50, W=0, dtype="bf16", n_clusters=2, q_noise=0.5,
                        n_plan=4, plan_span=16)
    inp = synth.make_step_inputs(wl, seed=1)
    g = bkv.geometry_of(inp.k, wl.n_q_heads)
    ws = torch.empty(bkv.bkv_workspace_size(g, wl.L, wl.R, wl.M, 0, wl.K), dtype=torch.uint8,
                     device=dev)
    scores = torch.empty(1, 1, wl.L, device=dev)
    bkv.bkv_score(g, inp.k.to(dev), wl.L, inp.recent.to(dev), wl.R, inp.beacons.to(dev), wl.M,
                  wl.M, 0.0, scores, ws)
    torch.cuda.synchronize()
    assert bkv.bkv_read_device_status()[0] == 0
    assert bool(torch.isfinite(scores).all()) and bool((scores > 0).all())
