"""bkv_score_noalloc: scoring on the library's built-in scratch array.

It exists for callers that cannot allocate device memory where they score
(for example code inside another runtime's execute callback that only hands
over its tensors, or a loop that must not allocate after start-up because a
pool allocator holds the device's memory).  Its results must equal those of
bkv_score with a caller workspace.  Two calls in a row, of different shapes and
dtypes, check that what the first call leaves in the shared array does not
leak into the second.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

RTOL, ATOL = 1e-3, 1e-6   # the score tolerance of the parity tests


def _case(synth, **kw):
    base = dict(name="noalloc", n_layers=2, n_q_heads=8, n_kv_heads=2, head_dim=128, L=900,
                R=24, M=40, K=100, W=0, dtype="bf16", n_clusters=4, q_noise=0.5, n_plan=16,
                plan_span=64, n_outlier_channels=2, n_beacons_in=40, capacity=1000)
    base.update(kw)
    return synth.Workload(**base)


def _both_paths(bkv, synth, wl, seed, dev):
    inp = synth.make_step_inputs(wl, seed=seed)
    g = bkv.geometry_of(inp.k, wl.n_q_heads)
    k, rq, bq = inp.k.to(dev), inp.recent.to(dev), inp.beacons.to(dev)
    ws = torch.empty(bkv.bkv_workspace_size(g, wl.L, wl.R, wl.M, 0, wl.K), dtype=torch.uint8,
                     device=dev)
    ref = torch.full((wl.n_layers, wl.n_kv_heads, wl.L), -7.0, device=dev)
    got = torch.full_like(ref, -7.0)
    bkv.bkv_score(g, k, wl.L, rq, wl.R, bq, wl.beacons_in, wl.M, 0.0, ref, ws)
    bkv.bkv_score_noalloc(g, k, wl.L, rq, wl.R, bq, wl.beacons_in, wl.M, 0.0, got)
    torch.cuda.synchronize()
    assert bkv.bkv_read_device_status()[0] == 0
    return ref.double().cpu().numpy(), got.double().cpu().numpy()


def test_noalloc_matches_workspace_path_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from kv_cache_compression_bkv_b200 import bkv, synth
    dev = torch.device("cuda:0")
    # first call: bf16, two observation groups (640 rows), ragged key tail
    wl1 = _case(synth, R=40, n_beacons_in=40)
    ref1, got1 = _both_paths(bkv, synth, wl1, seed=21, dev=dev)
    # second call right after: another shape and dtype on the same array
    wl2 = synth.WORKLOADS["tiny"].replace(W=0)
    ref2, got2 = _both_paths(bkv, synth, wl2, seed=22, dev=dev)
    for ref, got in ((ref1, got1), (ref2, got2)):
        # the same kernels on the same inputs: the results are identical, so
        # any leftover of the previous call in the shared array would show
        assert np.array_equal(got, ref)
        assert np.all(np.abs(got - ref) <= ATOL + RTOL * np.abs(ref))
        assert np.all(got > 0) and np.all(got <= 1.0 + 1e-6)


def test_noalloc_rejects_problems_beyond_the_array():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from kv_cache_compression_bkv_b200 import bkv
    dev = torch.device("cuda:0")
    # 2 layers x 8 KV heads x 600000 keys of partial maxima alone exceed 32 MiB
    Ly, Hkv, L = 2, 8, 600_000
    g = bkv.Geometry(Ly, 16, Hkv, 128, L, torch.bfloat16)
    assert 4 * Ly * Hkv * L > bkv.SCORE_NOALLOC_SCRATCH_BYTES
    k = torch.zeros(Ly, Hkv, L, 128, dtype=torch.bfloat16, device=dev)
    rq = torch.zeros(Ly, 16, 4, 128, dtype=torch.bfloat16, device=dev)
    out = torch.full((Ly, Hkv, L), -7.0, device=dev)
    with pytest.raises(bkv.BkvError) as e:
        bkv.bkv_score_noalloc(g, k, L, rq, 4, None, 0, 0, 0.0, out)
    assert e.value.status == 3  # BKV_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((out == -7.0).all())  # nothing was launched
