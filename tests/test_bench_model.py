"""The bench's work model at the 14B shape against the figures worked out by
hand from the workload (40 layers, 40/8 heads, d 128, L 32768, R 64, M 128,
K 6144, bf16): one contraction 2·960·32768·128·320 FLOP, the step's
algorithmic bytes, and one exp per logit."""
import pytest

import bench
from kv_cache_compression_bkv_b200 import synth


def test_work_model_14b():
    wl = synth.WORKLOADS["qwen3_14b"]
    wm = bench.work_model(wl)
    H, n_obs, L, d, K = 320, 5 * (64 + 128), 32768, 128, 6144
    assert wm["step_flop"] == pytest.approx(2 * n_obs * L * d * H)
    assert wm["step_flop"] == pytest.approx(2.577e12, rel=1e-3)
    per_head = L * d * 2 + n_obs * d * 2 + 8 * L + 8 * K + 4 * K * d * 2
    assert wm["step_bytes"] == pytest.approx(per_head * H)
    assert wm["step_bytes"] == pytest.approx(4.876e9, rel=1e-3)
    assert wm["step_exps"] == pytest.approx(n_obs * L * H)
    assert wm["compact"]["work"] == pytest.approx(4 * K * d * 2 * H)
    # FPS: M picks against M' + W union points of d channels, per query head,
    # as FMAs and (tensor cores) as 2 FLOP each
    assert wm["fps_fma"] == pytest.approx(1600 * 128 * (128 + 4096) * 128)
    assert wm["fps"]["work"] == pytest.approx(2 * 1600 * 128 * (128 + 4096) * 128)
    assert wm["fps"]["bound"] == "tensor" and wm["fps"]["unit"] == "FLOP"


def test_select_bytes_14b():
    """The select streams one word per key and writes K positions per head:
    the max form's merged order key, or one partial per group of at most 256
    observation rows for the mean (960 rows: 4 groups)."""
    wl = synth.WORKLOADS["qwen3_14b"]
    H, L, K = 320, 32768, 6144
    assert bench.work_model(wl, "max")["select"]["work"] == pytest.approx((4 * L + 4 * K) * H)
    assert bench.work_model(wl, "max")["select"]["work"] == pytest.approx(49_807_360)
    assert bench.work_model(wl, "mean")["select"]["work"] == pytest.approx((4 * 4 * L + 4 * K) * H)
    assert bench.work_model(wl, "mean")["select"]["work"] == pytest.approx(175_636_480)


def test_mufu_bound_14b():
    wm = bench.work_model(synth.WORKLOADS["qwen3_14b"])
    t = bench.mufu_bound_s(wm, {"sm_max_mhz": 1965.0})
    # 1.007e10 exps / (16 * 148 * 1.965e9 per second)
    assert t == pytest.approx(1.0066e10 / (16 * 148 * 1.965e9), rel=1e-3)
    assert 2.1e-3 < t < 2.2e-3
