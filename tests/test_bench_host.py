"""bench.py's roofline arithmetic on the host (no GPU): the grouped FFN's
algorithmic bytes and flops per launch, which bound applies to which batch, and
the fraction against the measured peaks."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

PEAKS = (6000.0, 1600.0, 1400.0, "measured")
H, I, k = 2816, 704, 8
EB = {0: 11894784, 1: 5964288, 2: 3159552}


def test_decode_is_bound_by_hbm_with_the_distinct_experts_bytes():
    r = bench.ffn_roofline(64, k, H, I, EB[0], 126.0, 0.25, PEAKS, None)
    alg = 126.0 * EB[0] + 64 * H * 2
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["alg_bytes_per_launch"] == int(alg)
    assert r["achieved"] == pytest.approx(alg / 0.25e-3 / 1e9, rel=1e-3)
    assert r["frac"] == pytest.approx(r["achieved"] / 6000.0, abs=1e-4)
    assert r["traffic"] is None and r["avg_launch_us"] == 250.0


def test_prefill_is_bound_by_the_tensor_pipe_against_the_sustained_peak():
    r = bench.ffn_roofline(1024, k, H, I, EB[2], 128.0, 0.4, PEAKS, (5.0e8, 4.2e8, "a capture"))
    flops = 2.0 * 1024 * k * 3 * H * I
    assert r["bound"] == "tensor" and r["peak"] == 1400.0
    assert r["alg_flops_per_launch"] == flops
    assert r["achieved"] == pytest.approx(flops / 0.4e-3 / 1e12, rel=1e-3)
    assert r["hbm"]["alg_bytes_per_launch"] == int(128 * EB[2] + 1024 * H * 2)
    assert r["traffic"] == 5.0e8 and r["traffic_alg_bytes"] == 4.2e8 and r["traffic_capture"] == "a capture"


def test_traffic_entries_name_their_capture():
    for key, val in bench.NCU_TRAFFIC_BYTES.items():
        assert len(key) == 2 and isinstance(val, tuple) and len(val) == 3
        assert val[0] > 0 and val[1] > 0 and "ncu" in val[2]
        # decode traffic is within a few percent of the algorithmic bytes; prefill
        # adds its fp32 rows and activation re-reads
        assert 1.0 <= val[0] / val[1] <= (1.4 if "prefill" in key[0] else 1.05)


class _FakeMoe:
    MOE_FFN_AUTO, MOE_FFN_GEMV, MOE_FFN_TC = 0, 1, 2


def test_launch_count_per_layer_step():
    m = _FakeMoe()
    # one token: fused route + permute, two GEMV launches, combine
    assert bench.launches_per_layer(m, 1, 8, 0, m.MOE_FFN_AUTO) == 1 + 2 + 1
    # one token through moe_layer_forward (the stacks): the routing inside the
    # first GEMV launch and the combine inside the second; not past its expert
    # count, on a forced path, or where AUTO takes the tensor cores
    assert bench.launches_per_layer(m, 1, 8, 0, m.MOE_FFN_AUTO, E=128) == 0 + 2 + 0
    assert bench.launches_per_layer(m, 1, 8, 0, m.MOE_FFN_AUTO, E=256) == 1 + 2 + 1
    assert bench.launches_per_layer(m, 1, 8, 0, m.MOE_FFN_GEMV, E=128) == 1 + 2 + 1
    assert bench.launches_per_layer(m, 1, 32, 0, m.MOE_FFN_AUTO, E=128) == 1 + 3 + 1
    # 8 tokens: fused route + permute, gather + two tensor-core launches, combine
    assert bench.launches_per_layer(m, 8, 8, 0, m.MOE_FFN_AUTO) == 1 + 3 + 1
    # 64 tokens: route and permute apart
    assert bench.launches_per_layer(m, 64, 8, 0, m.MOE_FFN_AUTO) == 2 + 3 + 1
    # the boundary of the one-launch routing, and forced paths
    assert bench.launches_per_layer(m, bench.FUSED_MAX_T, 8, 2, m.MOE_FFN_GEMV) == 1 + 2 + 1
    assert bench.launches_per_layer(m, bench.FUSED_MAX_T + 1, 1, 2, m.MOE_FFN_TC) == 2 + 3 + 1
