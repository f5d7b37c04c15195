"""The bench's per-step algorithmic work (the roofline's numerators), pinned to
closed forms of the workload shapes: cache bytes = sum of lengths x (r + d_rope)
x element size, plus weights, queries and outputs; FLOPs = 2 rows L (r + d_rope)
for the scores (TPLA adds a second RoPE term), 2 rows L r for P cKV, and the
absorb and up-projection GEMMs."""

import pytest

import bench
from mla_workloads import WORKLOADS, draw_lengths


@pytest.mark.parametrize("name,cache_mb,step_mb,gflop", [
    ("deepseek_v3", 1207.960, 1244.135, 293.132),
    ("llama2_7b", 150.995, 159.711, 9.261),
    ("tpla_dsv3", 1207.960, 1244.135, 310.311),
    ("deepseek_v3_fp8", 675.283, 711.459, 293.132),
])
def test_step_work_matches_closed_forms(name, cache_mb, step_mb, gflop):
    wl = WORKLOADS[name]
    lens = draw_lengths(wl).tolist()
    w = bench.step_work(wl, lens)
    assert w["cache_bytes"] / 1e6 == pytest.approx(cache_mb, abs=1e-3)
    assert w["step_bytes"] / 1e6 == pytest.approx(step_mb, abs=1e-3)
    assert w["step_flops"] / 1e9 == pytest.approx(gflop, abs=1e-3)


def test_dsv3_closed_forms():
    wl = WORKLOADS["deepseek_v3"]
    B, L, H, r, dr, dn, dv = 32, 32768, 128, 512, 64, 128, 128
    w = bench.step_work(wl, [L] * B)
    assert w["cache_bytes"] == B * L * (r + dr) * 2
    assert w["decode_flops"] == 2 * H * B * L * (r + dr) + 2 * H * B * L * r
    assert w["step_flops"] == w["decode_flops"] + 2 * B * H * dn * r + 2 * B * H * r * dv
    # FP8: 512 code bytes, a bf16 RoPE key and an fp32 scale per token
    w8 = bench.step_work(WORKLOADS["deepseek_v3_fp8"], [L] * B)
    assert w8["cache_bytes"] == B * L * (r + 2 * dr + 4)
