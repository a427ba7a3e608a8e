"""Host-side arithmetic of the benchmark, on the CPU: the algorithmic FLOPs per
MLP row, the launch counts it claims, the whole-job rate and the traffic scaling."""
import os
import sys

import nerf_inputs as S

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_mlp_flops_per_row_of_the_page_network():
    # 8 x 256 with the skip after layer 4, sigma 1, feature 256, direction 128 (on
    # [feature, gamma(d)] of 256 + 27), rgb 3: the 1,186,816 FLOPs the roofline uses
    assert bench.mlp_flops_per_row(S.WORKLOADS["full"].mlp) == bench.MLP_FLOP_PER_ROW == 1186816


def test_march_launch_counts():
    # ray generation, then per chunk of up to 2^19 rays: mask, 3-kernel scan, emit,
    # the scene function (hash grid 1 kernel, KiloNeRF 7) and compositing
    assert bench.march_launches_per_step("hashgrid", 1920 * 1080) == 1 + 4 * 7
    assert bench.march_launches_per_step("kilonerf", 800 * 800) == 1 + 2 * 13
    assert bench.march_launches_per_step("kilonerf", 1 << 19) == 1 + 13
    assert bench.march_launches_per_step("hashgrid", 100) == 1 + 7


def test_whole_job_rate_uses_the_slowest_rank():
    # 4 ranks x 640,000 rays x 10 steps over the slowest rank's 2 s
    assert bench.job_rays_per_s(640000, 4, 10, 2000.0) == 4 * 640000 * 10 / 2.0


def test_traffic_scales_with_the_rows_of_a_launch():
    # the captured fine launch at 256 x 256: 12,582,912 rows, 236.75 MB
    rows = 12582912
    t = bench.traffic_per_launch(bench.MLP_FLOP_PER_ROW * rows)
    assert abs(t - 236.75e6) < 1.0
    assert abs(bench.traffic_per_launch(2 * bench.MLP_FLOP_PER_ROW * rows) - 2 * t) < 1.0
