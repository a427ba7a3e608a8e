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
    # the captured fine launch at 256 x 256: 12,582,912 rows, 237.21 MB
    rows = 12582912
    t = bench.traffic_per_launch(bench.MLP_FLOP_PER_ROW * rows)
    assert abs(t - 237.21e6) < 1.0
    assert abs(bench.traffic_per_launch(2 * bench.MLP_FLOP_PER_ROW * rows) - 2 * t) < 1.0


def test_nerf_kernel_bytes_of_the_bench_frame():
    wl = S.WORKLOADS["full"]                    # 640,000 rays, 64 + 128 samples, W = 256
    b = bench.nerf_kernel_bytes(wl)
    assert b["composite"] == 640000 * (192 * 20 + 32)
    assert b["resample"] == 640000 * (64 * 16 + 12 + 192 * 4)
    assert b["dir_bias"] == 2 * 640000 * (12 + 128 * 4)
    tiny = bench.nerf_kernel_bytes(S.WORKLOADS["tiny"])   # coarse only: positions recomputed
    assert tiny["composite"] == 1024 * (64 * 16 + 32) and "resample" not in tiny


def test_nerf_launch_counts_and_rows():
    assert bench.nerf_launches_per_step(S.WORKLOADS["full"]) == 9
    assert bench.nerf_launches_per_step(S.WORKLOADS["tiny"]) == 5
    # precision TF32, 200x200: the 2^20-sample store takes 16,384 rays of the
    # coarse pass and 5,461 of the fine one per sub-batch (3 and 8 sub-batches),
    # each with the encoding, a weight split and a row GEMM per layer (10 layers)
    # and the heads: 1 + 2 * 2 + (3 + 8) * 22 + 1 + 1 launches (the ncu launch
    # list of that frame counts the same 249)
    assert bench.nerf_launches_per_step(S.WORKLOADS["small_tf32"]) == 249
    # the compact 4x128 network at 800x800 with precision TF32: 40 + 118 sub-batches,
    # the direction layer's 64 outputs on the CUDA-core row GEMM (one launch)
    import dataclasses
    compact = dataclasses.replace(S.WORKLOADS["full"], mlp=S.MLPShape(D=4, W=128, skip=1),
                                  precision=S.PREC_TF32)
    assert bench.nerf_launches_per_step(compact) == 1 + 2 * 2 + (40 + 118) * 13 + 1 + 1
    assert bench.rows_per_frame(S.WORKLOADS["full"]) == 640000 * 256
    assert bench.rows_per_frame(S.WORKLOADS["tiny"]) == 1024 * 64


def test_bandwidth_figures():
    kinds = {"composite": (20.0, 10), "resample": (0.0, 0)}
    out = bench.bandwidth_figures(kinds, {"composite": 4e9, "resample": 1e9}, 10, 8000.0, "x")
    assert set(out) == {"composite"}                     # untimed classes are left out
    assert abs(out["composite"]["achieved_gbs"] - 4e9 * 10 / 0.020 / 1e9) < 1e-6
    assert abs(out["composite"]["frac"] - out["composite"]["achieved_gbs"] / 8000.0) < 1e-12


def test_march_kernel_bytes():
    b = bench.march_kernel_bytes(S.WORKLOADS["hashgrid"], 100, 1000, False)
    assert b["network"] == 1000 * 532 and b["march_mask"] == 100 * 92 and "router" not in b
    k = bench.march_kernel_bytes(S.WORKLOADS["kilonerf"], 100, 1000, False)
    assert k["router"] == 16000 and "network" not in k
