"""The benchmark's multi-rank path on CPU: two gloo ranks, each with its own
camera and its own share of rays, no data exchange, and the max-over-ranks of
the per-rank device times (the only collective, outside the data path)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    import nerf_inputs as S
    from oracle import nerf as onerf

    wl = S.WORKLOADS["full"]
    cam = bench.rank_camera(wl, rank)
    # each rank generates its own rays (no exchange); report a checksum
    o, d = onerf.raygen(8, 8, wl.focal / 100, cam)
    local_ms = 100.0 + 25.0 * rank                     # a slower second rank
    dist.barrier()
    mx = bench.max_over_ranks(local_ms, dist, "cpu")
    out[rank] = (float(cam.sum()), float(d.sum()), mx,
                 bench.job_rays_per_s(wl.n_rays, world, 4, mx))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_without_exchange_and_reduce_max():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert sorted(out.keys()) == [0, 1]
    # distinct cameras and rays per rank
    assert out[0][0] != out[1][0] and out[0][1] != out[1][1]
    # both ranks agree on the slowest rank's time and the whole-job rate
    assert out[0][2] == out[1][2] == pytest.approx(125.0)
    assert out[0][3] == out[1][3] == pytest.approx(2 * 640000 * 4 / 0.125)


def test_rank_zero_renders_the_workload_camera():
    import bench
    import nerf_inputs as S
    wl = S.WORKLOADS["full"]
    np.testing.assert_array_equal(bench.rank_camera(wl, 0), wl.c2w())
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
