"""The entry point that allocates no device memory (nerf_march_compact_noalloc),
for callers that cannot call cudaMalloc: a host framework that owns all device
memory through its own allocator, or a render loop held to a fixed budget.

Its output must match the allocating march test entry point (nerf_test_march)
exactly, and the oracle's occupancy test (oracle.march.occupied) on the same
candidates: it is integer work (live-candidate decisions and their prefix sum).
Two calls in a row check that the shared static scratch carries nothing from
one call into the next. The file sorts last so that a run stopping at the first
failure has run every other test before it."""
import ctypes

import numpy as np
import pytest

import nerf_inputs as S
from oracle import march as omarch
from oracle import nerf as onerf

from gpu_cases import rays_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch
    from neural_radiance_field_b200 import build
    build.build()
    return torch


def _reference(torch, o, d, wl, K, occ):
    """Offsets and live entries from the allocating entry point's counts/flags."""
    import neural_radiance_field_b200 as nb
    R = o.shape[0]
    cnt = torch.empty(R, dtype=torch.int32, device="cuda")
    live = torch.empty(R, K, dtype=torch.uint8, device="cuda")
    nb.nerf_test_march(o, d, wl.near, wl.march_step, K, occ, cnt, live)
    cnt = cnt.cpu().numpy().astype(np.int64)
    flags = live.cpu().numpy().astype(bool)
    offsets = np.concatenate([[0], np.cumsum(cnt)])
    ray, k = np.nonzero(flags)                        # ray-major, k ascending
    entries = ((ray.astype(np.uint64) << 9) | k.astype(np.uint64)).astype(np.uint32)
    return offsets, entries


def _oracle(o, d, wl, K, dense):
    """Offsets and live entries from the oracle's voxel test of every candidate
    x = fl(o + fl(t_k d)), t_k = fl(near + fl(k step))."""
    x = onerf.points(o, d, np.broadcast_to(onerf.march_t(wl.near, wl.march_step, K),
                                           (o.shape[0], K)))
    flags = omarch.occupied(x, dense)
    offsets = np.concatenate([[0], np.cumsum(flags.sum(1))])
    ray, k = np.nonzero(flags)
    return offsets, ((ray.astype(np.uint64) << 9) | k.astype(np.uint64)).astype(np.uint32)


def _noalloc(torch, o, d, wl, K, occ):
    from neural_radiance_field_b200 import _capi
    R = o.shape[0]
    off = torch.full((R + 1,), -7, dtype=torch.int32, device="cuda")
    live = torch.full((R * K,), 0xFFFFFFF, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    rc = _capi.lib().nerf_march_compact_noalloc(
        ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(d.data_ptr()), R, wl.near,
        wl.march_step, K, ctypes.c_void_p(occ.data_ptr()), ctypes.c_void_p(off.data_ptr()),
        ctypes.c_void_p(live.data_ptr()), ctypes.c_void_p(st))
    assert rc == _capi.NERF_OK, _capi.lib().nerf_last_error(None)
    torch.cuda.synchronize()
    off = off.cpu().numpy().astype(np.int64)
    return off, live.cpu().numpy().view(np.uint32)[:off[-1]]


def test_noalloc_compaction_matches_allocating_entry_point_twice(torch):
    cases = [("hashgrid", 20001, 3), ("kilonerf", 7777, 8)]    # two calls, different inputs
    for key, n, seed in cases:
        wl = S.WORKLOADS[key]
        o, d = rays_for(wl)
        ids = S.ray_subset(wl.n_rays, n, seed)
        o, d = o[ids].contiguous(), d[ids].contiguous()
        packed, dense = S.occupancy_grid(wl.seed)
        occ = torch.from_numpy(packed.view(np.int32)).cuda()
        ref_off, ref_live = _reference(torch, o, d, wl, wl.n_coarse, occ)
        off, live = _noalloc(torch, o, d, wl, wl.n_coarse, occ)
        np.testing.assert_array_equal(off, ref_off)
        np.testing.assert_array_equal(live, ref_live)
        or_off, or_live = _oracle(o.cpu().numpy(), d.cpu().numpy(), wl, wl.n_coarse, dense)
        np.testing.assert_array_equal(off, or_off)
        np.testing.assert_array_equal(live, or_live)
        assert ref_off[-1] > 0


def test_noalloc_rejects_batches_beyond_its_scratch(torch):
    from neural_radiance_field_b200 import _capi
    buf = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(buf.data_ptr())
    rc = _capi.lib().nerf_march_compact_noalloc(p, p, (1 << 20) + 1, 2.0, 0.01, 64, p, p, p, None)
    assert rc == _capi.NERF_ERR_INVALID_ARG
    assert b"limit" in _capi.lib().nerf_last_error(None)
