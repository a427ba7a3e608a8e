"""Multi-view sweep: the rays of several cameras generated in one call
(camera-major) and rendered through one nerf_render call, checked against the
oracle ray by ray (global ray indices key the random draws on both sides)."""
import dataclasses

import numpy as np
import pytest

import nerf_inputs as S
from oracle import nerf as onerf

from gpu_cases import check_rays, oracle_render, oracle_weights, render_gpu, weights_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch
    from neural_radiance_field_b200 import build
    build.build()
    return torch


def sweep_rays(torch, wl, cams):
    import neural_radiance_field_b200 as nb
    R = len(cams) * wl.H * wl.W
    o = torch.empty(R, 3, device="cuda")
    d = torch.empty(R, 3, device="cuda")
    nb.nerf_raygen_batch(wl.H, wl.W, wl.focal, [c.ravel() for c in cams], o, d)
    torch.cuda.synchronize()
    return o, d


@pytest.mark.parametrize("n_cams,H,W", [(3, 13, 17), (33, 2, 3), (1, 1, 1)])
def test_raygen_batch_bit_exact(torch, n_cams, H, W):
    """Each camera's slice equals the oracle's rays for that camera alone;
    33 cameras cross the 32-camera launch boundary."""
    cams = S.orbit_c2ws(7, n_cams)
    wl = dataclasses.replace(S.WORKLOADS["small"], H=H, W=W)
    o, d = sweep_rays(torch, wl, cams)
    o, d = o.cpu().numpy(), d.cpu().numpy()
    hw = H * W
    for c, c2w in enumerate(cams):
        oo, dd = onerf.raygen(H, W, wl.focal, c2w)
        np.testing.assert_array_equal(o[c * hw:(c + 1) * hw], oo)
        np.testing.assert_array_equal(d[c * hw:(c + 1) * hw], dd)


def test_raygen_batch_rejects_bad_arguments(torch):
    import ctypes
    from neural_radiance_field_b200 import _capi
    c = (ctypes.c_float * 12)()
    L = _capi.lib()
    assert L.nerf_raygen_batch(4, 4, 10.0, 0, c, ctypes.c_void_p(1), ctypes.c_void_p(1), None) \
        == _capi.NERF_ERR_INVALID_ARG
    assert L.nerf_raygen_batch(4, 4, 0.0, 1, c, ctypes.c_void_p(1), ctypes.c_void_p(1), None) \
        == _capi.NERF_ERR_INVALID_ARG


def test_sweep_coarse_pass_bf16_one_call(torch):
    """Four orbit cameras at 40x48 through the bf16 8x256 network in one
    nerf_render call, coarse pass: every sampled ray meets the bf16 bar (kink
    rays: one of the two branches)."""
    wl = dataclasses.replace(S.WORKLOADS["full"], H=40, W=48, n_fine=0)
    cams = S.orbit_c2ws(wl.seed, 4)
    rays = [onerf.raygen(wl.H, wl.W, wl.focal, c) for c in cams]   # camera-major, as batched
    o = torch.from_numpy(np.ascontiguousarray(np.concatenate([r[0] for r in rays]))).cuda()
    d = torch.from_numpy(np.ascontiguousarray(np.concatenate([r[1] for r in rays]))).cuda()
    cw, fw = oracle_weights(wl)
    gpu = render_gpu(wl, o, d, weights_tensor(cw, wl.precision), None)
    R = o.shape[0]
    ids = S.ray_subset(R, 256, 11)
    ref = oracle_render(wl, o.cpu().numpy(), d.cpu().numpy(), ids, cw, fw, perturb=True)
    check_rays(wl, {k: v[ids] for k, v in gpu.items()}, ref, "4-camera sweep, bf16 coarse pass")
    # rays from every camera are in the sample
    assert len(set((ids // (wl.H * wl.W)).tolist())) == 4
