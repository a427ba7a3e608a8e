"""nerf_render's argument contract on a live context: every bad request is
rejected with NERF_ERR_INVALID_ARG before any launch (empty and oversized ray
batches, sample counts past the workspace, an empty or reversed depth range,
null buffers, march limits), and the context then still renders its maximum
batch, whose result matches the oracle."""
import ctypes

import numpy as np
import pytest

import nerf_inputs as S

from gpu_cases import (check_rays, make_renderer, oracle_render, oracle_weights, rays_for,
                       weights_tensor)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch
    from neural_radiance_field_b200 import build
    build.build()
    return torch


def test_render_rejects_bad_requests_then_renders_its_maximum_batch(torch):
    from neural_radiance_field_b200 import _capi
    wl = S.WORKLOADS["tiny"]                                 # 32 x 32 rays, 4 x 64 fp32, coarse only
    R = wl.n_rays
    o, d = rays_for(wl)
    cw, fw = oracle_weights(wl)
    cwt = weights_tensor(cw, wl.precision)
    fwt = weights_tensor(fw, wl.precision) if fw is not None else None
    rnd = make_renderer(wl, R)                               # max_rays = R exactly
    p = rnd.params(coarse_w=cwt, fine_w=fwt, seed=wl.seed, perturb=1)
    rgb = torch.empty(R + 1, 3, device="cuda")
    dep = torch.empty(R + 1, device="cuda")
    acc = torch.empty(R + 1, device="cuda")
    L = _capi.lib()
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())

    def call(n, near=wl.near, far=wl.far, nc=wl.n_coarse, nf=wl.n_fine, oo=o, out=rgb):
        return L.nerf_render(rnd.ctx, ptr(oo) if oo is not None else None, ptr(d), n, near, far,
                             nc, nf, ctypes.byref(p), ptr(out) if out is not None else None,
                             ptr(dep), ptr(acc), None)

    bad = _capi.NERF_ERR_INVALID_ARG
    assert call(0) == bad                                    # empty batch
    assert call(-3) == bad
    assert call(R + 1) == bad                                # past max_rays
    assert call(R, nc=wl.n_coarse + wl.n_fine + 1, nf=0) == bad   # past max_samples
    assert call(R, nc=0) == bad
    assert call(R, near=wl.far, far=wl.near) == bad          # reversed range
    assert call(R, near=wl.near, far=wl.near) == bad         # empty range
    assert call(R, oo=None) == bad                           # null rays
    assert call(R, out=None) == bad                          # null output
    # nothing was launched, and the maximum batch renders and matches the oracle
    rnd.render(o, d, wl.near, wl.far, wl.n_coarse, wl.n_fine, p, rgb[:R], dep[:R], acc[:R])
    torch.cuda.synchronize()
    rnd.sync_status()
    rnd.close()
    got = dict(rgb=rgb[:R].cpu().numpy(), depth=dep[:R].cpu().numpy(), acc=acc[:R].cpu().numpy())
    ids = np.arange(R)
    ref = oracle_render(wl, o.cpu().numpy(), d.cpu().numpy(), ids, cw, fw)
    check_rays(wl, got, ref, "tiny, maximum batch")


def test_march_render_rejects_bad_candidate_counts(torch):
    import neural_radiance_field_b200 as nb
    from neural_radiance_field_b200 import _capi
    wl = S.WORKLOADS["kilonerf"]
    R = 64
    packed, _ = S.occupancy_grid(wl.seed)
    occ = torch.from_numpy(packed.view(np.int32)).cuda()
    cells = torch.from_numpy(S.kilonerf_weights(wl.seed)).cuda()
    rnd = nb.Renderer(model=nb.NERF_MODEL_KILONERF, max_rays=R, max_samples=512)
    p = rnd.params(occupancy=occ, cell_w=cells, march_step=wl.march_step, ert_T=wl.ert_T)
    o = torch.zeros(R, 3, device="cuda")
    d = torch.ones(R, 3, device="cuda")
    out3 = torch.empty(R, 3, device="cuda")
    out1 = torch.empty(R, device="cuda")
    L = _capi.lib()
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    args = lambda nc, nf: (rnd.ctx, ptr(o), ptr(d), R, wl.near, wl.far, nc, nf, ctypes.byref(p),
                           ptr(out3), ptr(out1), ptr(out1), None)
    assert L.nerf_render(*args(513, 0)) == _capi.NERF_ERR_INVALID_ARG    # more than 512 candidates
    assert L.nerf_render(*args(342, 8)) == _capi.NERF_ERR_INVALID_ARG    # no fine pass in march mode
    assert L.nerf_render(*args(342, 0)) == _capi.NERF_OK
    torch.cuda.synchronize()
    rnd.sync_status()
    rnd.close()
