"""Training step (loss and parameter gradients) through nerf_loss_grad, against
the fp64 oracle of oracle/nerf_grad.py (itself pinned by finite differences).

Coarse-only steps have exact sample positions on both sides and are held to a
strict bar. With a fine pass, the fine positions come from the coarse weights
in fp32 (kernel) and fp64 (oracle); a random L = 10 field amplifies that
rounding, so the fine gradient is held to max(bar, 3 x the oracle's own spread
when its positions move by fp32 rounding), the criterion of the forward tests."""
import dataclasses

import numpy as np
import pytest

import nerf_inputs as S
from oracle import nerf_grad as og

from gpu_cases import rays_for

pytestmark = pytest.mark.gpu

REL = 1e-4      # gradient bar, relative to the largest gradient entry of the network


@pytest.fixture(scope="module")
def torch():
    import torch
    from neural_radiance_field_b200 import build
    build.build()
    return torch


def _gpu_step(torch, wl, o, d, cw, fw, target, perturb=1, precision=S.PREC_FP32):
    import neural_radiance_field_b200 as nb
    m = wl.mlp
    R = o.shape[0]
    rnd = nb.Renderer(D=m.D, W=m.W, skip=m.skip, sigma_act=wl.sigma_act, precision=precision,
                      last_delta_mode=wl.last_delta, white_bkgd=wl.white_bkgd, max_rays=R,
                      max_samples=wl.n_coarse + wl.n_fine)
    cwt = torch.from_numpy(cw).cuda()
    fwt = torch.from_numpy(fw).cuda() if fw is not None else None
    p = rnd.params(coarse_w=cwt, fine_w=fwt, seed=wl.seed, perturb=perturb)
    tgt = torch.from_numpy(target.astype(np.float32)).cuda()
    loss = torch.zeros(1, device="cuda")
    gc = torch.empty(cw.size, device="cuda")
    gf = torch.empty(cw.size, device="cuda") if fwt is not None else None
    rnd.loss_grad(o, d, wl.near, wl.far, wl.n_coarse, wl.n_fine, p, tgt, loss, gc, gf)
    torch.cuda.synchronize()
    rnd.sync_status()
    rnd.close()
    return (float(loss.item()), gc.cpu().numpy().astype(np.float64),
            gf.cpu().numpy().astype(np.float64) if gf is not None else None)


def _setup(key, H, W, **kw):
    wl = dataclasses.replace(S.WORKLOADS[key], H=H, W=W, precision=S.PREC_FP32, **kw)
    cw, _ = S.nerf_weights(wl.mlp, wl.seed, 0, wl.sigma_scale, S.PREC_FP32)
    fw, _ = S.nerf_weights(wl.mlp, wl.seed, 1, wl.sigma_scale, S.PREC_FP32) if wl.n_fine else (None, None)
    target = np.random.default_rng(wl.seed + 77).uniform(0.0, 1.0, size=(wl.n_rays, 3))
    return wl, cw, fw, target


COARSE_CASES = [
    dict(mlp=S.MLPShape(D=3, W=64, skip=0), last_delta=S.LAST_DELTA_TO_FAR),
    dict(mlp=S.MLPShape(D=4, W=128, skip=1), last_delta=S.LAST_DELTA_TO_FAR, white_bkgd=1),
    dict(mlp=S.MLPShape(D=2, W=64, skip=-1), last_delta=S.LAST_DELTA_TO_FAR,
         sigma_act=S.SIGMA_SOFTPLUS),
    dict(mlp=S.MLPShape(D=8, W=256, skip=4), last_delta=S.LAST_DELTA_TO_FAR),
    dict(mlp=S.MLPShape(D=3, W=64, skip=1), last_delta=S.LAST_DELTA_PAGE,
         sigma_act=S.SIGMA_SOFTPLUS, white_bkgd=1),
]


@pytest.mark.parametrize("kw", COARSE_CASES,
                         ids=lambda kw: f"D{kw['mlp'].D}W{kw['mlp'].W}s{kw['mlp'].skip}")
def test_coarse_step_matches_oracle(torch, kw):
    wl, cw, fw, target = _setup("small", 5, 7, n_fine=0, **kw)
    o, d = rays_for(wl)
    loss, gc, _ = _gpu_step(torch, wl, o, d, cw, None, target)
    ids = np.arange(wl.n_rays)
    ref_loss, ref_gc, _ = og.loss_and_grad(wl, o.cpu().numpy(), d.cpu().numpy(), ids, target,
                                           cw.astype(np.float64), None)
    assert abs(loss - ref_loss) <= 1e-5 * ref_loss, (loss, ref_loss)
    scale = np.abs(ref_gc).max()
    err = np.abs(gc - ref_gc).max()
    print(f"[train {kw['mlp']}] loss rel err {abs(loss - ref_loss) / ref_loss:.2e}, "
          f"grad max err / max|g| {err / scale:.2e}")
    assert err <= REL * scale + 1e-9, (err, scale, int(np.abs(gc - ref_gc).argmax()))


def test_many_tiles_step_matches_oracle(torch):
    """The 8 x 256 network on 800 rays x 64 samples (51,200 rows): the tensor-core
    row GEMMs walk two or three 128-row tiles per CTA and the weight gradients
    twenty-odd 16-row chunks per CTA through their three shared-memory stages, so
    every stage and tensor-memory buffer is reused, at the strict bar."""
    wl, cw, fw, target = _setup("small", 32, 25, n_fine=0, mlp=S.MLPShape(D=8, W=256, skip=4),
                                last_delta=S.LAST_DELTA_TO_FAR)
    o, d = rays_for(wl)
    loss, gc, _ = _gpu_step(torch, wl, o, d, cw, None, target)
    ids = np.arange(wl.n_rays)
    ref_loss, ref_gc, _ = og.loss_and_grad(wl, o.cpu().numpy(), d.cpu().numpy(), ids, target,
                                           cw.astype(np.float64), None)
    assert abs(loss - ref_loss) <= 1e-5 * ref_loss, (loss, ref_loss)
    scale = np.abs(ref_gc).max()
    err = np.abs(gc - ref_gc).max()
    print(f"[train 800 rays D8W256] loss rel err {abs(loss - ref_loss) / ref_loss:.2e}, "
          f"grad max err / max|g| {err / scale:.2e}")
    assert err <= REL * scale + 1e-9, (err, scale, int(np.abs(gc - ref_gc).argmax()))


def test_step_on_a_tf32_context(torch):
    """nerf_loss_grad on a context of precision TF32 (fp32 weights): the same
    training path and the same bar as FP32, 8 x 256 network, 35 rays."""
    wl, cw, fw, target = _setup("small", 5, 7, n_fine=0, mlp=S.MLPShape(D=8, W=256, skip=4),
                                last_delta=S.LAST_DELTA_TO_FAR)
    o, d = rays_for(wl)
    loss, gc, _ = _gpu_step(torch, wl, o, d, cw, None, target, precision=S.PREC_TF32)
    ref_loss, ref_gc, _ = og.loss_and_grad(wl, o.cpu().numpy(), d.cpu().numpy(), np.arange(wl.n_rays),
                                           target, cw.astype(np.float64), None)
    assert abs(loss - ref_loss) <= 1e-5 * ref_loss, (loss, ref_loss)
    scale = np.abs(ref_gc).max()
    err = np.abs(gc - ref_gc).max()
    print(f"[train tf32 context] grad max err / max|g| {err / scale:.2e}")
    assert err <= REL * scale + 1e-9


def test_coarse_and_fine_step(torch):
    wl, cw, fw, target = _setup("small", 4, 6, mlp=S.MLPShape(D=3, W=64, skip=0),
                                last_delta=S.LAST_DELTA_TO_FAR)
    o, d = rays_for(wl)
    loss, gc, gf = _gpu_step(torch, wl, o, d, cw, fw, target)
    o_np, d_np = o.cpu().numpy(), d.cpu().numpy()
    ids = np.arange(wl.n_rays)
    pos = og.sample_positions(wl, o_np, d_np, ids, cw)
    ref_loss, ref_gc, ref_gf = og.loss_and_grad(wl, o_np, d_np, ids, target, cw.astype(np.float64),
                                                fw.astype(np.float64), positions=pos)
    # the coarse network's gradient sees exact positions
    assert np.abs(gc - ref_gc).max() <= REL * np.abs(ref_gc).max() + 1e-9
    # the oracle's own spread under fp32-level moves of the fine positions
    rng = np.random.default_rng(3)
    spread_g = np.zeros_like(ref_gf)
    spread_l = 0.0
    for _ in range(3):
        t_all = pos[1].astype(np.float64)
        t_all = (t_all * (1.0 + 1.2e-7 * rng.standard_normal(t_all.shape))).astype(np.float32)
        t_all = np.sort(t_all, axis=-1)
        l2, _, g2 = og.loss_and_grad(wl, o_np, d_np, ids, target, cw.astype(np.float64),
                                     fw.astype(np.float64), positions=(pos[0], t_all))
        spread_g = np.maximum(spread_g, np.abs(g2 - ref_gf))
        spread_l = max(spread_l, abs(l2 - ref_loss))
    scale = np.abs(ref_gf).max()
    print(f"[train coarse+fine] coarse grad err {np.abs(gc - ref_gc).max() / np.abs(ref_gc).max():.2e}, "
          f"fine grad err {np.abs(gf - ref_gf).max() / scale:.2e}, "
          f"fine spread {spread_g.max() / scale:.2e}")
    bound = np.maximum(REL * scale, 3.0 * spread_g) + 1e-9
    assert (np.abs(gf - ref_gf) <= bound).all(), np.abs(gf - ref_gf).max() / scale
    assert abs(loss - ref_loss) <= max(1e-5 * ref_loss, 3.0 * spread_l)


def test_loss_grad_rejects_bf16_and_bad_arguments(torch):
    import ctypes
    import neural_radiance_field_b200 as nb
    from neural_radiance_field_b200 import _capi
    rnd = nb.Renderer(precision=S.PREC_BF16, max_rays=16, max_samples=192)
    p = rnd.params()
    fake = ctypes.c_void_p(16)
    st = _capi.lib().nerf_loss_grad(rnd.ctx, fake, fake, 4, 2.0, 6.0, 64, 0, ctypes.byref(p),
                                    fake, fake, fake, None, None)
    assert st == _capi.NERF_ERR_UNSUPPORTED
    rnd.close()
    rnd = nb.Renderer(precision=S.PREC_FP32, max_rays=16, max_samples=192)
    p = rnd.params()
    st = _capi.lib().nerf_loss_grad(rnd.ctx, fake, fake, 4, 2.0, 6.0, 64, 128, ctypes.byref(p),
                                    fake, fake, fake, None, None)
    assert st == _capi.NERF_ERR_INVALID_ARG        # fine pass without grad_fine / weights
    rnd.close()


def test_full_batch_is_the_mean_of_its_halves(torch):
    """The training step at its benchmark size (4096 rays of the 800 x 800 frame,
    coarse 64 + fine 128, the 8 x 256 network, fp32), where the oracle would take
    hours: with perturb = 0 every ray's samples are independent of its index, so
    the loss and the gradients of the batch are the means of those of its two
    halves (each term is normalised by its own 3 n). This exercises the launch
    configuration the benchmark times (row slices, atomics, full grids)."""
    import neural_radiance_field_b200 as nb
    wl = dataclasses.replace(S.WORKLOADS["full"], precision=S.PREC_FP32)
    m = wl.mlp
    B = 4096
    o_all, d_all = rays_for(wl)
    idx = torch.from_numpy(np.random.default_rng(17).choice(wl.n_rays, B, replace=False)).cuda()
    o, d = o_all[idx].contiguous(), d_all[idx].contiguous()
    cw, _ = S.nerf_weights(m, wl.seed, 0, wl.sigma_scale, S.PREC_FP32)
    fw, _ = S.nerf_weights(m, wl.seed, 1, wl.sigma_scale, S.PREC_FP32)
    target = torch.from_numpy(np.random.default_rng(18).uniform(0, 1, (B, 3)).astype(np.float32)).cuda()
    rnd = nb.Renderer(D=m.D, W=m.W, skip=m.skip, precision=S.PREC_FP32, max_rays=B,
                      max_samples=wl.n_coarse + wl.n_fine)
    # the context keeps raw pointers: the weight tensors must outlive every call
    cwt, fwt = torch.from_numpy(cw).cuda(), torch.from_numpy(fw).cuda()
    p = rnd.params(coarse_w=cwt, fine_w=fwt, seed=wl.seed, perturb=0)

    def step(sl):
        loss = torch.zeros(1, device="cuda")
        gc = torch.empty(cw.size, device="cuda")
        gf = torch.empty(fw.size, device="cuda")
        rnd.loss_grad(o[sl].contiguous(), d[sl].contiguous(), wl.near, wl.far, wl.n_coarse,
                      wl.n_fine, p, target[sl].contiguous(), loss, gc, gf)
        torch.cuda.synchronize()
        return float(loss.item()), gc.cpu().numpy().astype(np.float64), gf.cpu().numpy().astype(np.float64)

    lf, gcf, gff = step(slice(0, B))
    l1, gc1, gf1 = step(slice(0, B // 2))
    l2, gc2, gf2 = step(slice(B // 2, B))
    rnd.sync_status()
    rnd.close()
    assert abs(lf - 0.5 * (l1 + l2)) <= 1e-5 * lf
    for g, a, b in ((gcf, gc1, gc2), (gff, gf1, gf2)):
        scale = np.abs(g).max()
        assert scale > 0
        err = np.abs(g - 0.5 * (a + b)).max()
        print(f"[train 4096 additivity] max err / max|g| {err / scale:.2e}")
        assert err <= REL * scale, (err, scale)
