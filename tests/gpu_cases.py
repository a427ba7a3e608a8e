"""Shared set-up of the GPU parity tests: workloads as device tensors, renders
through the C ABI, and the matching oracle results. Inputs come from
nerf_inputs only; the oracle never sees a value produced on the GPU."""
from __future__ import annotations

import dataclasses

import numpy as np

import nerf_inputs as S
from oracle import nerf as onerf

# Tolerances (see the design notes, "Parity bar"):
TOL_FP32 = dict(rgb=1e-4, acc=1e-4, depth_rel=1e-3)      # depth: 1e-3 * (far - near)
TOL_BF16 = dict(rgb=2e-2, acc=2e-2, depth_far=2e-2)      # depth: 2e-2 * far
# Bounds on the raw network outputs that the MLP unit tests enforce. fp32: a
# K = 256..320 fp32 dot-product chain, ~K * 2^-24 relative per layer on O(1)
# values, with margin. bf16: operands and activations rounded to bf16 (2^-9
# relative) through 10 layers, accumulated with random signs, with margin.
RAW_BOUND = {S.PREC_FP32: 5e-5, S.PREC_BF16: 5e-3}
# Working-precision noise for the oracle's conditioning probe (rel, abs): the
# typical size of the kernel's rounding of a raw output, not a bound on it.
PROBE_NOISE = {S.PREC_FP32: (0.0, 2e-6), S.PREC_BF16: (2.0 ** -8, 0.0)}


def torch_mod():
    import torch
    return torch


def weights_tensor(flat, precision):
    torch = torch_mod()
    t = torch.from_numpy(np.ascontiguousarray(flat, dtype=np.float32))
    if precision == S.PREC_BF16:
        t = t.to(torch.bfloat16)
    return t.cuda()


def rays_for(wl):
    """GPU ray generation for the workload's camera (returns CUDA o, d)."""
    torch = torch_mod()
    import neural_radiance_field_b200 as nb
    o = torch.empty(wl.n_rays, 3, device="cuda")
    d = torch.empty(wl.n_rays, 3, device="cuda")
    nb.nerf_raygen(wl.H, wl.W, wl.focal, wl.c2w().ravel(), o, d)
    return o, d


def make_renderer(wl, max_rays=None):
    import neural_radiance_field_b200 as nb
    m = wl.mlp
    return nb.Renderer(D=m.D, W=m.W, skip=m.skip, sigma_act=wl.sigma_act, precision=wl.precision,
                       last_delta_mode=wl.last_delta, white_bkgd=wl.white_bkgd,
                       max_rays=max_rays or wl.n_rays, max_samples=wl.n_coarse + wl.n_fine)


def render_gpu(wl, o, d, cw, fw, rnd=None, perturb=1):
    torch = torch_mod()
    R = o.shape[0]
    own = rnd is None
    rnd = rnd or make_renderer(wl, R)
    rgb = torch.empty(R, 3, device="cuda")
    dep = torch.empty(R, device="cuda")
    acc = torch.empty(R, device="cuda")
    p = rnd.params(coarse_w=cw, fine_w=fw, seed=wl.seed, perturb=perturb)
    rnd.render(o, d, wl.near, wl.far, wl.n_coarse, wl.n_fine, p, rgb, dep, acc)
    rnd.sync_status()
    out = dict(rgb=rgb.cpu().numpy(), depth=dep.cpu().numpy(), acc=acc.cpu().numpy())
    if own:
        rnd.close()
    return out


def oracle_weights(wl):
    cw, _ = S.nerf_weights(wl.mlp, wl.seed, 0, wl.sigma_scale, wl.precision)
    fw, _ = S.nerf_weights(wl.mlp, wl.seed, 1, wl.sigma_scale, wl.precision) if wl.n_fine else (None, None)
    return cw, fw


def ray_errors(a, b):
    return dict(rgb=np.abs(a["rgb"] - b["rgb"]).max(-1), acc=np.abs(a["acc"] - b["acc"]),
                depth=np.abs(a["depth"] - b["depth"]))


def compare(gpu, ref, wl, ids=None, band=None):
    """Per-ray errors and the rays on which the pages' discontinuity leaves the
    result undetermined: in page mode (last interval 1e10) a ReLU density whose
    raw value lies within `band` of 0 at the last sample decides between an
    opaque and a transparent end of the ray."""
    g = {k: (v[ids] if ids is not None else v) for k, v in gpu.items()}
    err = ray_errors(g, ref)
    keep = np.ones(len(err["acc"]), dtype=bool)
    if band is not None and wl.sigma_act == S.SIGMA_RELU and wl.last_delta == S.LAST_DELTA_PAGE:
        keep = np.abs(ref["sigma_last_raw"]) >= band
    return err, keep


def probe_spread(wl, o_np, d_np, ids, cw, fw, ref, perturb=True, draws=4):
    """Per ray and output, the largest move of the oracle's own result when every
    raw network output is perturbed at the kernel's working precision (seeded
    draws). Where the inverse-CDF resampling of a random high-frequency field
    amplifies rounding, this spread exceeds the tolerance for any
    implementation at that precision."""
    rel, ab = PROBE_NOISE[wl.precision]
    spread = None
    for s in range(draws):
        p = onerf.render_nerf(wl, o_np[ids], d_np[ids], ids, cw, fw, perturb=perturb,
                              raw_noise=(101 + s, rel, ab))
        e = ray_errors(p, ref)
        spread = e if spread is None else {k: np.maximum(spread[k], e[k]) for k in e}
    return spread


def tolerances(wl):
    if wl.precision == S.PREC_BF16:
        return TOL_BF16["rgb"], TOL_BF16["acc"], TOL_BF16["depth_far"] * wl.far
    return TOL_FP32["rgb"], TOL_FP32["acc"], TOL_FP32["depth_rel"] * (wl.far - wl.near)


def small_variant(key, **kw):
    return dataclasses.replace(S.WORKLOADS[key], **kw)


def oracle_render(wl, o_np, d_np, ids, cw, fw, perturb=True):
    return onerf.render_nerf(wl, o_np[ids], d_np[ids], ids, cw, fw, perturb=perturb,
                             return_aux=True)
