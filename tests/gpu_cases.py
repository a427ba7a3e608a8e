"""Shared set-up of the GPU parity tests: workloads as device tensors, renders
through the C ABI, and the matching oracle results.

Inputs come from nerf_inputs and the oracle's own ray generation (uploaded to the
device), so the free-running comparisons give the oracle no value produced on the
GPU. The teacher-forced stages (test_gpu_fine_pass.py) do the opposite on purpose:
they hand the oracle one GPU intermediate at a time (the coarse weights, the merged
sample positions) so that each later stage is compared on identical inputs."""
from __future__ import annotations

import dataclasses

import numpy as np

import nerf_inputs as S
from oracle import nerf as onerf

# Tolerances (see the design notes, "Parity bar"):
TOL_FP32 = dict(rgb=1e-4, acc=1e-4, depth_rel=1e-3)      # depth: 1e-3 * (far - near)
TOL_BF16 = dict(rgb=2e-2, acc=2e-2, depth_rel=1e-3)      # depth: 1e-3 * (far - near)
# Bounds on the raw network outputs that the MLP unit tests enforce. fp32: a
# K = 256..320 fp32 dot-product chain, ~K * 2^-24 relative per layer on O(1)
# values, with margin. bf16: operands and activations rounded to bf16 (2^-9
# relative) through 10 layers, accumulated with random signs, with margin.
RAW_BOUND = {S.PREC_FP32: 5e-5, S.PREC_BF16: 5e-3, S.PREC_TF32: 5e-5}
# Unit bars of the compositing and sampling stages on identical inputs (fp32
# exp/expm1 and a 192-term sum; two rounded operands and three operations).
TOL_COMPOSITE = dict(rgb=1e-5, acc=1e-5, depth=1e-4)
TOL_DRAW = 2e-6


def torch_mod():
    import torch
    return torch


def weights_tensor(flat, precision):
    torch = torch_mod()
    t = torch.from_numpy(np.ascontiguousarray(flat, dtype=np.float32))
    if precision == S.PREC_BF16:
        t = t.to(torch.bfloat16)
    return t.cuda()


def gpu_rays_for(wl):
    """GPU ray generation for the workload's camera (returns CUDA o, d)."""
    torch = torch_mod()
    import neural_radiance_field_b200 as nb
    o = torch.empty(wl.n_rays, 3, device="cuda")
    d = torch.empty(wl.n_rays, 3, device="cuda")
    nb.nerf_raygen(wl.H, wl.W, wl.focal, wl.c2w().ravel(), o, d)
    return o, d


def rays_for(wl):
    """The oracle's rays for the workload's camera, uploaded (returns CUDA o, d).
    The GPU's own ray generation is bit-identical (test_raygen_bit_exact)."""
    torch = torch_mod()
    o, d = onerf.raygen(wl.H, wl.W, wl.focal, wl.c2w())
    return torch.from_numpy(np.ascontiguousarray(o)).cuda(), torch.from_numpy(d).cuda()


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


def tolerances(wl):
    t = TOL_BF16 if wl.precision == S.PREC_BF16 else TOL_FP32
    return t["rgb"], t["acc"], t["depth_rel"] * (wl.far - wl.near)


def has_kink(wl):
    """Page-mode last interval (1e10) with a ReLU density: acc jumps between 0
    and 1 where the last raw density crosses 0."""
    return wl.sigma_act == S.SIGMA_RELU and wl.last_delta == S.LAST_DELTA_PAGE


def kink_branches(wl, raw, t, d):
    """The oracle's two results of a page-mode ray whose last raw density lies
    within rounding of the ReLU kink: the open end (sigma_last = 0, alpha_last =
    0) and the opaque end (sigma_last > 0, so alpha_last = 1 with the 1e10
    interval). Both are correct renders of the inputs at working precision."""
    out = []
    for v in (0.0, 1.0):
        r = np.array(raw, dtype=np.float64, copy=True)
        r[:, -1, 3] = v
        rgb, dep, acc, _ = onerf.composite_pass(wl, r, t, d)
        out.append(dict(rgb=rgb, depth=dep, acc=acc))
    return out


def within(err, tol):
    ok = np.ones(len(err["acc"]), dtype=bool)
    for k in err:
        ok &= err[k] <= tol[k]
    return ok


def check_kink_rays(wl, gpu, raw, t, d, tol):
    """Every kink ray equals (within `tol`) one of the oracle's two branches;
    returns the number of rays that took each branch."""
    br = kink_branches(wl, raw, t, d)
    ok = [within(ray_errors(gpu, b), tol) for b in br]
    bad = ~(ok[0] | ok[1])
    assert not bad.any(), {k: ray_errors(gpu, br[0])[k][bad] for k in ("rgb", "acc", "depth")}
    return int(ok[0].sum()), int(ok[1].sum())


def small_variant(key, **kw):
    return dataclasses.replace(S.WORKLOADS[key], **kw)


def oracle_render(wl, o_np, d_np, ids, cw, fw, perturb=True):
    ref = onerf.render_nerf(wl, o_np[ids], d_np[ids], ids, cw, fw, perturb=perturb,
                            return_aux=True)
    ref["d"] = d_np[ids]
    return ref


def check_rays(wl, gpu, ref, label=""):
    """Ray-by-ray parity of a render with the oracle's result `ref` (a dict from
    oracle_render, whose raw_final / t_final are the last pass's raw outputs and
    positions, or the same keys for a teacher-forced pass): every ray within the
    workload's tolerance, except that on page-mode ReLU workloads a ray whose
    last raw density lies within twice the MLP bound of 0 must instead equal one
    of the oracle's two branches (kink_branches). Returns (errors, kink mask)."""
    trgb, tacc, tdep = tolerances(wl)
    tol = dict(rgb=trgb, acc=tacc, depth=tdep)
    err = ray_errors(gpu, ref)
    n = len(err["acc"])
    kink = np.zeros(n, dtype=bool)
    if has_kink(wl):
        kink = np.abs(ref["raw_final"][:, -1, 3]) < 2 * RAW_BOUND[wl.precision]
    bad = ~within(err, tol) & ~kink
    assert not bad.any(), (label, int(bad.sum()), {k: float(v[bad].max()) for k, v in err.items()})
    branches = (0, 0)
    if kink.any():
        branches = check_kink_rays(wl, {k: v[kink] for k, v in gpu.items()},
                                   ref["raw_final"][kink], ref["t_final"][kink], ref["d"][kink], tol)
    off = ~kink
    print(f"[{label}] rays {n}, kink {int(kink.sum())} (open/opaque {branches}); max err off kink: "
          + ", ".join(f"{k} {err[k][off].max() if off.any() else 0.0:.2e}" for k in err)
          + f" (tol rgb {trgb:.0e}, acc {tacc:.0e}, depth {tdep:.0e})")
    return err, kink


def traced_render(wl, o, d, cw, fw, ids, perturb=1):
    """Render the whole batch through nerf_render_trace (the kernels and launch
    shapes of nerf_render) and return, for the rays `ids`, the outputs and the
    render's intermediates as numpy arrays."""
    torch = torch_mod()
    R = o.shape[0]
    Nc, Nf = wl.n_coarse, wl.n_fine
    S_ = Nc + Nf
    dev = dict(device="cuda")
    bufs = dict(raw_coarse=torch.empty(R, Nc, 4, **dev), w_coarse=torch.empty(R, Nc, **dev),
                t_fine=torch.empty(R, max(Nf, 1), **dev),
                below=torch.empty(R, max(Nf, 1), dtype=torch.int32, **dev),
                t_all=torch.empty(R, S_, **dev), raw_fine=torch.empty(R, S_, 4, **dev))
    rgb = torch.empty(R, 3, **dev)
    dep = torch.empty(R, **dev)
    acc = torch.empty(R, **dev)
    with make_renderer(wl, R) as rnd:
        p = rnd.params(coarse_w=weights_tensor(cw, wl.precision),
                       fine_w=weights_tensor(fw, wl.precision) if fw is not None else None,
                       seed=wl.seed, perturb=perturb)
        rnd.render_trace(o, d, wl.near, wl.far, Nc, Nf, p, rgb, dep, acc, **bufs)
        rnd.sync_status()
    sel = torch.from_numpy(np.asarray(ids, dtype=np.int64)).cuda()
    out = {k: v[sel].cpu().numpy() for k, v in bufs.items()}
    out.update(rgb=rgb[sel].cpu().numpy(), depth=dep[sel].cpu().numpy(),
               acc=acc[sel].cpu().numpy())
    del bufs
    torch.cuda.empty_cache()
    return out


def draws(wl, ids, perturb):
    """The 24-bit inverse-CDF draws m of the rays (stream 1), or the evenly
    spaced draws (k + 0.5) / n_fine without perturbation."""
    from oracle import rng as orng
    ids = np.asarray(ids, dtype=np.int64)
    if perturb:
        return orng.draw_bits(wl.seed, ids[:, None], 1, np.arange(wl.n_fine)[None, :])
    return np.tile(((np.arange(wl.n_fine) * 2 + 1) << 23) // wl.n_fine, (len(ids), 1))


def staged_fine_pass(wl, n_check, seed_ids, perturb=1):
    """The fine pass (NeRF page, Section 2.6 render_rays) checked stage by stage,
    each stage on exactly the inputs the GPU's own previous stage produced:

    1. coarse network: the oracle's raw outputs at the stratified positions
       (bit-exact on both sides) against the render's raw_coarse, RAW_BOUND;
    2. coarse compositing: the oracle's weights from the render's raw_coarse
       against the weights the resampler used, TOL_COMPOSITE;
    3. sampler (sample_pdf) given the render's coarse weights: every bin
       bit-exact, every draw within TOL_DRAW, the sorted union bit-exact;
    4. fine network at the render's merged positions t_all, RAW_BOUND;
    5. fine compositing of the render's raw_fine, TOL_COMPOSITE;
    6. the fine pass given identical positions (teacher-forced t): the oracle's
       fine network and compositing at the render's t_all against the render's
       rgb / depth / acc, at the workload's tolerance on every ray (kink rays:
       one of the two branches).

    Returns the per-ray errors of stage 6."""
    o, d = rays_for(wl)
    cw, fw = oracle_weights(wl)
    ids = S.ray_subset(o.shape[0], n_check, seed_ids)
    g = traced_render(wl, o, d, cw, fw, ids, perturb)
    o_np, d_np = o.cpu().numpy()[ids], d.cpu().numpy()[ids]
    tag = f"{wl.name} {wl.H}x{wl.W}"
    bound = RAW_BOUND[wl.precision]
    # 1. coarse network
    t_c = onerf.stratified_t(wl.near, wl.far, wl.n_coarse, wl.seed, ids, bool(perturb))
    raw_c = onerf.network_pass(wl, cw, o_np, d_np, t_c)
    e1 = np.abs(g["raw_coarse"] - raw_c).max()
    assert e1 <= bound, ("coarse network", e1)
    # 2. coarse compositing of the render's own raw outputs
    _, _, _, w_ref = onerf.composite_pass(wl, g["raw_coarse"], t_c, d_np)
    e2 = np.abs(g["w_coarse"] - w_ref).max()
    assert e2 <= TOL_COMPOSITE["acc"], ("coarse weights", e2)
    # 3. inverse-CDF sampling from the render's coarse weights
    t_f, below = onerf.sample_pdf(onerf.midpoints(t_c), g["w_coarse"][:, 1:-1],
                                  draws(wl, ids, perturb))
    np.testing.assert_array_equal(g["below"], below)
    e3 = np.abs(g["t_fine"] - t_f).max()
    assert e3 <= TOL_DRAW, ("fine draws", e3)
    np.testing.assert_array_equal(g["t_all"], np.sort(np.concatenate([t_c, g["t_fine"]], 1), 1))
    # 4. fine network at the render's merged positions
    raw_f = onerf.network_pass(wl, fw, o_np, d_np, g["t_all"])
    e4 = np.abs(g["raw_fine"] - raw_f).max()
    assert e4 <= bound, ("fine network", e4)
    # 5. fine compositing of the render's own raw outputs
    rgb5, dep5, acc5, _ = onerf.composite_pass(wl, g["raw_fine"], g["t_all"], d_np)
    e5 = ray_errors(g, dict(rgb=rgb5, depth=dep5, acc=acc5))
    assert all(e5[k].max() <= TOL_COMPOSITE[k] for k in e5), {k: e5[k].max() for k in e5}
    # 6. the fine pass on identical positions
    rgb6, dep6, acc6, _ = onerf.composite_pass(wl, raw_f, g["t_all"], d_np)
    ref = dict(rgb=rgb6, depth=dep6, acc=acc6, raw_final=raw_f, t_final=g["t_all"], d=d_np)
    print(f"[staged {tag}] raw coarse {e1:.2e}, weights {e2:.2e}, bins exact, draws {e3:.2e}, "
          f"raw fine {e4:.2e}, compositing " + ", ".join(f"{k} {v.max():.2e}" for k, v in e5.items()))
    err, _ = check_rays(wl, g, ref, label=f"teacher-forced fine pass {tag}")
    return err
