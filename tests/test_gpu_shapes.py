"""Compact network shapes (the NAS-NeRF page's scene-specialised architectures:
other depths, widths and skip positions than the 8x256 baseline) through the
fp32 CUDA-core path, checked against the oracle ray by ray."""
import dataclasses

import numpy as np
import pytest

import nerf_inputs as S

from gpu_cases import (RAW_BOUND, compare, oracle_render, oracle_weights, probe_spread,
                       rays_for, render_gpu, tolerances, weights_tensor)

pytestmark = pytest.mark.gpu

SHAPES = [S.MLPShape(D=4, W=128, skip=1), S.MLPShape(D=2, W=64, skip=-1),
          S.MLPShape(D=6, W=256, skip=2), S.MLPShape(D=8, W=128, skip=4),
          S.MLPShape(D=1, W=128, skip=-1), S.MLPShape(D=3, W=64, skip=0)]


@pytest.fixture(scope="module")
def torch():
    import torch
    from neural_radiance_field_b200 import build
    build.build()
    return torch


def _run(wl, perturb=1, probe=False):
    o, d = rays_for(wl)
    cw, fw = oracle_weights(wl)
    gpu = render_gpu(wl, o, d, weights_tensor(cw, wl.precision),
                     weights_tensor(fw, wl.precision) if fw is not None else None, perturb=perturb)
    ids = np.arange(o.shape[0])
    o_np, d_np = o.cpu().numpy(), d.cpu().numpy()
    ref = oracle_render(wl, o_np, d_np, ids, cw, fw, perturb=bool(perturb))
    err, keep = compare(gpu, ref, wl, ids, band=2 * RAW_BOUND[wl.precision])
    spread = probe_spread(wl, o_np, d_np, ids, cw, fw, ref, perturb=bool(perturb)) if probe else None
    return err, keep, spread


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"D{s.D}W{s.W}skip{s.skip}")
def test_compact_shape_coarse_pass(torch, shape):
    """Coarse pass (exact sample positions on both sides): every ray off the
    page-mode kink within the fp32 bar."""
    wl = dataclasses.replace(S.WORKLOADS["small"], H=11, W=13, mlp=shape, n_fine=0)
    err, keep, _ = _run(wl)
    trgb, tacc, tdep = tolerances(wl)
    assert keep.mean() >= 0.8
    assert (err["rgb"][keep] <= trgb).all(), err["rgb"][keep].max()
    assert (err["acc"][keep] <= tacc).all(), err["acc"][keep].max()
    assert (err["depth"][keep] <= tdep).all(), err["depth"][keep].max()


def test_compact_shape_coarse_and_fine(torch):
    """Coarse + fine with a compact network: rays within the bar, or within three
    times the oracle's own spread under working-precision noise where resampling
    amplifies rounding (the criterion of the full-network tests)."""
    wl = dataclasses.replace(S.WORKLOADS["small"], H=9, W=10, mlp=S.MLPShape(D=4, W=128, skip=1))
    err, keep, spread = _run(wl, probe=True)
    trgb, tacc, tdep = tolerances(wl)
    tol = dict(rgb=trgb, acc=tacc, depth=tdep)
    strict = np.ones(len(keep), dtype=bool)
    consistent = np.ones(len(keep), dtype=bool)
    for k in err:
        strict &= err[k] <= tol[k]
        consistent &= err[k] <= np.maximum(tol[k], 3.0 * spread[k])
    assert (consistent | ~keep).all()
    assert strict.mean() >= 0.9
