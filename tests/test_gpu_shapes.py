"""Compact network shapes (the NAS-NeRF page's scene-specialised architectures:
other depths, widths and skip positions than the 8x256 baseline) through the
fp32 CUDA-core path and, for widths 128 and 256, precision TF32 (the layer
GEMMs on the tensor cores), checked against the oracle ray by ray."""
import dataclasses

import numpy as np
import pytest

import nerf_inputs as S

from gpu_cases import (check_rays, oracle_render, oracle_weights, rays_for, render_gpu,
                       staged_fine_pass, weights_tensor)

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


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"D{s.D}W{s.W}skip{s.skip}")
def test_compact_shape_coarse_pass(torch, shape):
    """Coarse pass (exact sample positions on both sides): every ray within the
    fp32 bar (kink rays: one of the two branches)."""
    wl = dataclasses.replace(S.WORKLOADS["small"], H=11, W=13, mlp=shape, n_fine=0)
    o, d = rays_for(wl)
    cw, fw = oracle_weights(wl)
    gpu = render_gpu(wl, o, d, weights_tensor(cw, wl.precision), None)
    ids = np.arange(o.shape[0])
    ref = oracle_render(wl, o.cpu().numpy(), d.cpu().numpy(), ids, cw, fw)
    check_rays(wl, gpu, ref, f"compact {shape}")


@pytest.mark.parametrize("shape", SHAPES[:3], ids=lambda s: f"D{s.D}W{s.W}skip{s.skip}")
def test_compact_shape_fine_pass_staged(torch, shape):
    """Coarse + fine with a compact network, stage by stage on identical inputs
    (bins bit-exact, fine pass within the fp32 bar on every ray)."""
    wl = dataclasses.replace(S.WORKLOADS["small"], H=9, W=10, mlp=shape)
    staged_fine_pass(wl, wl.n_rays, 0)


TF32_SHAPES = [s for s in SHAPES if s.W >= 128]


@pytest.mark.parametrize("shape", TF32_SHAPES, ids=lambda s: f"D{s.D}W{s.W}skip{s.skip}")
def test_compact_shape_tf32_coarse_pass(torch, shape):
    """The same coarse pass with precision TF32: every ray within the fp32 bar.
    At W = 128 the direction layer (64 outputs) runs on the CUDA-core row GEMM
    inside the tensor-core pass."""
    wl = dataclasses.replace(S.WORKLOADS["small_tf32"], H=11, W=13, mlp=shape, n_fine=0)
    o, d = rays_for(wl)
    cw, fw = oracle_weights(wl)
    gpu = render_gpu(wl, o, d, weights_tensor(cw, wl.precision), None)
    ids = np.arange(o.shape[0])
    ref = oracle_render(wl, o.cpu().numpy(), d.cpu().numpy(), ids, cw, fw)
    check_rays(wl, gpu, ref, f"compact tf32 {shape}")


def test_compact_shape_tf32_fine_pass_staged(torch):
    """Coarse + fine, precision TF32, D=4 W=128 with the skip after layer 1,
    stage by stage on identical inputs."""
    wl = dataclasses.replace(S.WORKLOADS["small_tf32"], H=9, W=10, mlp=TF32_SHAPES[0])
    staged_fine_pass(wl, wl.n_rays, 0)
