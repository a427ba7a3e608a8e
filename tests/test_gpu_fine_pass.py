"""The fine pass of the NeRF render ("Spatial Intelligence - Part 1: NeRF",
Section 2.6, render_rays and sample_pdf) against the oracle, stage by stage on
identical inputs (teacher forcing).

The render runs through nerf_render_trace in nerf_render's own kernels and
launch shapes, over the whole image. Each stage then gets exactly the values the
GPU's previous stage produced: the coarse weights go to the oracle's sample_pdf
(bins bit-exact, draws within 2e-6), and the merged positions t_all go to the
oracle's fine network and compositor. The fine-pass result is held to the
workload's bar on every sampled ray: rgb and acc within 1e-4 (fp32) or 2e-2
(bf16), depth within 1e-3 (far - near); a page-mode ray whose last raw density
sits on the ReLU kink must equal one of the oracle's two branches."""
import dataclasses

import pytest

import nerf_inputs as S

from gpu_cases import staged_fine_pass

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch
    from neural_radiance_field_b200 import build
    build.build()
    return torch


def test_staged_fine_pass_800x800_bf16(torch):
    """The benchmark's workload: 800x800, 64 + 128 samples, 8x256 bf16 network on
    the tensor cores."""
    staged_fine_pass(S.WORKLOADS["full"], 256, 3)


def test_staged_fine_pass_200x200_fp32(torch):
    """200x200, 64 + 128 samples, 8x256 fp32 network on the CUDA cores."""
    staged_fine_pass(S.WORKLOADS["small"], 384, 1)


def test_staged_fine_pass_200x200_tf32(torch):
    """The same with precision TF32: the fine network's 40,000 x 192 samples run
    in eight sub-batches of the activation store."""
    staged_fine_pass(S.WORKLOADS["small_tf32"], 384, 1)


def test_staged_fine_pass_unperturbed_to_far_white(torch):
    """Evenly spaced draws and jitter-free strata, the last interval reaching
    far (the closed-form reading), white background; ragged 21x23 image."""
    wl = dataclasses.replace(S.WORKLOADS["small"], H=21, W=23, last_delta=S.LAST_DELTA_TO_FAR,
                             white_bkgd=1)
    staged_fine_pass(wl, wl.n_rays, 0, perturb=0)


def test_staged_fine_pass_bf16_partial_draws(torch):
    """bf16 network with 37 fine draws (a ragged 101-sample union) on a 33x31
    image."""
    wl = dataclasses.replace(S.WORKLOADS["full"], H=33, W=31, focal=1.25 * 31, n_fine=37)
    staged_fine_pass(wl, 300, 5)
