"""The hash-grid encoding's backward (nerf_hash_encode_backward) against the
oracle's scatter-add (HashGrid3D.encode_backward, pinned by the adjoint
identity). The deterministic mode must also be bit-identical across runs."""
import numpy as np
import pytest

from oracle.hashgrid import HashGrid3D

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch
    from neural_radiance_field_b200 import build
    build.build()
    return torch


def _inputs(seed, n, lo=-1.5, hi=1.5):
    rng = np.random.default_rng(seed)
    x = rng.uniform(lo, hi, size=(n, 3)).astype(np.float32)
    x[:8] = np.array([[-1.5, -1.5, -1.5], [1.5, 1.5, 1.5], [1.5, -1.5, 0.0], [0.0, 0.0, 0.0],
                      [-1.5, 0.3, 1.5], [0.7, 1.5, -0.2], [1.4999, -1.4999, 0.5],
                      [-0.75, 0.75, 1.125]], dtype=np.float32)[: min(8, n)]
    g = rng.normal(size=(n, 32)).astype(np.float32)
    return x, g


def _gpu(torch, x, g, deterministic):
    import neural_radiance_field_b200 as nb
    hg = HashGrid3D()
    grad = torch.zeros(hg.n_entries, 2, device="cuda")
    nb.nerf_hash_encode_backward(torch.from_numpy(x).cuda(), torch.from_numpy(g).cuda(), grad,
                                 deterministic=deterministic)
    torch.cuda.synchronize()
    return grad.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("deterministic", [False, True])
def test_matches_oracle(torch, deterministic):
    x, g = _inputs(0, 3000)
    ref = HashGrid3D().encode_backward(x, g)
    got = _gpu(torch, x, g, deterministic)
    scale = np.abs(ref).max()
    err = np.abs(got - ref).max()
    print(f"[hash backward deterministic={deterministic}] max err / max|ref| {err / scale:.2e}")
    assert err <= 1e-5 * scale, err / scale
    # the rows the GPU touched are the oracle's
    assert np.array_equal(np.nonzero(np.abs(got).sum(1))[0], np.nonzero(np.abs(ref).sum(1))[0])


def test_deterministic_mode_is_bit_identical(torch):
    """Many points crowded into a small region (thousands of terms per row):
    two runs of the fixed-point mode agree bit for bit."""
    x, g = _inputs(1, 1 << 18, lo=-0.05, hi=0.05)
    a = _gpu(torch, x, g, True)
    b = _gpu(torch, x, g, True)
    assert np.array_equal(a, b)
    ref = HashGrid3D().encode_backward(x[:4096], g[:4096])
    small = _gpu(torch, x[:4096], g[:4096], True)
    assert np.abs(small - ref).max() <= 1e-5 * np.abs(ref).max()


def test_rejects_bad_arguments(torch):
    import ctypes
    from neural_radiance_field_b200 import _capi
    fake = ctypes.c_void_p(16)
    L = _capi.lib()
    assert L.nerf_hash_encode_backward(None, 4, fake, fake, 0, None) == _capi.NERF_ERR_INVALID_ARG
    assert L.nerf_hash_encode_backward(fake, 0, fake, fake, 1, None) == _capi.NERF_ERR_INVALID_ARG
