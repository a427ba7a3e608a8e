"""Pins of the training-step oracle (oracle/nerf_grad.py) against the
mathematics, not against itself: central finite differences of the same loss
(fp64, sample positions held fixed, as the detached sampling makes them),
equality of its forward with the render oracle, and finite differences of the
compositing backward alone."""
import dataclasses

import numpy as np
import pytest

import nerf_inputs as S
from oracle import nerf as onerf
from oracle import nerf_grad as og


def _case(shape, sigma_act, last_delta, white, n_coarse=12, n_fine=10, R=3, seed=21):
    wl = dataclasses.replace(S.WORKLOADS["tiny"], H=1, W=R, mlp=shape, sigma_act=sigma_act,
                             last_delta=last_delta, white_bkgd=white, n_coarse=n_coarse,
                             n_fine=n_fine, seed=seed)
    o, d = onerf.raygen(wl.H, wl.W, wl.focal, wl.c2w())
    cw, _ = S.nerf_weights(shape, seed, 0, 1.0, S.PREC_FP32)
    fw, _ = S.nerf_weights(shape, seed, 1, 1.0, S.PREC_FP32)
    target = np.random.default_rng(seed).uniform(0.0, 1.0, size=(R, 3))
    ids = np.arange(R)
    return wl, o, d, ids, target, cw.astype(np.float64), fw.astype(np.float64)


def _fd_indices(shape, rng, per_tensor=3):
    """A few parameter indices from every weight matrix and bias of the blob."""
    idx, off = [], 0
    for _, n, k in shape.layer_shapes():
        idx.extend((off + rng.choice(n * k, size=min(per_tensor, n * k), replace=False)).tolist())
        off += n * k
        idx.extend((off + rng.choice(n, size=min(per_tensor, n), replace=False)).tolist())
        off += n
    return np.array(idx)


CASES = [
    (S.MLPShape(D=3, W=8, skip=0), S.SIGMA_RELU, S.LAST_DELTA_TO_FAR, 0),
    (S.MLPShape(D=3, W=8, skip=1), S.SIGMA_SOFTPLUS, S.LAST_DELTA_PAGE, 1),
    (S.MLPShape(D=2, W=6, skip=-1), S.SIGMA_RELU, S.LAST_DELTA_TO_FAR, 1),
]


@pytest.mark.parametrize("shape,sigma_act,last_delta,white", CASES)
def test_gradient_matches_central_differences(shape, sigma_act, last_delta, white):
    wl, o, d, ids, target, cw, fw = _case(shape, sigma_act, last_delta, white)
    pos = og.sample_positions(wl, o, d, ids, cw.astype(np.float32))
    loss, gc, gf = og.loss_and_grad(wl, o, d, ids, target, cw, fw, positions=pos)
    assert gc.shape == cw.shape and gf.shape == fw.shape
    rng = np.random.default_rng(5)
    for which, flat, g in (("coarse", cw, gc), ("fine", fw, gf)):
        scale = np.abs(g).max()
        assert scale > 0
        for i in _fd_indices(shape, rng):
            h = 1e-6 * max(1.0, abs(flat[i]))
            up, dn = flat.copy(), flat.copy()
            up[i] += h
            dn[i] -= h
            args = (up, fw) if which == "coarse" else (cw, up)
            lu = og.loss_and_grad(wl, o, d, ids, target, *args, positions=pos, want_grad=False)[0]
            args = (dn, fw) if which == "coarse" else (cw, dn)
            ld = og.loss_and_grad(wl, o, d, ids, target, *args, positions=pos, want_grad=False)[0]
            fd = (lu - ld) / (2 * h)
            assert abs(fd - g[i]) <= 1e-6 * scale + 1e-10, (which, i, fd, g[i])


def test_loss_equals_the_render_oracle_mse():
    """The gradient module's forward is the render oracle's: its loss is the sum
    of the two passes' mean squared errors of render_nerf's colours."""
    shape = S.MLPShape(D=3, W=8, skip=1)
    wl, o, d, ids, target, cw, fw = _case(shape, S.SIGMA_RELU, S.LAST_DELTA_PAGE, 0,
                                          n_coarse=16, n_fine=8, R=4)
    loss, _, _ = og.loss_and_grad(wl, o, d, ids, target, cw, fw, want_grad=False)
    ref = onerf.render_nerf(wl, o, d, ids, cw.astype(np.float32), fw.astype(np.float32),
                            return_aux=True)
    mse = ((ref["rgb_c"] - target) ** 2).mean() + ((ref["rgb"] - target) ** 2).mean()
    assert abs(loss - mse) <= 1e-12 * max(1.0, mse)


def test_composite_backward_matches_central_differences():
    rng = np.random.default_rng(9)
    R, S_ = 2, 7
    sig_raw = rng.normal(0.0, 1.0, size=(R, S_))
    col_raw = rng.normal(0.0, 1.0, size=(R, S_, 3))
    delta = rng.uniform(0.05, 0.4, size=(R, S_))
    d_rgb = rng.normal(0.0, 1.0, size=(R, 3))
    for act in (S.SIGMA_RELU, S.SIGMA_SOFTPLUS):
        for white in (0, 1):
            def f(sr, cr):
                rgb, _, _, _ = onerf.composite(onerf.sigma_activation(sr, act), onerf.sigmoid(cr),
                                               np.zeros_like(sr), delta, white)
                return float((rgb * d_rgb).sum())
            ds, dc = og.composite_backward(sig_raw, col_raw, delta, act, white, d_rgb)
            h = 1e-6
            for (r, s) in [(0, 0), (0, 3), (1, 6), (1, 2)]:
                if act == S.SIGMA_RELU and abs(sig_raw[r, s]) < 10 * h:
                    continue
                a, b = sig_raw.copy(), sig_raw.copy()
                a[r, s] += h
                b[r, s] -= h
                assert abs((f(a, col_raw) - f(b, col_raw)) / (2 * h) - ds[r, s]) < 1e-7
                for c in range(3):
                    a, b = col_raw.copy(), col_raw.copy()
                    a[r, s, c] += h
                    b[r, s, c] -= h
                    assert abs((f(sig_raw, a) - f(sig_raw, b)) / (2 * h) - dc[r, s, c]) < 1e-7
