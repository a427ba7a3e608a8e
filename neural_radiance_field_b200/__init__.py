"""B200 forward NeRF renderer: a thin Python binding over libnerf.so.

Every function here only marshals torch tensors (device memory, the current
CUDA stream) into the C ABI of include/nerf.h; all the work runs in the
library's CUDA kernels. Importing this package does not load the library;
the first call does, and fails loudly when it is missing.
"""
from __future__ import annotations

import ctypes

from . import _capi
from ._capi import (NERF_BF16, NERF_FP32, NERF_TF32, NERF_LAST_1E10, NERF_LAST_TO_FAR, NERF_MODEL_HASHGRID,
                    NERF_MODEL_KILONERF, NERF_MODEL_MLP, NERF_SIGMA_RELU, NERF_SIGMA_SOFTPLUS,
                    NerfError, nerf_config, nerf_params)

__all__ = ["Renderer", "nerf_raygen", "nerf_raygen_batch", "nerf_hash_encode_backward", "nerf_test_stratified", "nerf_test_pe",
           "nerf_test_composite", "nerf_test_sample_pdf", "NerfError", "nerf_config",
           "nerf_params"]


def _ptr(t):
    if t is None:
        return None
    import torch
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _hptr(t):
    if t is None:
        return None
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous host tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def nerf_raygen(H, W, focal, c2w, rays_o, rays_d, stream=None):
    """c2w: 12 host floats (sequence or array); rays_o, rays_d: CUDA [H*W, 3]."""
    c = (ctypes.c_float * 12)(*[float(v) for v in list(c2w)])
    _capi.check(_capi.lib().nerf_raygen(int(H), int(W), float(focal), c, _ptr(rays_o),
                                        _ptr(rays_d), _stream(stream)))


def nerf_raygen_batch(H, W, focal, c2ws, rays_o, rays_d, stream=None):
    """c2ws: n_cams x 12 host floats; rays_o, rays_d: CUDA [n_cams*H*W, 3], camera-major."""
    flat = [float(v) for cam in c2ws for v in list(cam)]
    n_cams = len(flat) // 12
    if n_cams * 12 != len(flat):
        raise ValueError("each camera needs 12 values ([3][4] row-major)")
    c = (ctypes.c_float * len(flat))(*flat)
    _capi.check(_capi.lib().nerf_raygen_batch(int(H), int(W), float(focal), n_cams, c,
                                              _ptr(rays_o), _ptr(rays_d), _stream(stream)))


def nerf_test_stratified(rays_o, rays_d, near, far, n, seed, perturb, out_t, out_x=None,
                         stream=None):
    _capi.check(_capi.lib().nerf_test_stratified(
        _ptr(rays_o), _ptr(rays_d), rays_o.shape[0], float(near), float(far), int(n), int(seed),
        int(perturb), _ptr(out_t), _ptr(out_x), _stream(stream)))


def nerf_test_pe(x, L, out, stream=None):
    _capi.check(_capi.lib().nerf_test_pe(_ptr(x), x.shape[0], int(L), _ptr(out), _stream(stream)))


def nerf_test_composite(raw, t, rays_d, far, last_delta_mode, march_step, sigma_act, white_bkgd,
                        out_rgb, out_depth, out_acc, out_weights=None, stream=None):
    R, S = t.shape
    _capi.check(_capi.lib().nerf_test_composite(
        _ptr(raw), _ptr(t), _ptr(rays_d), R, S, float(far), int(last_delta_mode),
        float(march_step), int(sigma_act), int(white_bkgd), _ptr(out_rgb), _ptr(out_depth),
        _ptr(out_acc), _ptr(out_weights), _stream(stream)))


def nerf_test_sample_pdf(t_coarse, weights, n_fine, seed, perturb, out_t_fine=None,
                         out_below=None, out_t_all=None, stream=None):
    R, Nc = t_coarse.shape
    _capi.check(_capi.lib().nerf_test_sample_pdf(
        _ptr(t_coarse), _ptr(weights), R, Nc, int(n_fine), int(seed), int(perturb),
        _ptr(out_t_fine), _ptr(out_below), _ptr(out_t_all), _stream(stream)))


def nerf_test_march(rays_o, rays_d, near, step, K, occupancy, out_count, out_live=None,
                    stream=None):
    _capi.check(_capi.lib().nerf_test_march(
        _ptr(rays_o), _ptr(rays_d), rays_o.shape[0], float(near), float(step), int(K),
        _ptr(occupancy), _ptr(out_count), _ptr(out_live), _stream(stream)))


def nerf_test_route_cells(x, out_cell, out_cell_count, out_cell_offset, out_order=None,
                          stream=None):
    _capi.check(_capi.lib().nerf_test_route_cells(
        _ptr(x), x.shape[0], _ptr(out_cell), _ptr(out_cell_count), _ptr(out_cell_offset),
        _ptr(out_order), _stream(stream)))


def nerf_test_hash_encode(x, hash_table, out_feat, out_rows=None, stream=None):
    _capi.check(_capi.lib().nerf_test_hash_encode(
        _ptr(x), x.shape[0], _ptr(hash_table), _ptr(out_feat), _ptr(out_rows), _stream(stream)))


def nerf_hash_encode_backward(x, d_feat, grad_table, deterministic=False, stream=None):
    """Scatter-add of encoding gradients into grad_table (accumulated); see the header."""
    _capi.check(_capi.lib().nerf_hash_encode_backward(_ptr(x), x.shape[0], _ptr(d_feat),
                                                      _ptr(grad_table), int(bool(deterministic)),
                                                      _stream(stream)))


def nerf_test_sh(d, out, stream=None):
    _capi.check(_capi.lib().nerf_test_sh(_ptr(d), d.shape[0], _ptr(out), _stream(stream)))


class Renderer:
    """Owns a nerf_ctx (nerf_create / nerf_destroy). The arguments are the fields
    of nerf_config (include/nerf.h): precision NERF_FP32 (fused CUDA-core
    network), NERF_BF16 (the 8x256 network on the tensor cores with bf16
    weights) or NERF_TF32 (fp32 weights, the layers on the tensor cores as
    three tf32 products each, at fp32-level accuracy; W of 128 or 256)."""

    def __init__(self, model=NERF_MODEL_MLP, D=8, W=256, skip=4, L_pos=10, L_dir=4,
                 sigma_act=NERF_SIGMA_RELU, precision=NERF_FP32, last_delta_mode=NERF_LAST_1E10,
                 white_bkgd=0, max_rays=1 << 16, max_samples=192):
        self.cfg = nerf_config(model, D, W, skip, L_pos, L_dir, sigma_act, precision,
                               last_delta_mode, white_bkgd, max_rays, max_samples)
        h = ctypes.c_void_p()
        _capi.check(_capi.lib().nerf_create(ctypes.byref(self.cfg), ctypes.byref(h)))
        self.ctx = h

    def close(self):
        if getattr(self, "ctx", None):
            _capi.lib().nerf_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    @staticmethod
    def params(coarse_w=None, fine_w=None, occupancy=None, cell_w=None, hash_table=None,
               hash_mlp=None, march_step=0.0, ert_T=0.0, seed=0, perturb=1):
        """A nerf_params holding the device pointers of the given tensors. The
        library reads the tensors through these pointers on every call, so the
        returned object keeps references to them: they stay allocated for as long
        as it is alive, and a temporary passed here cannot be freed and its
        memory reused while the params are in use."""
        p = nerf_params()
        p._tensors = tuple(t for t in (coarse_w, fine_w, occupancy, cell_w, hash_table, hash_mlp)
                           if t is not None)
        p.coarse_w = coarse_w.data_ptr() if coarse_w is not None else None
        p.fine_w = fine_w.data_ptr() if fine_w is not None else None
        p.occupancy = occupancy.data_ptr() if occupancy is not None else None
        p.cell_w = cell_w.data_ptr() if cell_w is not None else None
        p.hash_table = hash_table.data_ptr() if hash_table is not None else None
        p.hash_mlp = hash_mlp.data_ptr() if hash_mlp is not None else None
        p.march_step = march_step
        p.ert_T = ert_T
        p.seed = seed
        p.perturb = perturb
        return p

    def render(self, rays_o, rays_d, near, far, n_coarse, n_fine, params, out_rgb, out_depth,
               out_acc, stream=None):
        _capi.check(_capi.lib().nerf_render(
            self.ctx, _ptr(rays_o), _ptr(rays_d), rays_o.shape[0], float(near), float(far),
            int(n_coarse), int(n_fine), ctypes.byref(params), _ptr(out_rgb), _ptr(out_depth),
            _ptr(out_acc), _stream(stream)), self.ctx)

    def render_trace(self, rays_o, rays_d, near, far, n_coarse, n_fine, params, out_rgb,
                     out_depth, out_acc, raw_coarse=None, w_coarse=None, t_fine=None, below=None,
                     t_all=None, raw_fine=None, stream=None):
        """nerf_render that also copies the render's intermediates into the given
        CUDA tensors (any may be None); see nerf_render_trace."""
        tr = _capi.nerf_trace(*[t.data_ptr() if t is not None else None for t in
                                (raw_coarse, w_coarse, t_fine, below, t_all, raw_fine)])
        for t in (raw_coarse, w_coarse, t_fine, below, t_all, raw_fine):
            _ptr(t)                                       # device and contiguous
        _capi.check(_capi.lib().nerf_render_trace(
            self.ctx, _ptr(rays_o), _ptr(rays_d), rays_o.shape[0], float(near), float(far),
            int(n_coarse), int(n_fine), ctypes.byref(params), _ptr(out_rgb), _ptr(out_depth),
            _ptr(out_acc), ctypes.byref(tr), _stream(stream)), self.ctx)

    def loss_grad(self, rays_o, rays_d, near, far, n_coarse, n_fine, params, target_rgb,
                  out_loss, grad_coarse, grad_fine=None, stream=None):
        """Training-step loss and gradients (fp32 contexts); see nerf_loss_grad."""
        _capi.check(_capi.lib().nerf_loss_grad(
            self.ctx, _ptr(rays_o), _ptr(rays_d), rays_o.shape[0], float(near), float(far),
            int(n_coarse), int(n_fine), ctypes.byref(params), _ptr(target_rgb), _ptr(out_loss),
            _ptr(grad_coarse), _ptr(grad_fine), _stream(stream)), self.ctx)

    def render_host(self, rays_o, rays_d, near, far, n_coarse, n_fine, params, out_rgb, out_depth,
                    out_acc, stream=None):
        _capi.check(_capi.lib().nerf_render_host(
            self.ctx, _hptr(rays_o), _hptr(rays_d), rays_o.shape[0], float(near), float(far),
            int(n_coarse), int(n_fine), ctypes.byref(params), _hptr(out_rgb), _hptr(out_depth),
            _hptr(out_acc), _stream(stream)), self.ctx)

    def test_mlp(self, weights, x, d, out_raw, stream=None):
        _capi.check(_capi.lib().nerf_test_mlp(self.ctx, _ptr(weights), _ptr(x), _ptr(d),
                                              x.shape[0], _ptr(out_raw), _stream(stream)),
                    self.ctx)

    def timing_enable(self, enable=True):
        _capi.check(_capi.lib().nerf_timing_enable(self.ctx, int(enable)), self.ctx)

    def timing_read(self):
        """(summed network-kernel ms, number of timed launches) since the last read."""
        ms = ctypes.c_double()
        n = ctypes.c_int64()
        _capi.check(_capi.lib().nerf_timing_read(self.ctx, ctypes.byref(ms), ctypes.byref(n)),
                    self.ctx)
        return ms.value, n.value

    def timing_read_kinds(self):
        """{kernel class: (summed ms, launches)} since the last read, for every
        class of nerf_timing_read_kinds."""
        n = len(_capi.TIMED_KINDS)
        ms = (ctypes.c_double * n)()
        cnt = (ctypes.c_int64 * n)()
        _capi.check(_capi.lib().nerf_timing_read_kinds(self.ctx, ms, cnt), self.ctx)
        return {k: (ms[i], cnt[i]) for i, k in enumerate(_capi.TIMED_KINDS)}

    def sync_status(self, stream=None):
        _capi.check(_capi.lib().nerf_sync_status(self.ctx, _stream(stream)), self.ctx)
