"""Oracle for the NeRF training step: the loss and its parameter gradients.

TEST INFRASTRUCTURE ONLY. Only tests/, the smoke check and bench.py's CPU
baseline may import this module; the product path never does.

What it computes (NeRF page, "7. Training loop"): for a batch of R rays,
    loss = mse(rgb_coarse, target) + mse(rgb_fine, target),
each mse being the mean over the R x 3 colour values. The fine sample positions
come from the coarse weights with the weights detached ("6. Hierarchical
sampling": gradients do not flow back through the sampling step), so for the
gradient they are constants. The gradients are those of the loss with respect
to every parameter of the coarse and fine networks, returned as flat blobs in
the layer order of the network blob (for each Linear: W row-major [N][K], then
b).

The backward is the chain rule applied to the forward definitions of
oracle.nerf: compositing (Section 1.3 / 2.5), the scene MLP F_theta (Section
2.4). Where the pages leave an activation's derivative at its kink open, the
ReLU's derivative at 0 is taken as 0 (the sub-gradient frameworks use). Parity
is pinned in tests by central finite differences of the same loss with the
positions held fixed. fp64 throughout.
"""
from __future__ import annotations

import numpy as np

from . import nerf as onerf
from . import rng

F32 = np.float32


# --------------------------------------------------------------------------
# Scene MLP with the intermediates kept, and its backward
# --------------------------------------------------------------------------

def mlp_forward_cache(shape, params, penc, denc):
    """nerf_mlp with every layer's input and output kept. penc [M, 63],
    denc [M, 27] (fp64). Returns raw [M, 4] and the cache."""
    h = penc
    ins, outs = [], []
    for i in range(shape.D):
        w, b = params[f"pts{i}"]
        ins.append(h)
        h = onerf.relu(h @ w.T + b)
        outs.append(h)
        if i == shape.skip:
            h = np.concatenate([h, penc], axis=-1)
    h_last = outs[-1]
    ws, bs = params["sigma"]
    wf, bf = params["feature"]
    wd, bd = params["dir"]
    wr, br = params["rgb"]
    sigma = h_last @ ws.T + bs
    feature = h_last @ wf.T + bf
    din = np.concatenate([feature, denc], axis=-1)
    hdir = onerf.relu(din @ wd.T + bd)
    rgb = hdir @ wr.T + br
    cache = dict(ins=ins, outs=outs, h_last=h_last, din=din, hdir=hdir)
    return np.concatenate([rgb, sigma], axis=-1), cache


def mlp_backward(shape, params, cache, d_raw):
    """Gradients of sum(d_raw * raw) with respect to every parameter.
    d_raw [M, 4] = (d rgb_raw, d sigma_raw). Returns name -> (dW [N,K], db [N])."""
    g = {}
    W = shape.W
    d_rgb, d_sig = d_raw[:, :3], d_raw[:, 3:4]
    hdir, din, h_last = cache["hdir"], cache["din"], cache["h_last"]
    wr, _ = params["rgb"]
    wd, _ = params["dir"]
    wf, _ = params["feature"]
    ws, _ = params["sigma"]
    g["rgb"] = (d_rgb.T @ hdir, d_rgb.sum(0))
    dz = (d_rgb @ wr) * (hdir > 0)
    g["dir"] = (dz.T @ din, dz.sum(0))
    d_feat = (dz @ wd)[:, :W]
    g["feature"] = (d_feat.T @ h_last, d_feat.sum(0))
    g["sigma"] = (d_sig.T @ h_last, d_sig.sum(0))
    dh = d_feat @ wf + d_sig @ ws
    for i in reversed(range(shape.D)):
        w, _ = params[f"pts{i}"]
        dz = dh * (cache["outs"][i] > 0)
        g[f"pts{i}"] = (dz.T @ cache["ins"][i], dz.sum(0))
        if i > 0:
            dh = (dz @ w)[:, :W]   # the skip layer's gamma(x) columns carry no parameters
    return g


def flatten_grads(shape, g):
    parts = []
    for name, n, k in shape.layer_shapes():
        dw, db = g[name]
        assert dw.shape == (n, k) and db.shape == (n,)
        parts.append(dw.ravel())
        parts.append(db)
    return np.concatenate(parts)


# --------------------------------------------------------------------------
# Compositing backward
# --------------------------------------------------------------------------

def composite_backward(sigma_raw, col_raw, delta, sigma_act, white_bkgd, d_rgb):
    """Gradients of sum(d_rgb * rgb) through rgb = sum_i w_i sigmoid(c_i)
    (+ 1 - acc on a white background), w_i = T_i alpha_i, alpha_i = 1 -
    exp(-sigma_i delta_i), T_i = exp(-sum_{j<i} sigma_j delta_j).
    sigma_raw [R,S], col_raw [R,S,3], delta [R,S], d_rgb [R,3].
    Returns d_sigma_raw [R,S], d_col_raw [R,S,3]."""
    sig = onerf.sigma_activation(sigma_raw, sigma_act)
    s = onerf.sigmoid(col_raw)
    tau = sig * delta
    excl = np.concatenate([np.zeros(tau.shape[:-1] + (1,)), np.cumsum(tau, -1)[..., :-1]], -1)
    T = np.exp(-excl)
    alpha = -np.expm1(-tau)
    w = T * alpha
    T_next = T * np.exp(-tau)                                   # T_{i+1}
    ws = w[..., None] * s                                       # w_j s_j
    # sum over j > i of w_j s_j (and of w_j), per sample i
    after_ws = np.cumsum(ws[..., ::-1, :], -2)[..., ::-1, :] - ws
    after_w = np.cumsum(w[..., ::-1], -1)[..., ::-1] - w
    d_tau = ((T_next[..., None] * s - after_ws) * d_rgb[:, None, :]).sum(-1)
    if white_bkgd:
        d_tau = d_tau - (T_next - after_w) * d_rgb.sum(-1, keepdims=True)
    d_sigma = d_tau * delta
    if sigma_act == 1:
        d_sigma_raw = d_sigma * onerf.sigmoid(sigma_raw)        # softplus'
    else:
        d_sigma_raw = d_sigma * (sigma_raw > 0)
    d_col_raw = d_rgb[:, None, :] * w[..., None] * s * (1.0 - s)
    return d_sigma_raw, d_col_raw


# --------------------------------------------------------------------------
# The training step's loss and gradients
# --------------------------------------------------------------------------

def sample_positions(wl, o, d, ray_ids, coarse_flat, seed=None, perturb=True):
    """Coarse stratified positions t_c [R, n_coarse] and, when wl.n_fine > 0, the
    sorted union t_all [R, n_coarse + n_fine] (fp32), drawn from the detached
    coarse weights exactly as oracle.nerf.render_nerf draws them."""
    shape = wl.mlp
    seed = wl.seed if seed is None else seed
    pc = onerf.split_params(shape, coarse_flat)
    o = np.asarray(o, dtype=F32)
    d = np.asarray(d, dtype=F32)
    ids = np.asarray(ray_ids, dtype=np.int64)
    t_c = onerf.stratified_t(wl.near, wl.far, wl.n_coarse, seed, ids, perturb)
    if wl.n_fine == 0:
        return t_c, None
    dn = np.linalg.norm(d.astype(np.float64), axis=-1)
    denc = onerf.positional_encoding(onerf.unit(d), shape.L_dir)
    raw = onerf._eval(shape, pc, o, d, t_c, denc)
    sig = onerf.sigma_activation(raw[..., 3], wl.sigma_act)
    col = onerf.sigmoid(raw[..., :3])
    delta = onerf.deltas(t_c, dn, wl.last_delta, far=wl.far)
    _, _, _, w_c = onerf.composite(sig, col, t_c, delta, wl.white_bkgd)
    bins = onerf.midpoints(t_c)
    if perturb:
        m = rng.draw_bits(seed, ids[:, None], 1, np.arange(wl.n_fine)[None, :])
    else:
        m = np.broadcast_to(((np.arange(wl.n_fine) * 2 + 1) << 23) // wl.n_fine,
                            (len(ids), wl.n_fine)).astype(np.int64)
    t_f, _ = onerf.sample_pdf(bins, w_c[:, 1:-1], m)
    t_all = np.sort(np.concatenate([t_c, t_f.astype(F32)], axis=-1), axis=-1)
    return t_c, t_all


def _pass(wl, params, o, d, t, target, n_total, want_grad):
    """One pass (a network over fixed positions t): its mse term and, if asked,
    the gradient of that term."""
    shape = wl.mlp
    R, S = t.shape
    x = onerf.points(o, d, t)
    penc = onerf.positional_encoding(x.astype(np.float64), shape.L_pos).reshape(R * S, -1)
    denc = onerf.positional_encoding(onerf.unit(d), shape.L_dir)
    denc_rows = np.repeat(denc, S, axis=0)
    raw, cache = mlp_forward_cache(shape, params, penc, denc_rows)
    raw = raw.reshape(R, S, 4)
    sig = onerf.sigma_activation(raw[..., 3], wl.sigma_act)
    col = onerf.sigmoid(raw[..., :3])
    dn = np.linalg.norm(np.asarray(d, dtype=np.float64), axis=-1)
    delta = onerf.deltas(t, dn, wl.last_delta, far=wl.far)
    rgb, _, _, _ = onerf.composite(sig, col, t, delta, wl.white_bkgd)
    err = rgb - target
    term = float((err ** 2).sum()) / (3.0 * n_total)
    if not want_grad:
        return term, None, rgb
    d_rgb = 2.0 * err / (3.0 * n_total)
    d_sig, d_col = composite_backward(raw[..., 3], raw[..., :3], delta, wl.sigma_act,
                                      wl.white_bkgd, d_rgb)
    d_raw = np.concatenate([d_col, d_sig[..., None]], axis=-1).reshape(R * S, 4)
    return term, mlp_backward(shape, params, cache, d_raw), rgb


def loss_and_grad(wl, o, d, ray_ids, target, coarse_flat, fine_flat=None, seed=None,
                  perturb=True, positions=None, want_grad=True, chunk=256):
    """The training step's loss (a float) and the gradient blobs (fp64 arrays in
    blob order; grad_fine is None without a fine pass). `positions` = (t_c,
    t_all) from sample_positions fixes the sample positions (the finite-
    difference pins hold them while the parameters move)."""
    shape = wl.mlp
    o = np.asarray(o, dtype=F32)
    d = np.asarray(d, dtype=F32)
    target = np.asarray(target, dtype=np.float64)
    R = len(o)
    if positions is None:
        positions = sample_positions(wl, o, d, ray_ids, coarse_flat, seed, perturb)
    t_c, t_all = positions
    pc = onerf.split_params(shape, coarse_flat)
    pf = onerf.split_params(shape, fine_flat) if t_all is not None else None
    loss = 0.0
    gc = gf = None
    for s0 in range(0, R, chunk):
        sl = slice(s0, min(R, s0 + chunk))
        term, g, _ = _pass(wl, pc, o[sl], d[sl], t_c[sl], target[sl], R, want_grad)
        loss += term
        if want_grad:
            gc = g if gc is None else {k: (gc[k][0] + g[k][0], gc[k][1] + g[k][1]) for k in gc}
        if t_all is not None:
            term, g, _ = _pass(wl, pf, o[sl], d[sl], t_all[sl], target[sl], R, want_grad)
            loss += term
            if want_grad:
                gf = g if gf is None else {k: (gf[k][0] + g[k][0], gf[k][1] + g[k][1]) for k in gf}
    if not want_grad:
        return loss, None, None
    return (loss, flatten_grads(shape, gc),
            flatten_grads(shape, gf) if gf is not None else None)
