"""Oracle for the NeRF render path: ray generation, stratified sampling, positional
encoding, the scene MLP, volume rendering, inverse-CDF resampling and the fine
pass. Test infrastructure only (see oracle/__init__.py).

Every function follows "Spatial Intelligence - Part 1: NeRF" (the NeRF page);
the section of the page is cited in each docstring.
"""
from __future__ import annotations

import numpy as np

from . import rng

F32 = np.float32


# --------------------------------------------------------------------------
# Ray generation (NeRF page, Section 2.2 "Ray generation", get_rays)
# --------------------------------------------------------------------------

def raygen(H: int, W: int, focal: float, c2w: np.ndarray):
    """Pinhole rays for every pixel, row-major (j over H outer, i over W inner).

    Camera-space direction ((i - W/2)/f, -(j - H/2)/f, -1), rotated by the upper
    3x3 of c2w and NOT normalised; origin = translation column. Evaluated in
    fp32 with products rounded and sums taken left to right, no fused
    multiply-add: d_r = (dx*c[r,0] + dy*c[r,1]) + dz*c[r,2].
    Returns (rays_o, rays_d), both fp32 [H*W, 3].
    """
    c = np.asarray(c2w, dtype=F32)
    j, i = np.meshgrid(np.arange(H, dtype=F32), np.arange(W, dtype=F32), indexing="ij")
    f = F32(focal)
    dx = (i - F32(W) * F32(0.5)) / f
    dy = -((j - F32(H) * F32(0.5)) / f)
    dz = F32(-1.0)
    d = np.empty((H, W, 3), dtype=F32)
    for r in range(3):
        d[..., r] = (dx * c[r, 0] + dy * c[r, 1]) + dz * c[r, 2]
    o = np.broadcast_to(c[:, 3], d.shape).astype(F32)
    return o.reshape(-1, 3), d.reshape(-1, 3)


# --------------------------------------------------------------------------
# Sampling along the ray (NeRF page, Section 1.4.2 "Hierarchical volume
# sampling": N_c stratified coarse samples; stratified_sample's body is not
# printed, so the usual reading is taken: N equal bins on [near, far] and one
# uniform jitter per bin)
# --------------------------------------------------------------------------

def stratified_t(near, far, n, seed, ray_ids, perturb=True):
    """t_i = near + (i + u_i) * (far - near) / n, i = 0..n-1, in fp32:
    step = fl((far - near) / n); s = fl(i + u); t = fl(near + fl(s * step)).
    u_i is draw (seed, ray, stream 0, i); without perturbation u = 0.5.
    Returns fp32 [len(ray_ids), n]."""
    ray_ids = np.asarray(ray_ids, dtype=np.int64)
    step = (F32(far) - F32(near)) / F32(n)
    idx = np.arange(n, dtype=np.int64)
    if perturb:
        u = rng.draw_uniform(seed, ray_ids[:, None], 0, idx[None, :]).astype(F32)
    else:
        u = np.full((len(ray_ids), n), 0.5, dtype=F32)
    s = idx.astype(F32)[None, :] + u
    return F32(near) + s * step


def march_t(near, step, n):
    """Fixed-step candidates t_k = fl(near + fl(k * step)), k = 0..n-1 (fp32)."""
    k = np.arange(n, dtype=F32)
    return F32(near) + k * F32(step)


def points(o, d, t):
    """x = o + t d for every sample (NeRF page, Section 1.3: r(t) = o + t d),
    evaluated in fp32 as fl(o + fl(t * d)). o, d fp32 [R,3]; t fp32 [R,S]."""
    o = np.asarray(o, dtype=F32)[:, None, :]
    d = np.asarray(d, dtype=F32)[:, None, :]
    t = np.asarray(t, dtype=F32)[..., None]
    return o + t * d


# --------------------------------------------------------------------------
# Positional encoding (NeRF page, Section 1.4.1, gamma(x); layout of the
# positional_encoding listing in Section 2.3)
# --------------------------------------------------------------------------

def positional_encoding(x, L: int):
    """gamma(x) = [x, sin(2^k pi x_c), cos(2^k pi x_c)] with the sin block and
    the cos block each ordered coordinate-major (index c*L + k), 3 + 6L values.
    The pi factor of the page's formula is kept. fp64."""
    x = np.asarray(x, dtype=np.float64)
    freqs = 2.0 ** np.arange(L, dtype=np.float64)
    ang = np.pi * x[..., :, None] * freqs            # [..., 3, L]
    sins = np.sin(ang).reshape(*x.shape[:-1], -1)
    coss = np.cos(ang).reshape(*x.shape[:-1], -1)
    return np.concatenate([x, sins, coss], axis=-1)


def unit(d):
    """Viewing direction d / ||d|| (fp64)."""
    d = np.asarray(d, dtype=np.float64)
    return d / np.linalg.norm(d, axis=-1, keepdims=True)


# --------------------------------------------------------------------------
# Scene MLP F_theta (NeRF page, Section 2.4 "The NeRF network")
# --------------------------------------------------------------------------

def split_params(shape, flat):
    """Slice a flat parameter blob (layer order of synth.MLPShape) into
    name -> (W [N,K], b [N]) in fp64."""
    flat = np.asarray(flat, dtype=np.float64)
    out, off = {}, 0
    for name, n, k in shape.layer_shapes():
        w = flat[off:off + n * k].reshape(n, k)
        off += n * k
        b = flat[off:off + n]
        off += n
        out[name] = (w, b)
    assert off == flat.size
    return out


def relu(a):
    return np.maximum(a, 0.0)


def nerf_mlp(shape, params, pts_enc, dir_enc):
    """Raw network output [rgb(3), sigma] per point.

    D layers of width W with ReLU; after layer `skip` the hidden state is
    concatenated with gamma(x) (hidden first); sigma = Linear(W,1)(h) and
    feature = Linear(W,W)(h), both without activation; h' = ReLU(Linear(W +
    dir_ch, W/2)([feature, gamma(d)])); rgb = Linear(W/2, 3)(h')."""
    h = pts_enc
    for i in range(shape.D):
        w, b = params[f"pts{i}"]
        h = relu(h @ w.T + b)
        if i == shape.skip:
            h = np.concatenate([h, pts_enc], axis=-1)
    ws, bs = params["sigma"]
    wf, bf = params["feature"]
    wd, bd = params["dir"]
    wr, br = params["rgb"]
    sigma = h @ ws.T + bs
    feature = h @ wf.T + bf
    h = relu(np.concatenate([feature, dir_enc], axis=-1) @ wd.T + bd)
    rgb = h @ wr.T + br
    return np.concatenate([rgb, sigma], axis=-1)


# --------------------------------------------------------------------------
# Volume rendering (NeRF page, Section 1.3 discrete quadrature; Section 2.5
# "Volume rendering in code")
# --------------------------------------------------------------------------

def sigmoid(a):
    return 1.0 / (1.0 + np.exp(-a))


def softplus(a):
    a = np.asarray(a, dtype=np.float64)
    return np.where(a > 30.0, a, np.log1p(np.exp(np.minimum(a, 30.0))))


def sigma_activation(raw_sigma, sigma_act: int):
    return softplus(raw_sigma) if sigma_act == 1 else relu(raw_sigma)


def deltas(t, d_norm, last_mode: int, far=None, step=None):
    """delta_i = (t_{i+1} - t_i) * ||d||; the last interval is 1e10 (the page's
    volume_render, mode 0), far - t_last (mode 1, the closed-form reading of
    T(t) on [t_n, t_f]), or the march step (mode 2). fp64."""
    t = np.asarray(t, dtype=np.float64)
    dist = t[..., 1:] - t[..., :-1]
    if last_mode == 0:
        last = np.full(t.shape[:-1] + (1,), 1e10)
    elif last_mode == 1:
        last = (far - t[..., -1:])
    else:
        last = np.full(t.shape[:-1] + (1,), float(step))
    dist = np.concatenate([dist, last], axis=-1)
    return dist * np.asarray(d_norm, dtype=np.float64)[..., None]


def composite(sigma, rgb, t, delta, white_bkgd=False):
    """Alpha compositing along each ray.

    alpha_i = 1 - exp(-sigma_i delta_i); T_i = prod_{j<i} (1 - alpha_j) =
    exp(-sum_{j<i} sigma_j delta_j); w_i = T_i alpha_i; C = sum w_i c_i;
    depth = sum w_i t_i (in t units, not divided by acc); acc = sum w_i;
    white background adds 1 - acc. The page's 1e-10 survival guard is not
    applied (the guard-free definition of T_i is the quantity approximated).
    sigma, t, delta [R,S]; rgb [R,S,3] (already activated). fp64.
    Returns rgb [R,3], depth [R], acc [R], weights [R,S]."""
    tau = np.asarray(sigma, dtype=np.float64) * np.asarray(delta, dtype=np.float64)
    excl = np.concatenate([np.zeros(tau.shape[:-1] + (1,)), np.cumsum(tau, axis=-1)[..., :-1]],
                          axis=-1)
    T = np.exp(-excl)
    alpha = -np.expm1(-tau)
    w = T * alpha
    acc = w.sum(-1)
    out = (w[..., None] * rgb).sum(-2)
    if white_bkgd:
        out = out + (1.0 - acc)[..., None]
    depth = (w * np.asarray(t, dtype=np.float64)).sum(-1)
    return out, depth, acc, w


# --------------------------------------------------------------------------
# Inverse-CDF resampling (NeRF page, Section 1.4.2 and Section 2.6
# "Hierarchical sampling", sample_pdf)
# --------------------------------------------------------------------------

def midpoints(t):
    """Bin edges for the fine pass: fl(0.5 * fl(t_i + t_{i+1})) in fp32."""
    t = np.asarray(t, dtype=F32)
    return F32(0.5) * (t[..., 1:] + t[..., :-1])


def sample_pdf(bins, weights, m):
    """Inverse-CDF draws from the piecewise-constant pdf of `weights` over `bins`.

    bins  fp32 [R, nb] (nb = len(weights) + 1 edges)
    weights [R, nb-1] (any float; the decision uses their fp32 values)
    m     int [R, N]: draws u = m * 2^-24
    Follows sample_pdf: weights + 1e-5, pdf = w / sum, cdf = cumsum with a
    leading 0, idx = searchsorted(cdf, u, right=True), below = max(idx-1, 0),
    above = min(idx, nb-1), t = b_below + (u - cdf_below) / max(cdf_above -
    cdf_below, 1e-5) * (b_above - b_below).

    The CDF is evaluated exactly: q_i = floor(fl32(w_i + 1e-5) * 2^32) as
    integers, C_k = sum_{i<k} q_i (C_0 = 0), and cdf_k <= u  <=>  C_k * 2^24 <=
    m * C_total. The interpolation is then fp64.
    Returns (t fp64 [R,N], below int [R,N])."""
    bins = np.asarray(bins, dtype=F32)
    wq = np.asarray(weights, dtype=F32) + F32(1e-5)
    q = np.floor(wq.astype(np.float64) * 2.0 ** 32).astype(np.uint64)
    C = np.concatenate([np.zeros(q.shape[:-1] + (1,), dtype=np.uint64), np.cumsum(q, axis=-1)],
                       axis=-1)                                   # [R, nb]
    total = C[..., -1:]
    m = np.asarray(m, dtype=np.uint64)
    lhs = C[:, None, :] * np.uint64(1 << 24)                      # [R,1,nb]
    rhs = (m * total)[..., None]                                  # [R,N,1]
    idx = (lhs <= rhs).sum(-1).astype(np.int64)                   # searchsorted right
    nb = C.shape[-1]
    below = np.maximum(idx - 1, 0)
    above = np.minimum(idx, nb - 1)
    cb = np.take_along_axis(C, below, axis=-1)
    ca = np.take_along_axis(C, above, axis=-1)
    num = (m * total - cb * np.uint64(1 << 24)).astype(np.float64)
    den = 2.0 ** 24 * np.maximum((ca - cb).astype(np.float64), 1e-5 * total.astype(np.float64))
    frac = num / den
    bb = np.take_along_axis(bins, below, axis=-1).astype(np.float64)
    ba = np.take_along_axis(bins, above, axis=-1).astype(np.float64)
    return bb + frac * (ba - bb), below


# --------------------------------------------------------------------------
# render_rays (NeRF page, Section 2.6: coarse pass -> sample_pdf -> sorted
# union -> fine pass; the final image is the fine output)
# --------------------------------------------------------------------------

def render_nerf(wl, o, d, ray_ids, coarse_flat, fine_flat=None, seed=None, perturb=True,
                chunk=512, return_aux=False, raw_noise=None):
    """Render rays (o, d fp32 [R,3], global indices ray_ids) with workload `wl`
    (a nerf_inputs.Workload). Returns dict with rgb [R,3], depth [R], acc [R]
    (fp64) and, with return_aux, the intermediates of both passes.

    raw_noise = (seed, rel, abs) is a conditioning probe for the tests, never
    part of the reference result: it perturbs every raw network output as
    raw * (1 + rel * n1) + abs * n2 with seeded standard normals, to measure how
    far a ray's result moves when the network is evaluated at a lower working
    precision (resampling and the page-mode last interval can amplify it)."""
    noise_rng = np.random.default_rng(raw_noise[0]) if raw_noise else None

    def net(shape, params, oo, dd, t, denc):
        out = _eval(shape, params, oo, dd, t, denc)
        if noise_rng is not None:
            out = (out * (1.0 + raw_noise[1] * noise_rng.standard_normal(out.shape))
                   + raw_noise[2] * noise_rng.standard_normal(out.shape))
        return out
    shape = wl.mlp
    seed = wl.seed if seed is None else seed
    pc = split_params(shape, coarse_flat)
    pf = split_params(shape, fine_flat) if fine_flat is not None else None
    o = np.asarray(o, dtype=F32)
    d = np.asarray(d, dtype=F32)
    ray_ids = np.asarray(ray_ids, dtype=np.int64)
    R = len(ray_ids)
    res = {k: [] for k in ("rgb", "depth", "acc", "t_c", "w_c", "t_f", "t_all", "below",
                           "rgb_c", "acc_c", "sigma_last_raw", "raw_final", "t_final")}
    for s in range(0, R, chunk):
        sl = slice(s, min(R, s + chunk))
        oo, dd, ids = o[sl], d[sl], ray_ids[sl]
        dn = np.linalg.norm(dd.astype(np.float64), axis=-1)
        denc = positional_encoding(unit(dd), shape.L_dir)
        # coarse pass
        t_c = stratified_t(wl.near, wl.far, wl.n_coarse, seed, ids, perturb)
        raw = net(shape, pc, oo, dd, t_c, denc)
        sig = sigma_activation(raw[..., 3], wl.sigma_act)
        col = sigmoid(raw[..., :3])
        delta = deltas(t_c, dn, wl.last_delta, far=wl.far)
        rgb_c, dep_c, acc_c, w_c = composite(sig, col, t_c, delta, wl.white_bkgd)
        res["t_c"].append(t_c)
        res["w_c"].append(w_c)
        res["rgb_c"].append(rgb_c)
        res["acc_c"].append(acc_c)
        if wl.n_fine == 0:
            res["sigma_last_raw"].append(raw[:, -1, 3])
            res["raw_final"].append(raw)
            res["t_final"].append(t_c)
            res["rgb"].append(rgb_c)
            res["depth"].append(dep_c)
            res["acc"].append(acc_c)
            continue
        # fine pass: the sample positions are fp32 values (the page keeps z_vals
        # in fp32 tensors), so the drawn t's are rounded to fp32 before the sort
        bins = midpoints(t_c)
        if perturb:
            m = rng.draw_bits(seed, ids[:, None], 1, np.arange(wl.n_fine)[None, :])
        else:
            m = np.broadcast_to(((np.arange(wl.n_fine) * 2 + 1) << 23) // wl.n_fine,
                                (len(ids), wl.n_fine)).astype(np.int64)
        t_f, below = sample_pdf(bins, w_c[:, 1:-1], m)
        t_f = t_f.astype(F32)
        t_all = np.sort(np.concatenate([t_c, t_f], axis=-1), axis=-1)
        raw = net(shape, pf, oo, dd, t_all, denc)
        sig = sigma_activation(raw[..., 3], wl.sigma_act)
        col = sigmoid(raw[..., :3])
        delta = deltas(t_all, dn, wl.last_delta, far=wl.far)
        rgb, dep, acc, _ = composite(sig, col, t_all, delta, wl.white_bkgd)
        res["sigma_last_raw"].append(raw[:, -1, 3])
        res["raw_final"].append(raw)
        res["t_final"].append(t_all)
        res["rgb"].append(rgb)
        res["depth"].append(dep)
        res["acc"].append(acc)
        res["t_f"].append(t_f)
        res["t_all"].append(t_all)
        res["below"].append(below)
    out = {k: np.concatenate(v, axis=0) for k, v in res.items() if v}
    if not return_aux:
        out = {k: out[k] for k in ("rgb", "depth", "acc")}
    return out


def _eval(shape, params, o, d, t, denc):
    x = points(o, d, t)                                        # fp32 [R,S,3]
    penc = positional_encoding(x.astype(np.float64), shape.L_pos)
    de = np.broadcast_to(denc[:, None, :], penc.shape[:-1] + (denc.shape[-1],))
    return nerf_mlp(shape, params, penc, de)


def network_pass(wl, flat, o, d, t, chunk=256):
    """One network pass of render_rays at given sample positions: the raw
    outputs [R,S,4] of F_theta (parameters `flat`, the workload's shape) at the
    points fl(o + fl(t d)) seen from d / ||d|| (NeRF page, Sections 2.3-2.4).
    o, d fp32 [R,3]; t fp32 [R,S]. fp64."""
    shape = wl.mlp
    params = split_params(shape, flat)
    o = np.asarray(o, dtype=F32)
    d = np.asarray(d, dtype=F32)
    t = np.asarray(t, dtype=F32)
    out = []
    for s in range(0, len(o), chunk):
        sl = slice(s, s + chunk)
        denc = positional_encoding(unit(d[sl]), shape.L_dir)
        out.append(_eval(shape, params, o[sl], d[sl], t[sl], denc))
    return np.concatenate(out, axis=0)


def composite_pass(wl, raw, t, d):
    """Volume rendering of one pass of render_rays from its raw network outputs
    (NeRF page, Section 2.5 volume_render): sigma = act(raw_sigma), c =
    sigmoid(raw_rgb), the workload's last interval, then `composite`.
    raw [R,S,4], t fp32 [R,S], d [R,3]. Returns rgb, depth, acc, weights (fp64)."""
    raw = np.asarray(raw, dtype=np.float64)
    dn = np.linalg.norm(np.asarray(d, dtype=F32).astype(np.float64), axis=-1)
    sig = sigma_activation(raw[..., 3], wl.sigma_act)
    col = sigmoid(raw[..., :3])
    delta = deltas(t, dn, wl.last_delta, far=wl.far)
    return composite(sig, col, t, delta, wl.white_bkgd)
