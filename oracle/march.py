"""Oracle for the marching scene functions: occupancy-grid empty-space skipping,
early ray termination, the KiloNeRF grid of tiny MLPs and the hash-grid
network. Test infrastructure only.

Sources: the KiloNeRF page (abstract: the scene is split over thousands of tiny
MLPs, each responsible for part of the scene); the Instant-NGP notebook
(Experiment 2 "Key takeaway": hash lookups + a tiny MLP, with empty-space
skipping in 3D); compositing from the NeRF page (Section 1.3). Grid sizes,
step sizes and the termination threshold are the workload parameters, not page
facts.
"""
from __future__ import annotations

import numpy as np

from . import hashgrid, nerf, sh

F32 = np.float32
GRID_RES = 128
GRID_MIN = -1.5
VOXEL = 3.0 / 128.0
KILO_CELLS = 16


def voxel_coords(x):
    """Voxel of each fp32 point: the v with b_v <= x < b_{v+1}, b_k = -1.5 +
    k*3/128 (exact in fp32 and fp64), per axis; -1 outside [-1.5, 1.5)."""
    x = np.asarray(x, dtype=F32).astype(np.float64)
    edges = GRID_MIN + np.arange(GRID_RES + 1, dtype=np.float64) * VOXEL
    v = np.searchsorted(edges, x, side="right") - 1
    v[(x < edges[0]) | (x >= edges[-1])] = -1
    return v


def occupied(x, dense):
    """Occupancy-grid test of fp32 points against dense bool[128,128,128]."""
    v = voxel_coords(x)
    inside = (v >= 0).all(axis=-1)
    vv = np.where(v < 0, 0, v)
    return inside & dense[vv[..., 0], vv[..., 1], vv[..., 2]]


def cell_id(x):
    """KiloNeRF cell of a point inside the grid: (voxel >> 3) per axis,
    id = (cx*16 + cy)*16 + cz."""
    v = voxel_coords(x)
    c = v // (GRID_RES // KILO_CELLS)
    return (c[..., 0] * KILO_CELLS + c[..., 1]) * KILO_CELLS + c[..., 2]


def _layers(flat, layout):
    out, off = {}, 0
    for name, n, k in layout:
        out[name] = (flat[..., off:off + n * k].reshape(flat.shape[:-1] + (n, k)),
                     flat[..., off + n * k:off + n * k + n])
        off += n * k + n
    return out, off


def kilonerf_eval(cell_params, cells, x, d_unit, L_pos=10, L_dir=4):
    """Evaluate every point with its OWN cell's MLP (no grouping):
    h1 = ReLU(W1 gamma(x) + b1); h2 = ReLU(W2 h1 + b2); sigma = ReLU(w.h2 + b);
    rgb = sigmoid(Wc [h2, gamma(d)] + bc). cell_params fp32 [n_cells, 3317];
    cells int [P]; x fp32 [P,3]; d_unit fp64 [P,3]. Returns sigma [P], rgb [P,3]."""
    from nerf_inputs import kilonerf_layout
    p, _ = _layers(np.asarray(cell_params, dtype=np.float64)[cells], kilonerf_layout())
    pe = nerf.positional_encoding(np.asarray(x, dtype=np.float64), L_pos)
    de = nerf.positional_encoding(d_unit, L_dir)

    def lin(name, a):
        w, b = p[name]
        return np.einsum("pnk,pk->pn", w, a) + b

    h1 = nerf.relu(lin("l1", pe))
    h2 = nerf.relu(lin("l2", h1))
    sigma = nerf.relu(lin("sigma", h2))[:, 0]
    rgb = nerf.sigmoid(lin("rgb", np.concatenate([h2, de], axis=-1)))
    return sigma, rgb


def hash_eval(grid, table, mlp_flat, x, d_unit):
    """Hash-grid scene function: enc = encode(x) (32); h = ReLU(D1 ReLU(D0 enc));
    sigma = ReLU(w.h + b); c = ReLU(C1 ReLU(C0 [h, SH16(d)])); rgb =
    sigmoid(Wrgb c + b). Returns sigma [P], rgb [P,3]."""
    from nerf_inputs import hash_mlp_layout
    p, _ = _layers(np.asarray(mlp_flat, dtype=np.float64), hash_mlp_layout())

    def lin(name, a):
        w, b = p[name]
        return a @ w.T + b

    enc = grid.encode(x, table)
    h = nerf.relu(lin("d1", nerf.relu(lin("d0", enc))))
    sigma = nerf.relu(lin("sigma", h))[:, 0]
    c = nerf.relu(lin("c0", np.concatenate([h, sh.real_sh(d_unit)], axis=-1)))
    c = nerf.relu(lin("c1", c))
    rgb = nerf.sigmoid(lin("rgb", c))
    return sigma, rgb


def render_march(wl, o, d, dense, evaluate):
    """March each ray over t_k = near + k*step, k < n_coarse (fp32 positions).

    Only occupied samples are evaluated and composited (empty space leaves T
    unchanged); each contributes with delta = step * ||d||. With early ray
    termination (wl.ert_T > 0) the ray stops before the first occupied sample
    whose transmittance T_k = exp(-sum sigma delta) is below wl.ert_T.
    `evaluate(ray_idx, x, d_unit) -> (sigma, rgb)` is the scene function.
    Returns dict rgb [R,3], depth [R], acc [R], n_live [R] (samples evaluated),
    ert_margin [R] (min over checked samples of |T_k/ert_T - 1|), fp64."""
    o = np.asarray(o, dtype=F32)
    d = np.asarray(d, dtype=F32)
    R = o.shape[0]
    t_all = nerf.march_t(wl.near, wl.march_step, wl.n_coarse)
    dn = np.linalg.norm(d.astype(np.float64), axis=-1)
    du = nerf.unit(d)
    S = np.zeros(R)
    rgb = np.zeros((R, 3))
    depth = np.zeros(R)
    acc = np.zeros(R)
    alive = np.ones(R, dtype=bool)
    n_live = np.zeros(R, dtype=np.int64)
    margin = np.full(R, np.inf)
    for k in range(wl.n_coarse):
        t = t_all[k]
        x = o + t * d                                   # fp32: fl(o + fl(t d))
        occ = occupied(x, dense) & alive
        if wl.ert_T > 0:
            # the stop decision is taken in fp32, the precision of the kernel
            T = np.exp(-S)
            margin = np.where(occ, np.minimum(margin, np.abs(T / wl.ert_T - 1.0)), margin)
            stop = occ & (T.astype(F32) < F32(wl.ert_T))
            alive &= ~stop
            occ &= ~stop
        idx = np.nonzero(occ)[0]
        if idx.size == 0:
            continue
        sigma, col = evaluate(idx, x[idx], du[idx])
        tau = sigma * (wl.march_step * dn[idx])
        w = np.exp(-S[idx]) * -np.expm1(-tau)
        S[idx] += tau
        rgb[idx] += w[:, None] * col
        depth[idx] += w * float(t)
        acc[idx] += w
        n_live[idx] += 1
    return {"rgb": rgb, "depth": depth, "acc": acc, "n_live": n_live, "ert_margin": margin}
