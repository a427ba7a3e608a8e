"""Pins of the oracle's scene functions that hold by construction, with no
implementation to compare against:

- the 3D hash-grid encoding reproduces a linear function of the vertex
  coordinates exactly (the Instant-NGP notebook's bilinear interpolation,
  HashGrid2D.encode, made trilinear: interpolation of a linear function is
  exact), which fixes the orientation of every corner weight and the axis
  order of the direct index;
- the hash-grid network routes an encoding feature to sigma through d0, d1
  and the sigma head, and the view encoding into the colour branch after the
  64 density features ([h, SH16], in that order);
- a KiloNeRF cell network routes gamma(x) through l1 and l2 to sigma, and its
  colour head reads [h2, gamma(d)] in that order.

Each pin is a function so that tests/test_oracle_mutations.py can show that
it fails when the mistake it guards is planted in the oracle."""
import math

import numpy as np

import nerf_inputs as S
from oracle import hashgrid, march, nerf


# ------------------------------------------------------------------ hash encoding

def _linear_tables(grid, coef):
    """Table rows of the direct levels holding f(ix, iy, iz) = coef . (ix, iy, iz,
    1) / N per feature (coef: [F][4]); hashed levels hold zeros."""
    table = np.zeros((grid.n_entries, grid.F), dtype=np.float64)
    for level, N in enumerate(grid.res):
        if not grid.direct[level]:
            continue
        ix, iy, iz = np.meshgrid(np.arange(N + 1), np.arange(N + 1), np.arange(N + 1),
                                 indexing="ij")
        idx = hashgrid.index_3d(ix.ravel(), iy.ravel(), iz.ravel(), N, grid.T, True)
        for f in range(grid.F):
            a, b, c, e = coef[f]
            table[grid.offsets[level] + idx, f] = (a * ix.ravel() + b * iy.ravel()
                                                   + c * iz.ravel()) / N + e
    return table


def pin_hash_trilinear_exact_on_linear_tables():
    grid = hashgrid.HashGrid3D()
    coef = [(0.7, -1.3, 2.1, 0.25), (-0.4, 0.9, 1.7, -0.5)]
    table = _linear_tables(grid, coef)
    x = np.random.default_rng(17).uniform(-1.5, 1.5, size=(400, 3)).astype(np.float32)
    enc = grid.encode(x, table)
    for level, N in enumerate(grid.res):
        if not grid.direct[level]:
            continue
        c = (grid.unit_coords(x) * np.float32(N)).astype(np.float64)   # the interpolated point
        for f in range(grid.F):
            a, b, cc, e = coef[f]
            want = (a * c[:, 0] + b * c[:, 1] + cc * c[:, 2]) / N + e
            np.testing.assert_allclose(enc[:, level * grid.F + f], want, atol=1e-12)


def test_hash_trilinear_exact_on_linear_tables():
    pin_hash_trilinear_exact_on_linear_tables()


# ------------------------------------------------------------------ hash-grid network

def _hash_mlp(set_fn):
    layout = S.hash_mlp_layout()
    blobs = {name: [np.zeros((n, k)), np.zeros(n)] for name, n, k in layout}
    set_fn(blobs)
    flat = np.concatenate([np.concatenate([blobs[name][0].ravel(), blobs[name][1]])
                           for name, _, _ in layout])
    return flat


def _real_sh_low(d):
    """Real spherical harmonics of bands 0 and 1 in closed form (index l*l + l + m,
    no Condon-Shortley phase): 1/(2 sqrt(pi)); sqrt(3/(4 pi)) (y, z, x)."""
    k = math.sqrt(3.0 / (4.0 * math.pi))
    return np.stack([np.full(len(d), 0.5 / math.sqrt(math.pi)), k * d[:, 1], k * d[:, 2],
                     k * d[:, 0]], axis=1)


def pin_hash_network_routing():
    grid = hashgrid.HashGrid3D()
    g = np.random.default_rng(18)
    table = g.uniform(-1, 1, size=(grid.n_entries, 2)).astype(np.float16)
    x = g.uniform(-1.5, 1.5, size=(300, 3)).astype(np.float32)
    du = nerf.unit(g.normal(size=(300, 3)))
    enc = grid.encode(x, table)
    for j in (0, 7, 31):
        for s in (0, 1, 2, 3):
            def setw(b, j=j, s=s):
                b["d0"][0][0, j] = 1.0              # encoding feature j -> h[0] -> sigma
                b["d1"][0][0, 0] = 1.0
                b["sigma"][0][0, 0] = 1.0
                b["c0"][0][0, 64 + s] = 1.0         # view feature s -> colour 0
                b["c1"][0][0, 0] = 1.0
                b["rgb"][0][0, 0] = 1.0
                b["d0"][1][5] = 0.7                 # a density feature -> colour 1
                b["d1"][0][3, 5] = 1.0
                b["c0"][0][1, 3] = 1.0
                b["c1"][0][1, 1] = 1.0
                b["rgb"][0][1, 1] = 1.0
                b["rgb"][1][2] = -0.3               # bias-only colour 2
            sigma, rgb = march.hash_eval(grid, table, _hash_mlp(setw), x, du)
            np.testing.assert_allclose(sigma, np.maximum(enc[:, j], 0.0), atol=1e-12)
            want0 = 1.0 / (1.0 + np.exp(-np.maximum(_real_sh_low(du)[:, s], 0.0)))
            np.testing.assert_allclose(rgb[:, 0], want0, atol=1e-12)
            np.testing.assert_allclose(rgb[:, 1], 1.0 / (1.0 + math.exp(-0.7)), atol=1e-12)
            np.testing.assert_allclose(rgb[:, 2], 1.0 / (1.0 + math.exp(0.3)), atol=1e-12)


def test_hash_network_routing():
    pin_hash_network_routing()


# ------------------------------------------------------------------ KiloNeRF cell network

def pin_kilonerf_routing():
    layout = S.kilonerf_layout()
    n_cells = 16 ** 3
    g = np.random.default_rng(19)
    x = g.uniform(-1.5, 1.5, size=(400, 3)).astype(np.float32)
    du = nerf.unit(g.normal(size=(400, 3)))
    cells = march.cell_id(x)
    blobs = {name: [np.zeros((n, k)), np.zeros(n)] for name, n, k in layout}
    blobs["l1"][0][0, 0] = 1.0           # gamma(x)[0] = x_0 -> h1[0] -> h2[4] -> sigma
    blobs["l2"][0][4, 0] = 1.0
    blobs["sigma"][0][0, 4] = 1.0
    blobs["rgb"][0][0, 32 + 0] = 1.0     # colour 0 <- gamma(d)[0] = d_x
    blobs["rgb"][0][1, 4] = 1.0          # colour 1 <- h2[4]
    blobs["rgb"][0][2, 32 + 3] = 1.0     # colour 2 <- gamma(d)[3] = sin(pi d_x)
    flat = np.concatenate([np.concatenate([blobs[n][0].ravel(), blobs[n][1]]) for n, _, _ in layout])
    params = np.tile(flat.astype(np.float32), (n_cells, 1))
    sigma, rgb = march.kilonerf_eval(params, cells, x, du)
    x0 = x[:, 0].astype(np.float64)
    sig = lambda a: 1.0 / (1.0 + np.exp(-a))
    np.testing.assert_allclose(sigma, np.maximum(x0, 0.0), atol=1e-12)
    np.testing.assert_allclose(rgb[:, 0], sig(du[:, 0]), atol=1e-12)
    np.testing.assert_allclose(rgb[:, 1], sig(np.maximum(x0, 0.0)), atol=1e-12)
    np.testing.assert_allclose(rgb[:, 2], sig(np.sin(np.pi * du[:, 0])), atol=1e-12)


def test_kilonerf_routing():
    pin_kilonerf_routing()
