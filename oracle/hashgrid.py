"""Oracle for the multiresolution hash-grid encoding. Test infrastructure only.

Follows the HashGrid2D class of the Instant-NGP notebook ("A shared toolkit"
section and Experiment 1): a geometric resolution schedule, one table per
level capped at T entries, direct indexing while the level's vertices fit the
table and an XOR-of-primes spatial hash otherwise, and interpolation of the
surrounding vertices' features with per-level concatenation. The 3D form adds
a third axis with the third prime and trilinear weights.
"""
from __future__ import annotations

import math

import numpy as np

F32 = np.float32
PRIMES = (1, 2654435761, 805459861)


def level_resolutions(L: int, N_min: int, N_max: int):
    """N_l = round(N_min * b^l), b = exp((ln N_max - ln N_min) / (L - 1));
    Python's round (ties to even) as in the notebook."""
    b = math.exp((math.log(N_max) - math.log(N_min)) / (L - 1))
    return [int(round(N_min * b ** l)) for l in range(L)]


def level_tables(res, T: int, dim: int):
    """(sizes, direct flags): size = min(T, (N+1)^dim); direct iff (N+1)^dim <= T."""
    sizes, direct = [], []
    for N in res:
        cells = (N + 1) ** dim
        sizes.append(min(T, cells))
        direct.append(cells <= T)
    return sizes, direct


def index_2d(ix, iy, N, T, direct):
    """Notebook _idx: ix*(N+1)+iy when direct, else (ix XOR iy*PI1) mod T,
    evaluated in int64 like the notebook's .long() arithmetic."""
    ix = np.asarray(ix, dtype=np.int64)
    iy = np.asarray(iy, dtype=np.int64)
    if direct:
        return ix * (N + 1) + iy
    return np.bitwise_xor(ix, iy * PRIMES[1]) % T


def index_3d(ix, iy, iz, N, T, direct):
    """3D form: (ix*(N+1)+iy)*(N+1)+iz when direct, else
    (ix*1 XOR iy*2654435761 XOR iz*805459861) mod T, in int64."""
    ix = np.asarray(ix, dtype=np.int64)
    iy = np.asarray(iy, dtype=np.int64)
    iz = np.asarray(iz, dtype=np.int64)
    if direct:
        return (ix * (N + 1) + iy) * (N + 1) + iz
    h = np.bitwise_xor(np.bitwise_xor(ix * PRIMES[0], iy * PRIMES[1]), iz * PRIMES[2])
    return h % T


class HashGrid3D:
    """3D multiresolution grid over the cube [-1.5, 1.5]^3.

    The unit-cube coordinate is x01 = fl((x + 1.5) / 3) in fp32; per level,
    c = fl(x01 * N) in fp32, c0 = floor(c), w = c - c0 (exact), corners
    clamped to [0, N]. Features are interpolated in fp64 with weights
    prod over axes of (w if the corner is the upper one else 1 - w).
    """

    def __init__(self, L=16, log2_T=19, F=2, N_min=16, N_max=2048):
        self.L, self.T, self.F = L, 1 << log2_T, F
        self.res = level_resolutions(L, N_min, N_max)
        self.sizes, self.direct = level_tables(self.res, self.T, 3)
        self.offsets = np.concatenate([[0], np.cumsum(self.sizes)]).astype(np.int64)

    @property
    def n_entries(self):
        return int(self.offsets[-1])

    def unit_coords(self, x):
        x = np.asarray(x, dtype=F32)
        return (x + F32(1.5)) / F32(3.0)

    def corners(self, x, level):
        """Per point and corner (dx,dy,dz loops in that order): global table
        row and interpolation weight (fp64). Returns (rows [P,8], w [P,8])."""
        N = self.res[level]
        c = self.unit_coords(x) * F32(N)
        c0 = np.floor(c)
        w = (c - c0).astype(np.float64)
        c0 = c0.astype(np.int64)
        rows, wts = [], []
        for dx in (0, 1):
            for dy in (0, 1):
                for dz in (0, 1):
                    ix = np.clip(c0[:, 0] + dx, 0, N)
                    iy = np.clip(c0[:, 1] + dy, 0, N)
                    iz = np.clip(c0[:, 2] + dz, 0, N)
                    idx = index_3d(ix, iy, iz, N, self.T, self.direct[level])
                    wx = w[:, 0] if dx else 1.0 - w[:, 0]
                    wy = w[:, 1] if dy else 1.0 - w[:, 1]
                    wz = w[:, 2] if dz else 1.0 - w[:, 2]
                    rows.append(self.offsets[level] + idx)
                    wts.append(wx * wy * wz)
        return np.stack(rows, axis=1), np.stack(wts, axis=1)

    def encode(self, x, table):
        """Encoding [P, L*F] (level-major, F features per level), fp64.
        table: [n_entries, F] (any float dtype, upcast exactly)."""
        table = np.asarray(table).astype(np.float64)
        feats = []
        for level in range(self.L):
            rows, wts = self.corners(x, level)
            feats.append((wts[:, :, None] * table[rows]).sum(axis=1))
        return np.concatenate(feats, axis=1)

    def encode_backward(self, x, d_feat):
        """Gradient of sum(d_feat * encode(x, table)) with respect to the table:
        every point adds, at each level, weight * d_feat[level] to each of its
        8 corner rows (the encoding is linear in the table, so this is its
        adjoint: the scatter-add that trains the grid, Instant-NGP notebook,
        Experiment 1, made 3D). d_feat [P, L*F]; returns [n_entries, F] fp64."""
        d_feat = np.asarray(d_feat, dtype=np.float64)
        grad = np.zeros((self.n_entries, self.F), dtype=np.float64)
        for level in range(self.L):
            rows, wts = self.corners(x, level)
            g = d_feat[:, level * self.F:(level + 1) * self.F]
            np.add.at(grad, rows.ravel(), (wts[:, :, None] * g[:, None, :]).reshape(-1, self.F))
        return grad


class HashGrid2D:
    """The notebook's 2D grid over [0,1]^2 (used for the printed pins)."""

    def __init__(self, L=8, T=2 ** 12, F=2, N_min=8, N_max=160):
        self.L, self.T, self.F = L, T, F
        self.res = level_resolutions(L, N_min, N_max)
        self.sizes, self.direct = level_tables(self.res, T, 2)

    def encode(self, x, tables):
        """Bilinear encoding [P, L*F] fp64; tables: list of [size_l, F]."""
        x = np.asarray(x, dtype=F32)
        feats = []
        for level, N in enumerate(self.res):
            c = x * F32(N)
            c0 = np.floor(c)
            w = (c - c0).astype(np.float64)
            c0 = c0.astype(np.int64)
            acc = 0.0
            for dx in (0, 1):
                for dy in (0, 1):
                    ix = np.clip(c0[:, 0] + dx, 0, N)
                    iy = np.clip(c0[:, 1] + dy, 0, N)
                    f = np.asarray(tables[level], dtype=np.float64)[
                        index_2d(ix, iy, N, self.T, self.direct[level])]
                    wx = w[:, 0] if dx else 1.0 - w[:, 0]
                    wy = w[:, 1] if dy else 1.0 - w[:, 1]
                    acc = acc + (wx * wy)[:, None] * f
            feats.append(acc)
        return np.concatenate(feats, axis=1)


def mlp_param_count(layer_sizes):
    """Parameters of a chain of Linear layers with biases (nn.Linear convention)."""
    return sum(a * b + b for a, b in zip(layer_sizes[:-1], layer_sizes[1:]))
