"""Seeded synthetic inputs for the renderer: cameras, network weights, hash tables,
occupancy grids and KiloNeRF cell weights.

This module only draws and lays out inputs. It holds none of the rendering
arithmetic (no ray generation, encoding, network evaluation or compositing), so
that both the CUDA path and the CPU oracle can take the same arrays from it
without sharing any of the method.

The workloads follow the shapes the pages render: the Blender "lego" scene of
"Spatial Intelligence - Part 1: NeRF" (Section 3, 800x800 views from a camera on
a sphere around the object, near 2 / far 6) stands in as seeded synthetic
cameras and random-init networks; no dataset and no trained weight is used.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

# Flat-parameter layouts -----------------------------------------------------

SIGMA_RELU = 0
SIGMA_SOFTPLUS = 1
PREC_FP32 = 0
PREC_BF16 = 1
PREC_TF32 = 2   # fp32 weights, layer products on the tensor cores (tf32 hi/lo, 3 passes)
LAST_DELTA_PAGE = 0   # last interval 1e10 (volume_render on the NeRF page)
LAST_DELTA_TO_FAR = 1  # last interval reaches t_f


@dataclasses.dataclass(frozen=True)
class MLPShape:
    """Shape of the NeRF scene network F_theta ("The NeRF network" section)."""
    D: int = 8
    W: int = 256
    skip: int = 4          # hidden state is concatenated with gamma(x) after layer `skip`
    L_pos: int = 10
    L_dir: int = 4

    @property
    def pos_ch(self) -> int:
        return 3 * (1 + 2 * self.L_pos)

    @property
    def dir_ch(self) -> int:
        return 3 * (1 + 2 * self.L_dir)

    def layer_shapes(self):
        """(name, N_out, K_in) of every Linear in blob order."""
        out = []
        for i in range(self.D):
            if i == 0:
                k = self.pos_ch
            elif i == self.skip + 1:
                k = self.W + self.pos_ch
            else:
                k = self.W
            out.append((f"pts{i}", self.W, k))
        out.append(("sigma", 1, self.W))
        out.append(("feature", self.W, self.W))
        out.append(("dir", self.W // 2, self.W + self.dir_ch))
        out.append(("rgb", 3, self.W // 2))
        return out

    def n_params(self) -> int:
        return sum(n * k + n for _, n, k in self.layer_shapes())


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returned as fp32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).reshape(a.shape)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """The bf16 bit patterns (uint16) of values that are already bf16-exact."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def xavier_uniform(rng, n_out, k_in):
    bound = math.sqrt(6.0 / (k_in + n_out))
    return rng.uniform(-bound, bound, size=(n_out, k_in)).astype(np.float32)


def nerf_weights(shape: MLPShape, seed: int, net: int, sigma_scale: float = 1.0,
                 precision: int = PREC_FP32):
    """Seeded weights of one NeRF network (net 0 = coarse, 1 = fine).

    Matrices are Xavier-uniform U(+-sqrt(6/(fan_in+fan_out))), biases U(+-0.1);
    the sigma head is multiplied by `sigma_scale`. With precision BF16 every
    parameter is rounded to bf16 and the returned fp32 values are bf16-exact.
    Returns (flat fp32 blob in layer_shapes order [W row-major (N,K), then b],
    dict name -> (W, b)).
    """
    rng = np.random.default_rng([seed, 1000 + net])
    params = {}
    flat = []
    for name, n, k in shape.layer_shapes():
        w = xavier_uniform(rng, n, k)
        b = rng.uniform(-0.1, 0.1, size=(n,)).astype(np.float32)
        if name == "sigma":
            w = (w * np.float32(sigma_scale)).astype(np.float32)
            b = (b * np.float32(sigma_scale)).astype(np.float32)
        if precision == PREC_BF16:
            w, b = bf16_round(w), bf16_round(b)
        params[name] = (w, b)
        flat.append(w.ravel())
        flat.append(b)
    return np.concatenate(flat).astype(np.float32), params


# Cameras -------------------------------------------------------------------

def look_at_c2w(az_deg: float, el_deg: float, radius: float = 4.0) -> np.ndarray:
    """Camera-to-world [3x4] fp32 for a camera on a sphere looking at the origin.

    Columns are right, up, back, position; the camera looks down its -z axis
    (the convention of get_rays on the NeRF page, "Ray generation").
    """
    az, el = math.radians(az_deg), math.radians(el_deg)
    p = radius * np.array([math.cos(el) * math.cos(az), math.cos(el) * math.sin(az),
                           math.sin(el)], dtype=np.float64)
    back = p / np.linalg.norm(p)
    right = np.cross(np.array([0.0, 0.0, 1.0]), back)
    right /= np.linalg.norm(right)
    up = np.cross(back, right)
    return np.stack([right, up, back, p], axis=1).astype(np.float32)


def seeded_camera(seed: int):
    rng = np.random.default_rng([seed, 7])
    az = float(rng.uniform(0.0, 360.0))
    el = float(rng.uniform(10.0, 60.0))
    return az, el


def orbit_c2ws(seed: int, n_frames: int = 24) -> list:
    """Cameras of a 360-degree orbit (the novel-view video of the NeRF page,
    Section 3): n_frames azimuths evenly spaced from the seeded camera's, at its
    elevation and radius 4. Returns a list of [3x4] fp32 arrays."""
    az0, el = seeded_camera(seed)
    return [look_at_c2w(az0 + 360.0 * k / n_frames, el) for k in range(n_frames)]


# Workloads -----------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    H: int
    W: int
    focal: float
    seed: int
    near: float = 2.0
    far: float = 6.0
    model: str = "nerf"          # nerf | kilonerf | hashgrid
    n_coarse: int = 64           # stratified samples (nerf) or candidate cap (march)
    n_fine: int = 0
    mlp: MLPShape | None = None
    sigma_act: int = SIGMA_RELU
    precision: int = PREC_FP32
    last_delta: int = LAST_DELTA_PAGE
    white_bkgd: int = 0
    march_step: float = 0.0
    ert_T: float = 0.0           # 0 disables early ray termination
    sigma_scale: float = 1.0
    az: float | None = None
    el: float | None = None

    @property
    def n_rays(self) -> int:
        return self.H * self.W

    def c2w(self) -> np.ndarray:
        if self.az is not None:
            return look_at_c2w(self.az, self.el)
        return look_at_c2w(*seeded_camera(self.seed))


# The five workloads. Sizes follow the pages' NeRF render (64 + 128 samples per
# ray, 8x256 network, 800x800 views, near 2 / far 6); the tiny, KiloNeRF and
# hash-grid shapes are the synthetic stand-ins described in the design notes.
# small_tf32 is the small workload on the TF32 precision (same weights, camera
# and samples).
WORKLOADS = {
    "tiny": Workload("tiny_nerf_32x32", 32, 32, 40.0, seed=0, n_coarse=64, n_fine=0,
                     mlp=MLPShape(D=4, W=64, skip=-1), sigma_act=SIGMA_SOFTPLUS,
                     az=45.0, el=30.0),
    "small": Workload("nerf_200x200_fp32", 200, 200, 250.0, seed=1, n_coarse=64, n_fine=128,
                      mlp=MLPShape(), sigma_scale=1.0),
    "small_tf32": Workload("nerf_200x200_tf32x3", 200, 200, 250.0, seed=1, n_coarse=64, n_fine=128,
                           mlp=MLPShape(), sigma_scale=1.0, precision=PREC_TF32),
    "full": Workload("nerf_800x800_bf16", 800, 800, 1000.0, seed=3, n_coarse=64, n_fine=128,
                     mlp=MLPShape(), precision=PREC_BF16, sigma_scale=1.0),
    "kilonerf": Workload("kilonerf_16cubed_800x800", 800, 800, 1000.0, seed=4, model="kilonerf",
                         n_coarse=342, march_step=3.0 / 256.0, ert_T=1e-3),
    "hashgrid": Workload("hashgrid_1920x1080", 1080, 1920, 2400.0, seed=5, model="hashgrid",
                         n_coarse=512, march_step=1.0 / 128.0),
}


# Occupancy grid -------------------------------------------------------------

GRID_RES = 128
GRID_MIN = -1.5
GRID_SIZE = 3.0


def occupancy_grid(seed: int, n_blobs: int = 16, frac: float = 0.1):
    """Seeded 128^3 binary occupancy grid, bit-packed (x-major, 32 bits/word).

    A sum of `n_blobs` isotropic Gaussians (centres U(-1.2,1.2)^3, widths
    U(0.1,0.35)) is evaluated at the voxel centres of [-1.5,1.5]^3 and the top
    floor(frac * 128^3) voxels are marked occupied (ties broken by linear index
    (ix*128+iy)*128+iz). Returns (packed uint32[65536], dense bool[128,128,128]).
    """
    rng = np.random.default_rng([seed, 31])
    centres = rng.uniform(-1.2, 1.2, size=(n_blobs, 3))
    widths = rng.uniform(0.1, 0.35, size=(n_blobs,))
    c = GRID_MIN + (np.arange(GRID_RES) + 0.5) * (GRID_SIZE / GRID_RES)
    X, Y, Z = np.meshgrid(c, c, c, indexing="ij")
    field = np.zeros(X.shape, dtype=np.float64)
    for (cx, cy, cz), s in zip(centres, widths):
        field += np.exp(-((X - cx) ** 2 + (Y - cy) ** 2 + (Z - cz) ** 2) / (2.0 * s * s))
    flat = field.ravel()
    n_occ = int(math.floor(frac * flat.size))
    order = np.lexsort((np.arange(flat.size), -flat))   # value desc, index asc
    dense = np.zeros(flat.size, dtype=bool)
    dense[order[:n_occ]] = True
    bits = dense.reshape(-1, 32).astype(np.uint64)
    packed = (bits << np.arange(32, dtype=np.uint64)).sum(axis=1).astype(np.uint32)
    return packed, dense.reshape(GRID_RES, GRID_RES, GRID_RES)


# KiloNeRF cells ------------------------------------------------------------

KILO_CELLS = 16
KILO_HIDDEN = 32


def kilonerf_layout(L_pos: int = 10, L_dir: int = 4, hidden: int = KILO_HIDDEN):
    """(name, N_out, K_in) of each per-cell Linear, in blob order."""
    pc, dc = 3 * (1 + 2 * L_pos), 3 * (1 + 2 * L_dir)
    return [("l1", hidden, pc), ("l2", hidden, hidden), ("sigma", 1, hidden),
            ("rgb", 3, hidden + dc)]


def kilonerf_weights(seed: int, n_cells: int = KILO_CELLS ** 3):
    """Per-cell tiny-MLP weights, fp32 [n_cells][3317] (Xavier + U(+-0.1) bias)."""
    rng = np.random.default_rng([seed, 41])
    parts = []
    for _, n, k in kilonerf_layout():
        bound = math.sqrt(6.0 / (k + n))
        parts.append(rng.uniform(-bound, bound, size=(n_cells, n * k)).astype(np.float32))
        parts.append(rng.uniform(-0.1, 0.1, size=(n_cells, n)).astype(np.float32))
    return np.ascontiguousarray(np.concatenate(parts, axis=1), dtype=np.float32)


# Hash grid -----------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class HashGridShape:
    """3D multiresolution hash grid (the 2D HashGrid2D of the Instant-NGP
    notebook, Experiment 1, extended to three axes)."""
    L: int = 16
    log2_T: int = 19
    F: int = 2
    N_min: int = 16
    N_max: int = 2048


HASH_ENTRIES = 6101902   # rows of the 16 concatenated level tables of HashGridShape()


def hashgrid_table(shape: HashGridShape, n_entries: int, seed: int, scale: float):
    """All levels' feature tables concatenated, fp16 [n_entries][F], U(+-scale)."""
    rng = np.random.default_rng([seed, 53])
    return rng.uniform(-scale, scale, size=(int(n_entries), shape.F)).astype(np.float16)


HASH_MLP_HIDDEN = 64
SH_DIM = 16


def hash_mlp_layout(n_feat: int = 32, hidden: int = HASH_MLP_HIDDEN, sh_dim: int = SH_DIM):
    return [("d0", hidden, n_feat), ("d1", hidden, hidden), ("sigma", 1, hidden),
            ("c0", hidden, hidden + sh_dim), ("c1", hidden, hidden), ("rgb", 3, hidden)]


def hash_mlp_weights(seed: int):
    rng = np.random.default_rng([seed, 67])
    flat = []
    for _, n, k in hash_mlp_layout():
        flat.append(xavier_uniform(rng, n, k).ravel())
        flat.append(rng.uniform(-0.1, 0.1, size=(n,)).astype(np.float32))
    return np.concatenate(flat).astype(np.float32)


# Generic seeded arrays for unit cases --------------------------------------

def uniform(seed: int, shape, lo=-1.0, hi=1.0, dtype=np.float32):
    return np.random.default_rng([seed, 97]).uniform(lo, hi, size=shape).astype(dtype)


def ray_subset(n_rays: int, n_sample: int, seed: int):
    """Sorted seeded subset of ray indices (uniform without replacement)."""
    rng = np.random.default_rng([seed, 113])
    return np.sort(rng.choice(n_rays, size=min(n_sample, n_rays), replace=False)).astype(np.int64)
