"""Pins of the CPU oracle against facts fixed independently of it: values the
pages print, closed forms of the rendering integral, invariants, textbook or
library routines, and brute force on tiny inputs. CPU only."""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import nerf_inputs as S
from oracle import hashgrid, march, nerf, rng, sh

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------ RNG

def test_splitmix64_known_answers():
    kat = golden("splitmix64_kat.json")["state0_outputs"]
    state = 0
    for want in kat:
        assert int(rng.mix(np.uint64(state))) == int(want, 16)
        state = (state + 0x9E3779B97F4A7C15) % (1 << 64)


def test_uniform_draws_are_uniform_and_distinct_per_stream():
    from scipy import stats
    u0 = rng.draw_uniform(3, np.arange(4000)[:, None], 0, np.arange(64)[None, :]).ravel()
    u1 = rng.draw_uniform(3, np.arange(4000)[:, None], 1, np.arange(64)[None, :]).ravel()
    assert stats.kstest(u0, "uniform").pvalue > 1e-3
    assert stats.kstest(u1, "uniform").pvalue > 1e-3
    assert abs(np.corrcoef(u0, u1)[0, 1]) < 0.01
    assert u0.min() >= 0.0 and u0.max() < 1.0
    assert np.all(u0 * 2 ** 24 == np.floor(u0 * 2 ** 24))   # 24-bit, fp32-exact


# ------------------------------------------------------------------ rays

def test_raygen_identity_camera_exact_values():
    # Identity rotation, camera at (0,0,4): d = ((i - W/2)/f, -(j - H/2)/f, -1)
    c2w = np.array([[1, 0, 0, 0], [0, 1, 0, 0], [0, 0, 1, 4]], dtype=np.float32)
    H, W, f = 3, 4, 2.0
    o, d = nerf.raygen(H, W, f, c2w)
    assert o.shape == (12, 3) and d.shape == (12, 3)
    for j in range(H):
        for i in range(W):
            r = j * W + i
            assert d[r].tolist() == [(i - W / 2) / f, -(j - H / 2) / f, -1.0]
            assert o[r].tolist() == [0.0, 0.0, 4.0]


def test_raygen_centre_pixel_looks_at_origin():
    wl = S.WORKLOADS["small"]
    c2w = wl.c2w()
    o, d = nerf.raygen(wl.H, wl.W, wl.focal, c2w)
    centre = (wl.H // 2) * wl.W + wl.W // 2
    np.testing.assert_array_equal(d[centre], -c2w[:, 2])
    # the centre ray points at the origin: o + t d = 0 for t = |o|
    p = o[centre].astype(np.float64)
    dd = d[centre].astype(np.float64)
    assert np.linalg.norm(p + np.linalg.norm(p) * dd) < 1e-5
    # rotation preserves the camera-space norm sqrt(dx^2 + dy^2 + 1)
    j, i = np.divmod(np.arange(wl.n_rays), wl.W)
    ref = np.sqrt(((i - wl.W / 2) / wl.focal) ** 2 + ((j - wl.H / 2) / wl.focal) ** 2 + 1)
    np.testing.assert_allclose(np.linalg.norm(d.astype(np.float64), axis=1), ref, rtol=1e-6)


def test_stratified_samples_lie_in_their_bins():
    t = nerf.stratified_t(2.0, 6.0, 64, 5, np.arange(100))
    lo = 2.0 + np.arange(64) * (4.0 / 64)
    assert np.all(t >= lo) and np.all(t <= lo + 4.0 / 64)
    assert np.all(np.diff(t, axis=1) >= 0)
    mid = nerf.stratified_t(2.0, 6.0, 64, 5, np.arange(3), perturb=False)
    np.testing.assert_array_equal(mid[0], (lo + 2.0 / 64).astype(np.float32))


# ------------------------------------------------------------------ PE

def test_positional_encoding_dims_from_page():
    g = golden("nerf_page_dims.json")["pe_dims"]
    x = np.zeros((1, 3))
    assert nerf.positional_encoding(x, g["L_pos"]).shape[-1] == g["pos_dims"]
    assert nerf.positional_encoding(x, g["L_dir"]).shape[-1] == g["dir_dims"]


def test_positional_encoding_special_values_and_layout():
    # x = (1/2, 1/6, 0): sin(pi x) = (1, 1/2, 0), cos(pi x) = (0, sqrt3/2, 1)
    L = 3
    e = nerf.positional_encoding(np.array([[0.5, 1.0 / 6.0, 0.0]]), L)[0]
    np.testing.assert_array_equal(e[:3], [0.5, 1.0 / 6.0, 0.0])
    sin0 = e[3:3 + 3 * L][0::L]        # frequency 0 of each coordinate (coordinate-major)
    cos0 = e[3 + 3 * L:][0::L]
    np.testing.assert_allclose(sin0, [1.0, 0.5, 0.0], atol=1e-15)
    np.testing.assert_allclose(cos0, [0.0, math.sqrt(3) / 2, 1.0], atol=1e-15)


def test_positional_encoding_double_angle_recurrence():
    L = 10
    x = np.random.default_rng(0).uniform(-1.5, 1.5, size=(200, 3))
    e = nerf.positional_encoding(x, L)
    s = e[:, 3:3 + 3 * L].reshape(200, 3, L)
    c = e[:, 3 + 3 * L:].reshape(200, 3, L)
    np.testing.assert_allclose(s[..., 1:], 2 * s[..., :-1] * c[..., :-1], atol=1e-12)
    np.testing.assert_allclose(c[..., 1:], 1 - 2 * s[..., :-1] ** 2, atol=1e-12)
    np.testing.assert_allclose(s ** 2 + c ** 2, 1.0, atol=1e-14)


# ------------------------------------------------------------------ MLP

def test_layer_widths_and_param_counts():
    g = golden("nerf_page_dims.json")["network"]
    shape = S.MLPShape()
    ls = dict((n, (o, k)) for n, o, k in shape.layer_shapes())
    assert ls["pts5"][1] == g["skip_layer_input_width"]
    assert ls["dir"] == (g["dir_width"], g["dir_layer_input_width"])
    p = golden("instant_ngp_2d_levels.json")["experiment_2"]
    assert hashgrid.mlp_param_count(p["hash_mlp"]["layers"]) == p["hash_mlp"]["params"]
    assert hashgrid.mlp_param_count(p["pe_mlp"]["layers"]) == p["pe_mlp"]["params"]
    # blob size = the same convention applied to every Linear of the network
    assert shape.n_params() == sum(n * k + n for _, n, k in shape.layer_shapes())
    flat, _ = S.nerf_weights(shape, 0, 0)
    assert flat.size == shape.n_params()


def _zero_params(shape):
    return {name: (np.zeros((n, k)), np.zeros(n)) for name, n, k in shape.layer_shapes()}


def test_mlp_bias_only_network():
    shape = S.MLPShape(D=3, W=8, skip=0, L_pos=2, L_dir=1)
    p = _zero_params(shape)
    p["rgb"] = (p["rgb"][0], np.array([0.1, -0.2, 0.3]))
    p["sigma"] = (p["sigma"][0], np.array([0.7]))
    out = nerf.nerf_mlp(shape, p, np.ones((5, shape.pos_ch)), np.ones((5, shape.dir_ch)))
    np.testing.assert_array_equal(out, np.tile([0.1, -0.2, 0.3, 0.7], (5, 1)))


def test_mlp_skip_concatenates_hidden_then_encoding():
    # Layer skip+1 sees [h, gamma(x)]: route gamma(x)[j] to unit 0 through the
    # second block of its input and read it out as sigma.
    shape = S.MLPShape(D=3, W=4, skip=0, L_pos=1, L_dir=1)
    p = _zero_params(shape)
    j = 4
    w1 = np.zeros((4, shape.W + shape.pos_ch))
    w1[0, shape.W + j] = 1.0
    p["pts1"] = (w1, np.zeros(4))
    p["pts2"] = (np.eye(4), np.zeros(4))
    p["sigma"] = (np.array([[1.0, 0, 0, 0]]), np.zeros(1))
    penc = np.random.default_rng(1).uniform(0.1, 1.0, size=(6, shape.pos_ch))
    out = nerf.nerf_mlp(shape, p, penc, np.zeros((6, shape.dir_ch)))
    np.testing.assert_allclose(out[:, 3], penc[:, j])


def test_mlp_direction_branch_sees_feature_then_direction():
    shape = S.MLPShape(D=2, W=4, skip=-1, L_pos=1, L_dir=1)
    p = _zero_params(shape)
    wd = np.zeros((2, shape.W + shape.dir_ch))
    wd[0, shape.W + 1] = 1.0              # h'_0 = gamma(d)[1]
    wd[1, 0] = 1.0                        # h'_1 = feature_0 = bias 0.5
    p["dir"] = (wd, np.zeros(2))
    p["feature"] = (np.zeros((4, 4)), np.array([0.5, 0, 0, 0]))
    p["rgb"] = (np.array([[1.0, 0], [0, 1.0], [1.0, 1.0]]), np.zeros(3))
    denc = np.random.default_rng(2).uniform(0.1, 1.0, size=(3, shape.dir_ch))
    out = nerf.nerf_mlp(shape, p, np.zeros((3, shape.pos_ch)), denc)
    np.testing.assert_allclose(out[:, 0], denc[:, 1])
    np.testing.assert_allclose(out[:, 1], 0.5)
    np.testing.assert_allclose(out[:, 2], denc[:, 1] + 0.5)


# ------------------------------------------------------------------ compositing

def test_composite_constant_medium_closed_form():
    # C(r) = c (1 - exp(-sigma ||d|| (t_f - t_n))) for constant (c, sigma)
    near, far, n = 2.0, 6.0, 64
    t = np.tile(near + np.arange(n) * (far - near) / n, (4, 1))
    dnorm = np.array([1.0, 1.3, 0.7, 2.0])
    sigma = np.full((4, n), 0.37)
    c = np.array([0.2, 0.5, 0.9])
    rgb = np.broadcast_to(c, (4, n, 3))
    delta = nerf.deltas(t, dnorm, 1, far=far)
    out, depth, acc, w = nerf.composite(sigma, rgb, t, delta)
    want = 1 - np.exp(-0.37 * dnorm * (far - near))
    np.testing.assert_allclose(acc, want, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out, want[:, None] * c, atol=1e-12)
    assert np.all(w >= 0)


def test_composite_invariants_random():
    g = np.random.default_rng(3)
    t = np.sort(g.uniform(2, 6, size=(50, 64)), axis=1)
    sigma = np.maximum(g.normal(0, 3, size=(50, 64)), 0)
    rgb = g.uniform(0, 1, size=(50, 64, 3))
    dn = g.uniform(0.8, 1.5, size=50)
    # telescoping: sum w = 1 - T_{N+1} <= 1 (to-far mode)
    delta = nerf.deltas(t, dn, 1, far=6.0)
    _, _, acc, w = nerf.composite(sigma, rgb, t, delta)
    assert np.all(w >= 0)
    np.testing.assert_allclose(acc, 1 - np.exp(-(sigma * delta).sum(1)), atol=1e-12)
    assert np.all(acc <= 1 + 1e-15)
    # page mode: any density in the last sample makes the ray opaque
    sigma[:, -1] = 0.5
    _, _, acc, _ = nerf.composite(sigma, rgb, t, nerf.deltas(t, dn, 0))
    np.testing.assert_allclose(acc, 1.0, atol=1e-12)
    # no density, no opacity; white background shows through
    out, depth, acc, _ = nerf.composite(np.zeros_like(sigma), rgb, t, delta, white_bkgd=True)
    assert np.all(acc == 0) and np.all(depth == 0) and np.all(out == 1)


def test_composite_single_opaque_sample_depth():
    t = np.tile(np.linspace(2, 6, 16), (1, 1))
    sigma = np.zeros((1, 16))
    sigma[0, 5] = 1e6
    rgb = np.zeros((1, 16, 3))
    rgb[0, 5] = [0.25, 0.5, 0.75]
    out, depth, acc, _ = nerf.composite(sigma, rgb, t, nerf.deltas(t, np.ones(1), 0))
    np.testing.assert_allclose(depth, t[0, 5], atol=1e-12)
    np.testing.assert_allclose(out[0], [0.25, 0.5, 0.75], atol=1e-12)


def test_composite_brute_force_with_survival_guard():
    # The page's volume_render keeps a 1e-10 survival guard in the cumulative
    # product; scalar loops with the guard agree with the guard-free oracle to
    # within N * 1e-10.
    g = np.random.default_rng(4)
    t = np.sort(g.uniform(2, 6, size=(3, 12)), axis=1)
    sigma = np.maximum(g.normal(0, 2, size=(3, 12)), 0)
    rgb = g.uniform(0, 1, size=(3, 12, 3))
    dn = np.array([1.0, 1.2, 0.9])
    out, depth, acc, _ = nerf.composite(sigma, rgb, t, nerf.deltas(t, dn, 0))
    for r in range(3):
        T, cr, dr, ar = 1.0, [0.0, 0.0, 0.0], 0.0, 0.0
        for i in range(12):
            dist = (t[r, i + 1] - t[r, i]) if i < 11 else 1e10
            a = 1.0 - math.exp(-sigma[r, i] * dist * dn[r])
            wi = T * a
            cr = [cr[k] + wi * rgb[r, i, k] for k in range(3)]
            dr += wi * t[r, i]
            ar += wi
            T *= 1.0 - a + 1e-10
        np.testing.assert_allclose(out[r], cr, atol=2e-9)
        assert abs(depth[r] - dr) < 1e-8 and abs(acc[r] - ar) < 2e-9


# ------------------------------------------------------------------ sampler

def test_sample_pdf_uniform_weights_give_uniform_samples():
    R, nb = 4, 63
    bins = np.tile(np.linspace(2, 6, nb, dtype=np.float32), (R, 1))
    w = np.full((R, nb - 1), 0.25)
    N = 128
    m = np.tile(((np.arange(N) * 2 + 1) << 23) // N, (R, 1))
    t, below = nerf.sample_pdf(bins, w, m)
    u = (np.arange(N) + 0.5) / N
    np.testing.assert_allclose(t, np.tile(bins[0, 0] + u * (bins[0, -1] - bins[0, 0]), (R, 1)),
                               atol=1e-9)


def test_sample_pdf_ks_uniform_with_random_draws():
    from scipy import stats
    bins = np.linspace(0, 1, 63, dtype=np.float32)[None, :]
    m = rng.draw_bits(9, np.zeros((1, 1), dtype=np.int64), 1, np.arange(4096)[None, :])
    t, _ = nerf.sample_pdf(bins, np.full((1, 62), 0.1), m)
    assert stats.kstest(t[0], "uniform").pvalue > 1e-3


def test_sample_pdf_delta_weight_concentrates_samples():
    bins = np.linspace(2, 6, 63, dtype=np.float32)[None, :]
    w = np.zeros((1, 62))
    w[0, 17] = 1.0
    m = rng.draw_bits(1, np.zeros((1, 1), dtype=np.int64), 1, np.arange(128)[None, :])
    t, below = nerf.sample_pdf(bins, w, m)
    inside = (t >= bins[0, 17]) & (t <= bins[0, 18])
    # all but the draws that land in the 1e-5 floors of the 61 other bins
    assert inside.sum() >= 124
    assert (below == 17).sum() == inside.sum()


def pin_sample_pdf_ties_go_right():
    """searchsorted(cdf, u, right=True) (the page's sample_pdf): a draw that
    lands exactly on a CDF value takes the bin that starts there. With 62 equal
    weights the CDF after 31 of them is exactly 1/2, so u = 1/2 (m = 2^23) has
    below = 31; the drawn position is the bin edge either way."""
    t = np.tile(np.arange(64, dtype=np.float32) * np.float32(0.0625) + np.float32(2.0), (3, 1))
    w = np.full((3, 62), 0.25, dtype=np.float32)
    m = np.array([[1 << 23], [(1 << 23) - 1], [(1 << 23) + 1]])
    tf, below = nerf.sample_pdf(nerf.midpoints(t), w, m)
    assert below[0, 0] == 31 and below[1, 0] == 30 and below[2, 0] == 31, below.ravel()
    bins = nerf.midpoints(t)
    np.testing.assert_allclose(tf[0, 0], float(bins[0, 31]), atol=1e-12)


def test_sample_pdf_ties_go_right():
    pin_sample_pdf_ties_go_right()


def test_sample_pdf_bin_choice_matches_exact_rational_search():
    g = np.random.default_rng(5)
    R, nb, N = 6, 63, 128
    bins = np.sort(g.uniform(2, 6, size=(R, nb)).astype(np.float32), axis=1)
    w = (g.exponential(size=(R, nb - 1)) * (g.uniform(size=(R, nb - 1)) < 0.4)).astype(np.float32)
    m = rng.draw_bits(2, np.arange(R)[:, None], 1, np.arange(N)[None, :])
    t, below = nerf.sample_pdf(bins, w, m)
    for r in range(R):
        ww = [Fraction(float(np.float32(x) + np.float32(1e-5))) for x in w[r]]
        tot = sum(ww)
        cdf = [Fraction(0)]
        for x in ww:
            cdf.append(cdf[-1] + x / tot)
        for k in range(N):
            u = Fraction(int(m[r, k]), 1 << 24)
            idx = sum(1 for c in cdf if c <= u)       # searchsorted(right=True)
            assert below[r, k] == max(idx - 1, 0)
            lo, hi = max(idx - 1, 0), min(idx, nb - 1)
            frac = (u - cdf[lo]) / max(cdf[hi] - cdf[lo], Fraction(1, 100000))
            width = float(bins[r, hi]) - float(bins[r, lo])
            want = float(bins[r, lo]) + float(frac) * width
            # the integer CDF quantises each weight to 2^-32: the interpolation
            # moves by at most that error over the bin's (clamped) mass
            mass = max(cdf[hi] - cdf[lo], Fraction(1, 100000))
            bound = 2 * nb * 2.0 ** -32 / (float(tot) * float(mass)) * width + 1e-12
            assert abs(t[r, k] - want) <= bound


# ------------------------------------------------------------------ hash grid

def test_hashgrid_2d_level_table_printed_in_notebook():
    g = golden("instant_ngp_2d_levels.json")["experiment_1"]
    p = g["params"]
    grid = hashgrid.HashGrid2D(L=p["L"], T=p["T"], F=p["F"], N_min=p["N_min"], N_max=p["N_max"])
    assert grid.res == g["resolution"]
    assert [(n + 1) ** 2 for n in grid.res] == g["grid_vertices"]
    assert grid.direct == g["direct"]


def test_hashgrid_2d_hashed_level_counts_printed_in_notebook():
    g = golden("instant_ngp_2d_levels.json")["experiment_4"]
    for T, n_hashed in g["hashed_levels"].items():
        grid = hashgrid.HashGrid2D(T=int(T))
        assert sum(not d for d in grid.direct) == n_hashed


def test_hashgrid_3d_schedule():
    grid = hashgrid.HashGrid3D()
    assert grid.res[0] == 16 and grid.res[-1] == 2048
    assert grid.res == sorted(grid.res)
    assert grid.direct == [True] * 5 + [False] * 11
    assert grid.n_entries == 6101902


def test_hash_direct_index_is_lexicographic_bijection():
    N, T = 6, 1 << 19
    ix, iy, iz = np.meshgrid(np.arange(N + 1), np.arange(N + 1), np.arange(N + 1), indexing="ij")
    idx = hashgrid.index_3d(ix.ravel(), iy.ravel(), iz.ravel(), N, T, True)
    np.testing.assert_array_equal(idx, np.arange((N + 1) ** 3))
    idx2 = hashgrid.index_2d(ix[:, :, 0].ravel(), iy[:, :, 0].ravel(), N, 4096, True)
    np.testing.assert_array_equal(idx2, np.arange((N + 1) ** 2))


def test_hash_index_xor_structure():
    g = np.random.default_rng(6)
    T = 1 << 19
    a, b, c = (g.integers(0, 2049, size=1000) for _ in range(3))
    z = np.zeros_like(a)
    h = hashgrid.index_3d(a, b, c, 2048, T, False)
    hx = hashgrid.index_3d(a, z, z, 2048, T, False)
    hy = hashgrid.index_3d(z, b, z, 2048, T, False)
    hz = hashgrid.index_3d(z, z, c, 2048, T, False)
    np.testing.assert_array_equal(hx, a % T)               # prime 1 on x
    np.testing.assert_array_equal(h, hx ^ hy ^ hz)
    assert h.min() >= 0 and h.max() < T
    # y and z primes: the low 19 bits of iy * 2654435761 and iz * 805459861
    np.testing.assert_array_equal(hy, (b * 2654435761) & (T - 1))
    np.testing.assert_array_equal(hz, (c * 805459861) & (T - 1))


def test_hash_encoding_partition_of_unity_and_vertices():
    grid = hashgrid.HashGrid3D()
    x = np.random.default_rng(7).uniform(-1.5, 1.5, size=(300, 3)).astype(np.float32)
    ones = np.ones((grid.n_entries, 2), dtype=np.float16)
    np.testing.assert_allclose(grid.encode(x, ones), 1.0, atol=1e-12)
    pin_hash_vertices_read_their_entry()


def pin_hash_vertices_read_their_entry():
    """A point on a vertex of level 0 (N = 16) reads exactly that vertex's entry
    (the notebook's interpolation weights are 1 at the lower corner when the
    fractional part is 0). At level 0 the point x = 3v/16 - 1.5 maps back to c =
    v exactly: 3v/16 and x + 1.5 are exact in fp32, and (3v/16)/3 = v/16 is
    representable, so the correctly rounded quotient is exact."""
    grid = hashgrid.HashGrid3D()
    level, N = 0, grid.res[0]
    assert N == 16
    table = np.random.default_rng(8).uniform(-1, 1, size=(grid.n_entries, 2)).astype(np.float16)
    v = np.random.default_rng(16).integers(0, N, size=(200, 3))
    xv = (np.float32(3.0) * v.astype(np.float32) / np.float32(16.0) - np.float32(1.5)).astype(np.float32)
    c = grid.unit_coords(xv) * np.float32(N)
    np.testing.assert_array_equal(c, v.astype(np.float32))       # the guard holds on every point
    enc = grid.encode(xv, table)
    row = grid.offsets[level] + (v[:, 0] * (N + 1) + v[:, 1]) * (N + 1) + v[:, 2]
    np.testing.assert_allclose(enc[:, 0:2], table[row].astype(np.float64), atol=1e-12)


def test_hash_encoding_2d_bilinear_is_exact_on_linear_tables():
    # A table holding a linear function of the vertex coordinates is reproduced
    # exactly by bilinear interpolation (direct levels only).
    grid = hashgrid.HashGrid2D(L=3, T=1 << 14, N_min=4, N_max=16)
    assert all(grid.direct)
    tables = []
    for N in grid.res:
        ix, iy = np.meshgrid(np.arange(N + 1), np.arange(N + 1), indexing="ij")
        f = np.stack([ix.ravel() / N, 2 * iy.ravel() / N - 0.5], axis=1)
        tables.append(f)
    x = np.random.default_rng(9).uniform(0, 1, size=(100, 2)).astype(np.float32)
    enc = grid.encode(x, tables)
    for level, N in enumerate(grid.res):
        c = x * np.float32(N)
        np.testing.assert_allclose(enc[:, 2 * level], c[:, 0].astype(np.float64) / N, atol=1e-12)
        np.testing.assert_allclose(enc[:, 2 * level + 1], 2 * c[:, 1].astype(np.float64) / N - 0.5,
                                   atol=1e-12)


# ------------------------------------------------------------------ SH

def test_sh_addition_theorem_and_orthonormality():
    d = np.random.default_rng(10).normal(size=(500, 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    Y = sh.real_sh(d)
    for l in range(4):
        np.testing.assert_allclose((Y[:, l * l:(l + 1) ** 2] ** 2).sum(1), (2 * l + 1) / (4 * np.pi),
                                   atol=1e-12)
    # Gauss-Legendre in cos(theta) x uniform in phi integrates degree <= 6 exactly
    xg, wg = np.polynomial.legendre.leggauss(8)
    ph = np.arange(16) * 2 * np.pi / 16
    Z, P = np.meshgrid(xg, ph, indexing="ij")
    W = np.outer(wg, np.full(16, 2 * np.pi / 16)).ravel()
    s = np.sqrt(1 - Z ** 2)
    dirs = np.stack([s * np.cos(P), s * np.sin(P), Z], axis=-1).reshape(-1, 3)
    Yq = sh.real_sh(dirs)
    np.testing.assert_allclose(Yq.T @ (W[:, None] * Yq), np.eye(16), atol=1e-12)


def test_sh_matches_scipy_without_condon_shortley_phase():
    from scipy.special import sph_harm_y
    d = np.random.default_rng(11).normal(size=(50, 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    th = np.arccos(d[:, 2])
    ph = np.arctan2(d[:, 1], d[:, 0])
    Y = sh.real_sh(d)
    for l in range(4):
        for m in range(-l, l + 1):
            c = sph_harm_y(l, abs(m), th, ph) * (-1) ** abs(m)      # remove the CS phase
            want = c.real if m == 0 else math.sqrt(2) * (c.real if m > 0 else c.imag)
            np.testing.assert_allclose(Y[:, l * l + l + m], want, atol=1e-12)


# ------------------------------------------------------------------ march

def test_voxel_coords_match_exact_rationals():
    g = np.random.default_rng(12)
    x = g.uniform(-1.6, 1.6, size=(2000, 3)).astype(np.float32)
    edges = (-1.5 + np.arange(129) * 3 / 128).astype(np.float32)
    x[:200] = g.choice(edges, size=(200, 3))                        # exact boundaries
    x[200:300] = np.nextafter(g.choice(edges, size=(100, 3)), np.float32(-9))
    x[300:310] = np.float32(-2 ** -100)
    v = march.voxel_coords(x)
    for p in range(310 + 200):
        for a in range(3):
            q = Fraction(float(x[p, a]))
            k = math.floor((q + Fraction(3, 2)) * 128 / 3)
            assert v[p, a] == (k if 0 <= k < 128 else -1)


def test_occupancy_and_cell_routing():
    packed, dense = S.occupancy_grid(4)
    assert dense.sum() == int(0.1 * 128 ** 3)
    # the bit-packed form holds the same grid (x-major, bit = index & 31)
    idx = np.arange(128 ** 3)
    bits = (packed[idx >> 5] >> (idx & 31).astype(np.uint32)) & 1
    np.testing.assert_array_equal(bits.astype(bool), dense.ravel())
    x = np.random.default_rng(13).uniform(-1.5, 1.5, size=(1000, 3)).astype(np.float32)
    v = march.voxel_coords(x)
    np.testing.assert_array_equal(march.occupied(x, dense), dense[v[:, 0], v[:, 1], v[:, 2]])
    c = march.cell_id(x)
    np.testing.assert_array_equal(c, ((v[:, 0] // 8) * 16 + v[:, 1] // 8) * 16 + v[:, 2] // 8)


def test_kilonerf_points_use_their_own_cell():
    # every cell's sigma head is bias-only with bias = cell id: sigma = cell id
    n_cells = 16 ** 3
    p = np.zeros((n_cells, 3317), dtype=np.float32)
    off = 32 * 63 + 32 + 32 * 32 + 32 + 32        # start of the sigma bias
    p[:, off] = np.arange(n_cells)
    x = np.random.default_rng(14).uniform(-1.5, 1.5, size=(500, 3)).astype(np.float32)
    du = nerf.unit(np.random.default_rng(15).normal(size=(500, 3)))
    cells = march.cell_id(x)
    sigma, rgb = march.kilonerf_eval(p, cells, x, du)
    np.testing.assert_array_equal(sigma, cells.astype(np.float64))
    np.testing.assert_allclose(rgb, 0.5)


def test_render_march_constant_medium_and_termination():
    dense = np.ones((128, 128, 128), dtype=bool)
    import dataclasses
    wl = dataclasses.replace(S.WORKLOADS["kilonerf"], ert_T=0.0)
    o = np.array([[0.0, 0.0, 4.0]], dtype=np.float32)
    d = np.array([[0.0, 0.0, -1.0]], dtype=np.float32)
    sig, col = 0.9, np.array([0.3, 0.6, 0.1])

    def const(idx, x, du):
        return np.full(len(idx), sig), np.tile(col, (len(idx), 1))

    r = march.render_march(wl, o, d, dense, const)
    # samples at t in [2.5, 5.5) lie inside the cube z in (-1.5, 1.5]
    t = nerf.march_t(wl.near, wl.march_step, wl.n_coarse)
    z = o[0, 2] + t * d[0, 2]
    n_in = int(((z >= -1.5) & (z < 1.5)).sum())
    assert r["n_live"][0] == n_in
    want = 1 - math.exp(-sig * wl.march_step * n_in)
    np.testing.assert_allclose(r["acc"][0], want, atol=1e-12)
    np.testing.assert_allclose(r["rgb"][0], want * col, atol=1e-12)
    # early termination: stop before the first sample with T < 1e-3
    wl2 = dataclasses.replace(wl, ert_T=1e-3)
    r2 = march.render_march(wl2, o, d, dense, lambda i, x, du: (np.full(len(i), 30.0),
                                                                 np.tile(col, (len(i), 1))))
    tau = 30.0 * wl.march_step
    k_stop = next(k for k in range(1, 1000) if math.exp(-k * tau) < 1e-3)
    assert r2["n_live"][0] == k_stop
    np.testing.assert_allclose(r2["acc"][0], 1 - math.exp(-k_stop * tau), atol=1e-12)


# ------------------------------------------------------------------ end to end

def _tiny_render_scalar(shape, params, o, d, t_list, seed_u, perturb, near, far, n):
    """Pure-Python scalar render of one ray, coarse pass only (page mode)."""
    raw = []
    dn = math.sqrt(sum(float(v) ** 2 for v in d))
    du = [float(v) / dn for v in d]

    def pe(v, L):
        out = list(v)
        out += [math.sin(2 ** k * math.pi * v[c]) for c in range(3) for k in range(L)]
        out += [math.cos(2 ** k * math.pi * v[c]) for c in range(3) for k in range(L)]
        return out

    def lin(name, a):
        w, b = params[name]
        return [sum(w[i][k] * a[k] for k in range(len(a))) + b[i] for i in range(len(b))]

    de = pe(du, shape.L_dir)
    for t in t_list:
        x = [float(np.float32(o[c]) + np.float32(t) * np.float32(d[c])) for c in range(3)]
        pex = pe(x, shape.L_pos)
        h = pex
        for i in range(shape.D):
            h = [max(0.0, v) for v in lin(f"pts{i}", h)]
            if i == shape.skip:
                h = h + pex
        s = lin("sigma", h)[0]
        f = lin("feature", h)
        hh = [max(0.0, v) for v in lin("dir", f + de)]
        raw.append((lin("rgb", hh), s))
    C, T, acc = [0.0] * 3, 1.0, 0.0
    for i, (rgb, s) in enumerate(raw):
        dist = ((t_list[i + 1] - t_list[i]) if i + 1 < len(t_list) else 1e10) * dn
        sigma = math.log1p(math.exp(s)) if s < 30 else s
        a = 1 - math.exp(-sigma * dist)
        w = T * a
        C = [C[k] + w / (1 + math.exp(-rgb[k])) for k in range(3)]
        acc += w
        T *= 1 - a
    return C, acc


def test_end_to_end_tiny_image_brute_force():
    import dataclasses
    shape = S.MLPShape(D=2, W=8, skip=0, L_pos=3, L_dir=2)
    wl = dataclasses.replace(S.WORKLOADS["tiny"], H=2, W=2, focal=1.5, mlp=shape, n_coarse=8)
    flat, _ = S.nerf_weights(shape, 21, 0)
    o, d = nerf.raygen(wl.H, wl.W, wl.focal, wl.c2w())
    ids = np.arange(4)
    res = nerf.render_nerf(wl, o, d, ids, flat)
    params = nerf.split_params(shape, flat)
    params = {k: (v[0].tolist(), v[1].tolist()) for k, v in params.items()}
    t = nerf.stratified_t(wl.near, wl.far, wl.n_coarse, wl.seed, ids)
    for r in range(4):
        C, acc = _tiny_render_scalar(shape, params, o[r], d[r], [float(v) for v in t[r]],
                                     wl.seed, True, wl.near, wl.far, wl.n_coarse)
        np.testing.assert_allclose(res["rgb"][r], C, atol=1e-10)
        np.testing.assert_allclose(res["acc"][r], acc, atol=1e-10)
