"""Pins of the hash-grid encoding's backward (oracle/hashgrid.py,
HashGrid3D.encode_backward) against the mathematics: the adjoint identity of a
linear map, a one-entry brute force through the forward, and a point on a grid
vertex, where one corner carries the whole weight."""
import numpy as np

from oracle.hashgrid import HashGrid3D


def _points(rng, n):
    return rng.uniform(-1.5, 1.5, size=(n, 3)).astype(np.float32)


def test_adjoint_identity():
    """<encode_backward(x, g), table> == <g, encode(x, table)> for any table, g."""
    hg = HashGrid3D()
    rng = np.random.default_rng(0)
    x = _points(rng, 40)
    g = rng.normal(size=(40, hg.L * hg.F))
    table = rng.normal(size=(hg.n_entries, hg.F))
    lhs = float((hg.encode_backward(x, g) * table).sum())
    rhs = float((g * hg.encode(x, table)).sum())
    assert abs(lhs - rhs) <= 1e-10 * max(1.0, abs(rhs))


def test_brute_force_single_entries():
    """The derivative of sum(g * encode) with respect to one table entry, taken
    through the forward (the encoding is linear: a unit change is exact)."""
    hg = HashGrid3D()
    rng = np.random.default_rng(1)
    x = _points(rng, 5)
    g = rng.normal(size=(5, hg.L * hg.F))
    grad = hg.encode_backward(x, g)
    base = np.zeros((hg.n_entries, hg.F))
    f0 = float((g * hg.encode(x, base)).sum())
    touched = np.unique(np.concatenate([hg.corners(x, l)[0].ravel() for l in (0, 7, 15)]))
    for row in list(touched[:6]) + [int(rng.integers(hg.n_entries))]:
        for f in range(hg.F):
            t = base.copy()
            t[row, f] = 1.0
            d = float((g * hg.encode(x, t)).sum()) - f0
            assert abs(d - grad[row, f]) <= 1e-12, (row, f, d, grad[row, f])


def test_vertex_point_goes_to_one_row():
    """A point on a vertex of level 0's grid (c exactly integral on every axis)
    sends its whole level-0 gradient to that vertex's row."""
    hg = HashGrid3D()
    N = hg.res[0]
    # x01 = i / N exactly representable and (x + 1.5) / 3 rounds to it
    i = np.array([3, 7, 11])
    x01 = (i / N).astype(np.float32)
    x = (x01.astype(np.float64) * 3.0 - 1.5).astype(np.float32)[None, :]
    assert np.array_equal(hg.unit_coords(x) * np.float32(N), i.astype(np.float32)[None, :])
    g = np.zeros((1, hg.L * hg.F))
    g[0, 0:2] = [2.0, -3.0]
    grad = hg.encode_backward(x, g)
    rows, wts = hg.corners(x, 0)
    assert wts[0, 0] == 1.0
    assert np.array_equal(np.nonzero(grad[:, 0])[0], [rows[0, 0]])
    assert np.array_equal(grad[rows[0, 0]], [2.0, -3.0])
