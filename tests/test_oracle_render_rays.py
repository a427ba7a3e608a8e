"""A scalar brute force of the whole render_rays of "Spatial Intelligence - Part
1: NeRF" (Sections 2.2-2.6: get_rays, the stratified coarse samples,
positional_encoding, the NeRF network, volume_render, sample_pdf over the
midpoints with the interior coarse weights, the sorted union and the fine pass,
whose output is the result) on a 4x4 image, against oracle.nerf.render_nerf.

The brute force is written ray by ray and sample by sample in plain Python
floats, with the transmittance as the page's running product of (1 - alpha)
rather than the oracle's exp(-cumsum). Where the page leaves the arithmetic open
it takes the readings that the oracle documents, implemented independently:
fp32 ray directions, sample positions and points; the inverse CDF exact over
the fp32 values w + 1e-5 quantised to 2^-32 (evaluated here with Python
integers and Fractions; pinned against the page's float CDF in
test_oracle_pins.py); the drawn positions rounded to fp32. Without the 1e-10
survival guard the two agree to rounding (1e-9); the guard itself moves a pass
by at most 2 S 1e-10 (checked on the same positions)."""
import dataclasses
import math
from fractions import Fraction

import numpy as np

import nerf_inputs as S
from oracle import nerf
from oracle import rng

F32 = np.float32


def _pe(v, L):
    out = [float(c) for c in v]
    out += [math.sin(2.0 ** k * math.pi * float(v[c])) for c in range(3) for k in range(L)]
    out += [math.cos(2.0 ** k * math.pi * float(v[c])) for c in range(3) for k in range(L)]
    return out


def _network(shape, p, x, de):
    """raw (r, g, b, sigma) of the page's network at one point."""
    def lin(name, a):
        w, b = p[name]
        return [sum(w[i][k] * a[k] for k in range(len(a))) + b[i] for i in range(len(b))]
    pex = _pe(x, shape.L_pos)
    h = pex
    for i in range(shape.D):
        h = [max(0.0, v) for v in lin(f"pts{i}", h)]
        if i == shape.skip:
            h = h + pex
    sigma = lin("sigma", h)[0]
    feat = lin("feature", h)
    hd = [max(0.0, v) for v in lin("dir", feat + de)]
    return lin("rgb", hd) + [sigma]


def _volume_render(raws, ts, dn, white, guard):
    """Page mode (last interval 1e10), ReLU density, sigmoid colour; the
    transmittance is the running product of (1 - alpha) (+ 1e-10 with guard)."""
    n = len(ts)
    T, rgb, depth, acc, ws = 1.0, [0.0, 0.0, 0.0], 0.0, 0.0, []
    for i in range(n):
        dist = ((ts[i + 1] - ts[i]) if i + 1 < n else 1e10) * dn
        sigma = max(0.0, raws[i][3])
        alpha = 1.0 - math.exp(-sigma * dist)
        w = T * alpha
        ws.append(w)
        for c in range(3):
            rgb[c] += w / (1.0 + math.exp(-raws[i][c]))
        depth += w * ts[i]
        acc += w
        T *= (1.0 - alpha) + (1e-10 if guard else 0.0)
    if white:
        rgb = [v + 1.0 - acc for v in rgb]
    return rgb, depth, acc, ws


def _sample_pdf(bins, weights, ms):
    """Inverse-CDF draws: q_i = floor(fl32(w_i + 1e-5) 2^32), C_k = sum_{i<k} q_i,
    idx = #{k : C_k <= u C_total} (searchsorted right), below/above clamped,
    t = b_below + (u C_total - C_below) / max(C_above - C_below, 1e-5 C_total)
    (b_above - b_below), with u = m 2^-24, rounded to fp32."""
    q = [math.floor(float(F32(F32(w) + F32(1e-5))) * 2.0 ** 32) for w in weights]
    C = [0]
    for v in q:
        C.append(C[-1] + v)
    tot = C[-1]
    nb = len(C)
    out, belows = [], []
    for m in ms:
        u = Fraction(int(m), 1 << 24)
        idx = sum(1 for c in C if c <= u * tot)
        lo, hi = max(idx - 1, 0), min(idx, nb - 1)
        frac = (u * tot - C[lo]) / max(Fraction(C[hi] - C[lo]), Fraction(tot, 100000))
        t = Fraction(float(bins[lo])) + frac * (Fraction(float(bins[hi])) - Fraction(float(bins[lo])))
        out.append(float(F32(float(t))))
        belows.append(lo)
    return out, belows


def brute_force_render_rays(wl, coarse_flat, fine_flat, guard=False):
    shape = wl.mlp
    pc = {k: (v[0].tolist(), v[1].tolist()) for k, v in nerf.split_params(shape, coarse_flat).items()}
    pf = {k: (v[0].tolist(), v[1].tolist()) for k, v in nerf.split_params(shape, fine_flat).items()}
    c = wl.c2w().astype(F32)
    f = F32(wl.focal)
    res = {k: [] for k in ("rgb", "depth", "acc", "t_f", "below", "rgb_guard", "acc_guard")}
    step = F32(F32(wl.far) - F32(wl.near)) / F32(wl.n_coarse)
    for j in range(wl.H):
        for i in range(wl.W):
            ray = j * wl.W + i
            # get_rays: ((i - W/2)/f, -(j - H/2)/f, -1) rotated by c2w, fp32
            dx = F32(F32(F32(i) - F32(F32(wl.W) * F32(0.5))) / f)
            dy = -F32(F32(F32(j) - F32(F32(wl.H) * F32(0.5))) / f)
            dz = F32(-1.0)
            d = [F32(F32(F32(dx * c[r, 0]) + F32(dy * c[r, 1])) + F32(dz * c[r, 2])) for r in range(3)]
            o = [c[r, 3] for r in range(3)]
            dn = math.sqrt(sum(float(v) ** 2 for v in d))
            de = _pe([float(v) / dn for v in d], shape.L_dir)

            def point(t):
                return [F32(o[r] + F32(F32(t) * d[r])) for r in range(3)]

            # coarse: N_c strata, one jitter each
            tc = []
            for k in range(wl.n_coarse):
                u = F32(rng.draw_uniform(wl.seed, ray, 0, k))
                tc.append(float(F32(F32(wl.near) + F32(F32(F32(k) + u) * step))))
            raw_c = [_network(shape, pc, point(t), de) for t in tc]
            _, _, _, wc = _volume_render(raw_c, tc, dn, wl.white_bkgd, guard=False)
            # sample_pdf over the midpoints with the interior weights
            bins = [F32(F32(0.5) * F32(F32(tc[k]) + F32(tc[k + 1]))) for k in range(wl.n_coarse - 1)]
            ms = [rng.draw_bits(wl.seed, ray, 1, k) for k in range(wl.n_fine)]
            tf, below = _sample_pdf(bins, wc[1:-1], ms)
            t_all = sorted(tc + tf)
            raw_f = [_network(shape, pf, point(t), de) for t in t_all]
            rgb, depth, acc, _ = _volume_render(raw_f, t_all, dn, wl.white_bkgd, guard=False)
            rgb_g, _, acc_g, _ = _volume_render(raw_f, t_all, dn, wl.white_bkgd, guard=True)
            for k, v in (("rgb", rgb), ("depth", depth), ("acc", acc), ("t_f", tf),
                         ("below", below), ("rgb_guard", rgb_g), ("acc_guard", acc_g)):
                res[k].append(v)
    return {k: np.array(v) for k, v in res.items()}


def tiny_coarse_fine_workload():
    shape = S.MLPShape(D=2, W=8, skip=0, L_pos=3, L_dir=2)
    return dataclasses.replace(S.WORKLOADS["small"], H=4, W=4, focal=5.0, mlp=shape, n_coarse=16,
                               n_fine=24, seed=23)


def pin_render_rays_brute_force():
    wl = tiny_coarse_fine_workload()
    cw, _ = S.nerf_weights(wl.mlp, wl.seed, 0)
    fw, _ = S.nerf_weights(wl.mlp, wl.seed, 1)
    bf = brute_force_render_rays(wl, cw, fw)
    o, d = nerf.raygen(wl.H, wl.W, wl.focal, wl.c2w())
    ref = nerf.render_nerf(wl, o, d, np.arange(wl.n_rays), cw, fw, return_aux=True)
    np.testing.assert_array_equal(ref["below"], bf["below"])
    np.testing.assert_array_equal(ref["t_f"].astype(F32), bf["t_f"].astype(F32))
    for k in ("rgb", "depth", "acc"):
        np.testing.assert_allclose(ref[k], bf[k], rtol=0, atol=1e-9, err_msg=k)
    return wl, bf, ref


def test_render_rays_brute_force_4x4():
    wl, bf, ref = pin_render_rays_brute_force()
    # the image is not degenerate: partly transparent, and the fine pass differs
    # from the coarse one
    assert 0.05 < ref["acc"].mean() < 0.999
    assert np.abs(ref["rgb"] - ref["rgb_c"]).max() > 1e-3
    # the page's 1e-10 survival guard moves a pass by at most 2 S 1e-10
    S_ = wl.n_coarse + wl.n_fine
    assert np.abs(bf["acc_guard"] - bf["acc"]).max() <= 2 * S_ * 1e-10
    assert np.abs(bf["rgb_guard"] - bf["rgb"]).max() <= 2 * S_ * 1e-10
