"""The oracle's pins catch the mistakes they guard.

Each case plants one plausible mistake in a copy of an oracle function (its
source with one expression changed, compiled into the oracle module's
namespace and patched in for the duration of the test), then runs the pin that
guards it and requires the pin to fail. The oracle itself is never changed on
disk. The mistakes: a swapped trilinear weight, a transposed direct index, the
colour branch of either scene network reading its inputs in the wrong order, a
skipped layer, the fine pass drawing from the wrong coarse weights or bins,
skipping the sort, returning the coarse result, an inclusive transmittance
scan, searchsorted on the wrong side, and positional encoding without pi."""
import inspect
import textwrap

import pytest

from oracle import hashgrid, march, nerf

import test_oracle_pins as pins
import test_oracle_render_rays as rr
import test_oracle_scene_pins as scene


def mutated(owner, name, old, new):
    """`owner.name` recompiled from its source with `old` replaced by `new`."""
    fn = getattr(owner, name)
    src = textwrap.dedent(inspect.getsource(fn))
    assert src.count(old) == 1, (name, old)
    module = inspect.getmodule(fn)
    ns = dict(module.__dict__)
    exec(compile(src.replace(old, new), f"<{name} with a planted mistake>", "exec"), ns)
    return ns[name]


CASES = [
    # (id, owner, function, old, new, pins that must fail)
    ("trilinear weight swapped", hashgrid.HashGrid3D, "corners",
     "wx = w[:, 0] if dx else 1.0 - w[:, 0]", "wx = 1.0 - w[:, 0] if dx else w[:, 0]",
     [scene.pin_hash_trilinear_exact_on_linear_tables, pins.pin_hash_vertices_read_their_entry]),
    ("direct index transposed", hashgrid, "index_3d",
     "(ix * (N + 1) + iy) * (N + 1) + iz", "(iz * (N + 1) + iy) * (N + 1) + ix",
     [pins.test_hash_direct_index_is_lexicographic_bijection,
      pins.pin_hash_vertices_read_their_entry]),
    ("hash colour input [SH, h]", march, "hash_eval",
     "np.concatenate([h, sh.real_sh(d_unit)], axis=-1)",
     "np.concatenate([sh.real_sh(d_unit), h], axis=-1)",
     [scene.pin_hash_network_routing]),
    ("hash density layer d1 skipped", march, "hash_eval",
     'h = nerf.relu(lin("d1", nerf.relu(lin("d0", enc))))', 'h = nerf.relu(lin("d0", enc))',
     [scene.pin_hash_network_routing]),
    ("KiloNeRF colour input [gamma(d), h2]", march, "kilonerf_eval",
     "np.concatenate([h2, de], axis=-1)", "np.concatenate([de, h2], axis=-1)",
     [scene.pin_kilonerf_routing]),
    ("KiloNeRF l2 skipped", march, "kilonerf_eval",
     'h2 = nerf.relu(lin("l2", h1))', "h2 = h1",
     [scene.pin_kilonerf_routing]),
    ("pdf from w[:, :-2]", nerf, "render_nerf", "w_c[:, 1:-1]", "w_c[:, :-2]",
     [rr.pin_render_rays_brute_force]),
    ("bins at the samples, not the midpoints", nerf, "render_nerf",
     "bins = midpoints(t_c)", "bins = t_c[:, 1:]",
     [rr.pin_render_rays_brute_force]),
    ("union not sorted", nerf, "render_nerf",
     "t_all = np.sort(np.concatenate([t_c, t_f], axis=-1), axis=-1)",
     "t_all = np.concatenate([t_c, t_f], axis=-1)",
     [rr.pin_render_rays_brute_force]),
    ("coarse result returned", nerf, "render_nerf",
     'res["rgb"].append(rgb)\n', 'res["rgb"].append(rgb_c)\n',
     [rr.pin_render_rays_brute_force]),
    ("inclusive transmittance", nerf, "composite",
     "T = np.exp(-excl)", "T = np.exp(-np.cumsum(tau, axis=-1))",
     [rr.pin_render_rays_brute_force, pins.test_composite_constant_medium_closed_form]),
    ("searchsorted left", nerf, "sample_pdf", "(lhs <= rhs)", "(lhs < rhs)",
     [pins.pin_sample_pdf_ties_go_right]),
    ("positional encoding without pi", nerf, "positional_encoding",
     "np.pi * x[..., :, None] * freqs", "x[..., :, None] * freqs",
     [rr.pin_render_rays_brute_force, pins.test_positional_encoding_special_values_and_layout]),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_pin_fails_on_planted_mistake(monkeypatch, case):
    _, owner, name, old, new, guards = case
    monkeypatch.setattr(owner, name, mutated(owner, name, old, new))
    for pin in guards:
        with pytest.raises(AssertionError):
            pin()


def test_pins_pass_on_the_oracle_as_it_stands():
    for case in CASES:
        for pin in case[5]:
            pin()
