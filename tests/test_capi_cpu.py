"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point that include/nerf.h declares, and rejects bad arguments
before touching a device."""
import ctypes
import os
import re

import pytest

from neural_radiance_field_b200 import _capi
from neural_radiance_field_b200 import build as nbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    nbuild.build()
    return _capi.lib()


def header_functions():
    with open(os.path.join(ROOT, "include", "nerf.h")) as f:
        text = f.read()
    return re.findall(r"NERF_API\s+[\w\s\*]+?\b(nerf_\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    names = header_functions()
    for n in ("nerf_create", "nerf_render", "nerf_destroy", "nerf_render_host", "nerf_raygen"):
        assert n in names
    assert set(names) == set(_capi.SIGNATURES), "binding and header disagree"


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name


def test_create_rejects_bad_configs_without_a_device(lib):
    h = ctypes.c_void_p()
    cfg = _capi.nerf_config(0, 8, 256, 4, 10, 4, 0, 0, 0, 0, 0, 192)      # max_rays = 0
    assert lib.nerf_create(ctypes.byref(cfg), ctypes.byref(h)) == _capi.NERF_ERR_INVALID_ARG
    assert h.value is None
    assert b"max_rays" in lib.nerf_last_error(None)
    cfg = _capi.nerf_config(0, 8, 96, 4, 10, 4, 0, 0, 0, 0, 16, 192)      # W = 96
    assert lib.nerf_create(ctypes.byref(cfg), ctypes.byref(h)) == _capi.NERF_ERR_UNSUPPORTED
    cfg = _capi.nerf_config(0, 4, 128, 3, 10, 4, 0, 0, 0, 0, 16, 192)     # skip after the last layer
    assert lib.nerf_create(ctypes.byref(cfg), ctypes.byref(h)) == _capi.NERF_ERR_UNSUPPORTED
    cfg = _capi.nerf_config(0, 9, 128, -1, 10, 4, 0, 0, 0, 0, 16, 192)    # D = 9
    assert lib.nerf_create(ctypes.byref(cfg), ctypes.byref(h)) == _capi.NERF_ERR_UNSUPPORTED
    cfg = _capi.nerf_config(0, 4, 64, -1, 10, 4, 0, 1, 0, 0, 16, 192)     # bf16 tiny
    assert lib.nerf_create(ctypes.byref(cfg), ctypes.byref(h)) == _capi.NERF_ERR_UNSUPPORTED
    cfg = _capi.nerf_config(0, 4, 64, -1, 10, 4, 0, 2, 0, 0, 16, 192)     # TF32 at W = 64
    assert lib.nerf_create(ctypes.byref(cfg), ctypes.byref(h)) == _capi.NERF_ERR_UNSUPPORTED
    assert b"TF32" in lib.nerf_last_error(None)
    cfg = _capi.nerf_config(0, 8, 256, 4, 10, 4, 0, 3, 0, 0, 16, 192)     # precision 3
    assert lib.nerf_create(ctypes.byref(cfg), ctypes.byref(h)) == _capi.NERF_ERR_INVALID_ARG
    cfg = _capi.nerf_config(7, 8, 256, 4, 10, 4, 0, 0, 0, 0, 16, 192)     # unknown model
    assert lib.nerf_create(ctypes.byref(cfg), ctypes.byref(h)) == _capi.NERF_ERR_INVALID_ARG
    cfg = _capi.nerf_config(2, 8, 256, 4, 10, 4, 0, 2, 0, 0, 16, 512)     # hash grid, precision 2
    assert lib.nerf_create(ctypes.byref(cfg), ctypes.byref(h)) == _capi.NERF_ERR_INVALID_ARG
    assert b"precision" in lib.nerf_last_error(None)
    assert lib.nerf_create(None, ctypes.byref(h)) == _capi.NERF_ERR_INVALID_ARG


def test_unit_entry_points_reject_null_and_bad_sizes(lib):
    assert lib.nerf_test_pe(None, 4, 10, None, None) == _capi.NERF_ERR_INVALID_ARG
    fake = ctypes.c_void_p(16)   # never dereferenced: validation fails first
    assert lib.nerf_test_pe(fake, 0, 10, fake, None) == _capi.NERF_ERR_INVALID_ARG
    assert lib.nerf_test_sample_pdf(fake, fake, 4, 32, 128, 0, 1, fake, None, None, None) \
        == _capi.NERF_ERR_INVALID_ARG
    assert lib.nerf_test_composite(fake, fake, fake, 4, 600, 6.0, 0, 0.0, 0, 0, fake, fake, fake,
                                   None, None) == _capi.NERF_ERR_INVALID_ARG
    assert lib.nerf_raygen(0, 4, 1.0, None, fake, fake, None) == _capi.NERF_ERR_INVALID_ARG
    assert lib.nerf_render(None, fake, fake, 4, 2.0, 6.0, 64, 0, None, fake, fake, fake, None) \
        == _capi.NERF_ERR_INVALID_ARG
    assert lib.nerf_destroy(None) == _capi.NERF_OK


def test_params_keep_their_tensors_alive():
    """The context reads weights through raw pointers on every call, so the
    params object must keep the tensors it points at: a temporary passed to
    params() is not freed (and its memory reused) while the params are alive."""
    import gc
    import weakref
    import torch
    import neural_radiance_field_b200 as nb
    w = torch.arange(8, dtype=torch.float32)
    ref = weakref.ref(w)
    p = nb.Renderer.params(coarse_w=w, fine_w=torch.ones(8), seed=1)
    del w
    gc.collect()
    assert ref() is not None and p.coarse_w == ref().data_ptr()
    del p
    gc.collect()
    assert ref() is None


def header_prototypes():
    """name -> (return type, parameter count) of every NERF_API declaration."""
    text = open(os.path.join(ROOT, "include", "nerf.h")).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    out = {}
    for m in re.finditer(r"NERF_API\s+([\w\s\*]+?)\b(nerf_\w+)\s*\(([^;]*?)\)\s*;", text, flags=re.S):
        ret, name, params = m.group(1).strip(), m.group(2), m.group(3).strip()
        n = 0 if params in ("", "void") else len(params.split(","))
        out[name] = (ret, n)
    return out


def test_binding_signatures_match_the_header():
    """Every ctypes prototype of the binding has the header's parameter count and
    a matching return type, so no call can shift or drop an argument."""
    import ctypes
    protos = header_prototypes()
    assert set(protos) == set(_capi.SIGNATURES)
    for name, (ret, n) in protos.items():
        res, args = _capi.SIGNATURES[name]
        assert len(args) == n, (name, len(args), n)
        if "char" in ret:
            assert res is ctypes.c_char_p, name
        else:
            assert ret.endswith("nerf_status") and res is ctypes.c_int, (name, ret)
