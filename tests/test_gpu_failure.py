"""Failure detection without a GPU fault: a bounded device wait on a barrier
that nothing completes gives up, reports the timeout bit, and leaves the
context usable for the next render."""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    import torch
    from neural_radiance_field_b200 import _capi, build
    import neural_radiance_field_b200 as nb
    build.build()
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    waited = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = _capi.lib().nerf_test_bounded_wait(20000, ctypes.c_void_p(flag.data_ptr()),
                                            ctypes.c_void_p(waited.data_ptr()), st)
    assert rc == _capi.NERF_OK
    torch.cuda.synchronize()
    assert int(flag.item()) & 2                       # timeout bit
    assert int(waited.item()) >= 20000                # waited out the bound
    assert int(waited.item()) < 2000000
    # the context still renders
    x = torch.rand(1000, 3, device="cuda")
    out = torch.empty(1000, 3 + 6 * 4, device="cuda")
    nb.nerf_test_pe(x, 4, out)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    # argument errors are reported before any launch
    assert _capi.lib().nerf_test_bounded_wait(0, ctypes.c_void_p(flag.data_ptr()), None, st) \
        == _capi.NERF_ERR_INVALID_ARG
