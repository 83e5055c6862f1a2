"""Failure handling on the GPU without a fault: a bounded wait that runs out.

The bounded mbarrier wait every kernel uses is run on a barrier that nothing completes.  It
must give up after its time limit, raise the timeout bit of the device error word, and leave
the context usable: vsa_get_device_error maps the word to VSA_ERR_TIMEOUT and later work runs.
"""
import time

import pytest
import torch

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from block_sparse_attention_31_b200 import _lib
else:
    _lib = None


def test_bounded_wait_times_out_and_context_survives():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    waited = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    t0 = time.monotonic()
    _lib.vsa_selftest_wait_timeout(err, waited)
    status = _lib.lib.vsa_get_device_error(_lib._ptr(err), _lib._stream(None), None)
    elapsed = time.monotonic() - t0
    assert status == _lib.VSA_ERR_TIMEOUT
    assert err.item() & _lib.VSA_DEVERR_TIMEOUT
    assert waited.item() == 0
    assert 0.5 < elapsed < 30.0
    # the context still works
    x = torch.linspace(-4, 4, 1024, device="cuda")
    yp, ym = torch.empty_like(x), torch.empty_like(x)
    _lib.vsa_selftest_exp2(x, yp, ym)
    torch.cuda.synchronize()
    assert torch.allclose(ym, torch.exp2(x), rtol=1e-5)
