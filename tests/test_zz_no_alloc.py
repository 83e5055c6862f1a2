"""vsa_profile_heads_static: head profiling for callers that cannot allocate device memory.

Some users run this library inside a host framework that has already reserved all device
memory for its own pool, or on a latency-critical path that must not call cudaMalloc (which
can synchronise the device).  They cannot hand vsa_profile_heads a workspace, so the library
offers a variant that keeps its scratch in a fixed array of its own.  This test calls that
variant through the C ABI, twice in a row on the same inputs, and checks each result against
the workspace-taking entry point.  It also checks that a shape too large for the fixed array
is refused before anything is launched, and that the variant still works after the device's
context was reset (its array's address is looked up per call, never cached).  The file is
collected last, so a run that stops at its first failure has run every other test before it.
"""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from block_sparse_attention_31_b200 import _lib
else:
    _lib = None


def _profile_with_workspace(q, k, v, shape, params, H):
    ws_bytes = _lib.vsa_profile_workspace_size(shape, params)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    kinds = torch.full((H,), 7, dtype=torch.uint8, device="cuda")
    mse = torch.zeros(H * 2, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.vsa_profile_heads(q, k, v, shape, params, kinds, mse, ws, ws_bytes, err)
    assert _lib.vsa_get_device_error(err) == 0
    return kinds.cpu().numpy(), mse.cpu().numpy().reshape(-1, 2)


def _profile_static(q, k, v, shape, params, H):
    kinds = torch.full((H,), 7, dtype=torch.uint8, device="cuda")
    mse = torch.full((H * 2,), -1.0, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.vsa_profile_heads_static(q, k, v, shape, params, kinds, mse, err)
    assert _lib.vsa_get_device_error(err) == 0
    return kinds.cpu().numpy(), mse.cpu().numpy().reshape(-1, 2)


def _close(got, want):
    # same tolerance as the other profiling checks: 2% on each error, 1e-4 absolute floor
    return np.all(np.abs(got - want) <= np.maximum(2e-2 * np.abs(want), 1e-4))


@pytest.mark.parametrize("wl,w_s,w_t", [
    (synthetic.Workload("no-alloc small", 1, 4, 6, 8, 16, 128, 128, "bf16", "profiled"), 1, 40),
    (synthetic.WAN, 2, 140),
])
def test_static_scratch_matches_workspace_entry_point(wl, w_s, w_t):
    q, k, v = (t.cuda() for t in synthetic.make_qkv(wl))
    shape = _lib.make_shape(wl.B, wl.H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block)
    params = _lib.make_params(w_s, w_t, profile_frac=wl.profile_frac)
    want_kinds, want_mse = _profile_with_workspace(q, k, v, shape, params, wl.H)
    for _ in range(2):  # the fixed scratch is reused; the second call must not see stale state
        kinds, mse = _profile_static(q, k, v, shape, params, wl.H)
        assert np.array_equal(kinds, want_kinds)
        assert _close(mse, want_mse), (mse, want_mse)


def test_static_scratch_refuses_oversized_shapes():
    assert _lib.vsa_profile_static_scratch_bytes() == 16 << 20
    wl = synthetic.HUNYUAN
    shape = _lib.make_shape(wl.B, wl.H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block)
    params = _lib.make_params(3, 337, profile_frac=0.01)
    dummy = torch.zeros(16, dtype=torch.bfloat16, device="cuda")   # never read: refused first
    kinds = torch.zeros(wl.H, dtype=torch.uint8, device="cuda")
    mse = torch.zeros(wl.H * 2, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(_lib.VsaError) as exc:
        _lib.vsa_profile_heads_static(dummy, dummy, dummy, shape, params, kinds, mse, err)
    assert exc.value.status == _lib.VSA_ERR_WORKSPACE
    assert _lib.vsa_get_device_error(err) == 0


# Child process: device buffers come from the driver API (no torch CUDA state), the library
# resets the context through its own runtime, and the same call on new buffers must give the
# same bits as before the reset.
_RESET_CHILD = textwrap.dedent("""
    import ctypes, sys
    import numpy as np
    sys.path.insert(0, sys.argv[1])
    import synthetic
    from block_sparse_attention_31_b200 import _lib

    cu = ctypes.CDLL("libcuda.so.1")
    def ck(r):
        assert r == 0, f"driver call failed: {r}"
    def context():
        dev, ctx = ctypes.c_int(), ctypes.c_void_p()
        ck(cu.cuDeviceGet(ctypes.byref(dev), 0))
        ck(cu.cuDevicePrimaryCtxRetain(ctypes.byref(ctx), dev))
        ck(cu.cuCtxSetCurrent(ctx))
    def upload(arr):
        p = ctypes.c_uint64()
        ck(cu.cuMemAlloc_v2(ctypes.byref(p), ctypes.c_size_t(max(arr.nbytes, 16))))
        ck(cu.cuMemcpyHtoD_v2(ctypes.c_uint64(p.value), arr.ctypes.data_as(ctypes.c_void_p),
                              ctypes.c_size_t(arr.nbytes)))
        return p.value
    def download(arr, p):
        ck(cu.cuMemcpyDtoH_v2(arr.ctypes.data_as(ctypes.c_void_p), ctypes.c_uint64(p), ctypes.c_size_t(arr.nbytes)))

    wl = synthetic.Workload("reset", 1, 4, 6, 8, 16, 128, 128, "bf16", "profiled")
    q, k, v = (t.view(__import__("torch").int16).numpy().copy() for t in synthetic.make_qkv(wl))
    shape = _lib.make_shape(wl.B, wl.H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block)
    params = _lib.make_params(1, 40, profile_frac=wl.profile_frac)

    def run():
        dq, dk, dv = upload(q), upload(k), upload(v)
        kinds = np.full(wl.H, 7, dtype=np.uint8)
        mse = np.full(2 * wl.H, -1.0, dtype=np.float32)
        err = np.zeros(1, dtype=np.int32)
        dkinds, dmse, derr = upload(kinds), upload(mse), upload(err)
        _lib.vsa_profile_heads_static(dq, dk, dv, shape, params, dkinds, dmse, derr, stream=0)
        assert _lib.vsa_get_device_error(derr, stream=0) == 0
        download(kinds, dkinds)
        download(mse, dmse)
        return kinds, mse

    ck(cu.cuInit(0))
    context()
    k1, m1 = run()
    _lib.vsa_selftest_device_reset()
    context()
    k2, m2 = run()
    assert np.array_equal(k1, k2), (k1, k2)
    assert np.array_equal(m1.view(np.uint32), m2.view(np.uint32)), (m1, m2)
    assert set(k1.tolist()) <= {0, 1} and (m1 >= 0).all()
    print("reset ok", k1.tolist())
""")


def test_static_scratch_after_context_reset():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, "-c", _RESET_CHILD, root], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-4000:]
    assert "reset ok" in res.stdout
