"""CPU checks of the C-ABI library: it loads, exports every declared entry point, and its
host-side planning helpers and argument validation behave as documented.  No kernel runs.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synthetic
from block_sparse_attention_31_b200 import _lib

FAKE = 0x10000  # 16-byte-aligned non-null address; never dereferenced (validation fails first)


def test_every_declared_symbol_is_exported():
    names = _lib.declared_symbols()
    assert len(names) >= 18
    for n in names:
        assert hasattr(_lib.lib, n), n
    assert _lib.lib.vsa_version() >= 100
    for s in range(7):
        assert _lib.status_string(s)


@pytest.mark.parametrize("wl", [synthetic.WAN, synthetic.HUNYUAN, synthetic.TINY,
                                synthetic.Workload("ragged", 1, 1, 7, 5, 9, 64, 64, "bf16", "profiled")])
@pytest.mark.parametrize("target", [1.0, 0.35, 0.18, 0.13, 0.05])
def test_pattern_window_matches_oracle(wl, target):
    shape = _lib.make_shape(wl.B, wl.H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block)
    for kind in (oracle.SPATIAL, oracle.TEMPORAL):
        w, kept = _lib.vsa_pattern_window(shape, kind, target)
        assert w == oracle.window_for_target(kind, wl.F, wl.Hl, wl.Wl, wl.block, target)
        assert kept == pytest.approx(oracle.kept_fraction(kind, wl.F, wl.Hl, wl.Wl, wl.block, w), abs=1e-15)


def test_wan_grid_window_table():
    # the smallest windows reaching each kept fraction of the sweep on the 21x30x52 grid (block 128)
    shape = _lib.make_shape(1, 12, 21, 30, 52, 128, 128)
    got = {t: (_lib.vsa_pattern_window(shape, 0, t)[0], _lib.vsa_pattern_window(shape, 1, t)[0])
           for t in (1.0, 0.35, 0.18, 0.13, 0.05)}
    assert got == {1.0: (20, 1548), 0.35: (4, 298), 0.18: (2, 140), 0.13: (1, 98), 0.05: (0, 31)}


@pytest.mark.parametrize("F,Hl,Wl,block,w_s,w_t", [(21, 30, 52, 128, 2, 140), (4, 8, 8, 64, 0, 0),
                                                   (7, 5, 9, 64, 1, 7), (33, 45, 80, 128, 3, 337)])
def test_max_kv_matches_oracle(F, Hl, Wl, block, w_s, w_t):
    shape = _lib.make_shape(1, 2, F, Hl, Wl, 128, block)
    got = _lib.vsa_max_kv(shape, _lib.make_params(w_s, w_t))
    ks = oracle.pattern_keep(oracle.SPATIAL, F, Hl, Wl, block, w_s).sum(axis=1).max()
    kt = oracle.pattern_keep(oracle.TEMPORAL, F, Hl, Wl, block, w_t).sum(axis=1).max()
    assert got == max(ks, kt)


def test_cube_shape_helpers():
    wl = synthetic.WAN_6X
    shape = _lib.make_shape(1, 12, wl.F, wl.Hl, wl.Wl, 128, 128, wl.cube)
    assert _lib.vsa_layout_rows(shape) == oracle.layout_rows(oracle.CUBE, wl.F, wl.Hl, wl.Wl, wl.cube) == 229376
    assert _lib.vsa_num_blocks(shape) == 1792
    assert _lib.vsa_max_kv(shape, _lib.make_params(0, 0, topk=32)) >= 33
    assert _lib.vsa_mask_workspace_size(shape, _lib.make_params(topk=32)) == 8 * (2 * 12 * 1792 * 128 + 12 * 1792 * 1792)


@pytest.mark.parametrize("N", [256, 32760, 118800, 7 * 5 * 9])
def test_profile_rows_matches_oracle(N):
    shape = _lib.make_shape(1, 1, 1, 1, N, 64, 64)
    assert _lib.vsa_profile_rows(shape, _lib.make_params(profile_frac=0.01)) == oracle.profile_rows(N, 0.01)


def _status(fn, *args):
    return fn(*args)


def test_shape_validation():
    p = _lib.make_params()
    out = ctypes.c_int64()
    lib = _lib.lib
    assert lib.vsa_layout_rows(ctypes.byref(_lib.make_shape(1, 1, 4, 8, 8, 96, 64)), ctypes.byref(out)) == \
        _lib.VSA_ERR_UNSUPPORTED
    assert lib.vsa_layout_rows(ctypes.byref(_lib.make_shape(1, 1, 4, 8, 8, 64, 32)), ctypes.byref(out)) == \
        _lib.VSA_ERR_UNSUPPORTED
    assert lib.vsa_layout_rows(ctypes.byref(_lib.make_shape(0, 1, 4, 8, 8, 64, 64)), ctypes.byref(out)) == \
        _lib.VSA_ERR_INVALID_ARG
    # cube volume must equal the block
    assert lib.vsa_layout_rows(ctypes.byref(_lib.make_shape(1, 1, 8, 8, 8, 64, 128, (4, 4, 2))),
                               ctypes.byref(out)) == _lib.VSA_ERR_UNSUPPORTED
    assert lib.vsa_layout_rows(None, ctypes.byref(out)) == _lib.VSA_ERR_INVALID_ARG
    w = ctypes.c_int()
    assert lib.vsa_pattern_window(ctypes.byref(_lib.make_shape(1, 1, 4, 8, 8, 64, 64)), 2, 0.5, ctypes.byref(w),
                                  None) == _lib.VSA_ERR_INVALID_ARG
    assert lib.vsa_pattern_window(ctypes.byref(_lib.make_shape(1, 1, 4, 8, 8, 64, 64)), 0, 1.5, ctypes.byref(w),
                                  None) == _lib.VSA_ERR_INVALID_ARG
    assert p.profile_frac == 0.01


def test_kernel_entry_points_validate_before_launch():
    lib = _lib.lib
    shape = _lib.make_shape(1, 2, 4, 8, 8, 64, 64)
    params = _lib.make_params(0, 0)
    s = ctypes.c_void_p(0)
    # null / misaligned pointers
    assert lib.vsa_permute(None, 1, FAKE, FAKE, ctypes.byref(shape), FAKE, s) == _lib.VSA_ERR_INVALID_ARG
    assert lib.vsa_permute(FAKE + 2, 1, FAKE, FAKE, ctypes.byref(shape), FAKE, s) == _lib.VSA_ERR_INVALID_ARG
    assert lib.vsa_permute(FAKE, 7, FAKE, FAKE, ctypes.byref(shape), FAKE, s) == _lib.VSA_ERR_INVALID_ARG
    assert lib.vsa_unpermute(FAKE, FAKE, FAKE, 1, None, FAKE, ctypes.byref(shape), FAKE, s) == \
        _lib.VSA_ERR_INVALID_ARG
    # workspace too small
    assert lib.vsa_profile_heads(FAKE, FAKE, FAKE, ctypes.byref(shape), ctypes.byref(params), FAKE, FAKE, FAKE, 16,
                                 FAKE, s) == _lib.VSA_ERR_WORKSPACE
    bad = _lib.make_params(0, 0, profile_frac=0.0)
    assert lib.vsa_profile_heads(FAKE, FAKE, FAKE, ctypes.byref(shape), ctypes.byref(bad), FAKE, FAKE, FAKE, 1 << 30,
                                 FAKE, s) == _lib.VSA_ERR_INVALID_ARG
    assert lib.vsa_build_mask(FAKE, None, None, ctypes.byref(shape), ctypes.byref(params), FAKE, FAKE, FAKE, 0,
                              None, 0, FAKE, s) == _lib.VSA_ERR_INVALID_ARG
    io = _lib.QKVO(FAKE, FAKE, None, FAKE, None)
    assert lib.vsa_sparse_attn_fwd(ctypes.byref(io), None, FAKE, FAKE, FAKE, 4, None, ctypes.byref(shape), 0.0,
                                   FAKE, s) == _lib.VSA_ERR_INVALID_ARG
    assert lib.vsa_block_order(FAKE, FAKE, FAKE, 4, ctypes.byref(shape), None, s) == _lib.VSA_ERR_INVALID_ARG
    assert lib.vsa_block_order(FAKE, FAKE, FAKE, 0, ctypes.byref(shape), FAKE, s) == _lib.VSA_ERR_INVALID_ARG
    io = _lib.QKVO(FAKE, FAKE, FAKE, FAKE, None)
    assert lib.vsa_attention(ctypes.byref(io), 1, ctypes.byref(shape), ctypes.byref(params), 0, FAKE, None, FAKE, 8,
                             FAKE, s) == _lib.VSA_ERR_WORKSPACE
    # profiling needs bf16 input; cube selection needs cube dims
    assert lib.vsa_attention(ctypes.byref(io), 0, ctypes.byref(shape), ctypes.byref(params), 0, FAKE, None, FAKE,
                             1 << 40, FAKE, s) == _lib.VSA_ERR_UNSUPPORTED
    assert lib.vsa_attention(ctypes.byref(io), 1, ctypes.byref(shape), ctypes.byref(params), 2, FAKE, None, FAKE,
                             1 << 40, FAKE, s) == _lib.VSA_ERR_INVALID_ARG
    assert lib.vsa_get_device_error(None, s, None) == _lib.VSA_ERR_INVALID_ARG
    # in-kernel layout: cube shapes are refused on the host, missing buffers too
    cube_shape = _lib.make_shape(1, 2, 8, 8, 8, 64, 128, (4, 4, 8))
    io = _lib.QKVO(FAKE, FAKE, FAKE, FAKE, None)
    assert lib.vsa_sparse_attn_fwd_natural(ctypes.byref(io), FAKE, FAKE, FAKE, 4, None, ctypes.byref(cube_shape), 0.0,
                                           FAKE, s) == _lib.VSA_ERR_UNSUPPORTED
    io = _lib.QKVO(FAKE, None, FAKE, FAKE, None)
    assert lib.vsa_sparse_attn_fwd_natural(ctypes.byref(io), FAKE, FAKE, FAKE, 4, None, ctypes.byref(shape), 0.0,
                                           FAKE, s) == _lib.VSA_ERR_INVALID_ARG
    assert lib.vsa_selftest_wait_timeout(None, FAKE, s) == _lib.VSA_ERR_INVALID_ARG


def test_in_kernel_layout_drops_the_permuted_copies():
    shape = _lib.make_shape(1, 12, 21, 30, 52, 128, 128)
    copies = _lib.vsa_attention_workspace_size(shape, _lib.make_params(2, 140), 1, 0)
    fused = _lib.vsa_attention_workspace_size(shape, _lib.make_params(2, 140, layout_in_kernel=True), 1, 0)
    per_tensor = 12 * 32760 * 128 * 2
    assert copies - fused >= 4 * per_tensor          # Q, K, V, O copies
    # fp32 inputs and cube shapes keep the copies
    f32_fused = _lib.vsa_attention_workspace_size(shape, _lib.make_params(2, 140, layout_in_kernel=True), 0, 1)
    assert f32_fused > 0 and f32_fused == _lib.vsa_attention_workspace_size(shape, _lib.make_params(2, 140), 0, 1)


def test_workspace_sizes_monotone():
    shape = _lib.make_shape(1, 12, 21, 30, 52, 128, 128)
    p = _lib.make_params(2, 140)
    a = _lib.vsa_attention_workspace_size(shape, p, 1, 0)
    b = _lib.vsa_attention_workspace_size(shape, p, 1, 1)
    assert a > b > 4 * 12 * 32760 * 128 * 2
    assert _lib.vsa_profile_workspace_size(shape, p) > 12 * 384 * 128 * 2
    ob, oi, oc, mk = _lib.vsa_attention_workspace_layout(shape, p, 1, 1)
    assert ob == 0 and oi > ob and oc > oi and mk == _lib.vsa_max_kv(shape, p)
    assert np.all(np.array([ob, oi, oc]) % 256 == 0)


def test_semantic_entry_points_validate_before_launch():
    """Semantic-permutation entry points: bad counts, budgets, shapes, workspaces and
    pointer pairs are refused on the host, and the workspace sizes follow the documented
    layout."""
    lib = _lib.lib
    s = ctypes.c_void_p(0)
    shape = _lib.make_shape(1, 2, 4, 8, 8, 64, 64)          # N = 256
    cube = _lib.make_shape(1, 2, 8, 8, 8, 64, 128, (4, 4, 8))
    # offsets and chunk offsets B*H*(C+1) int32, norms B*H*C fp32, two bf16 halves B*H*C*d,
    # the update's chunk sums B*H*M*d (fp64 twice, int32 once), M = ceil(N/128) + C, the sort's
    # segment histograms B*H*8*C int32, one flag per head and the chunk -> cluster map B*H*M
    # int32; each piece 256-aligned
    m16, m64 = 2 + 16, 2 + 64
    assert _lib.vsa_kmeans_workspace_size(shape, 16) == (2 * 256 + 256 + 2 * 4096 + 2 * (2 * m16 * 64 * 8)
                                                        + 2 * m16 * 64 * 4 + 1024 + 256 + 256)
    assert _lib.vsa_kmeans_workspace_size(shape, 64) == (2 * 768 + 512 + 2 * 16384 + 2 * (2 * m64 * 64 * 8)
                                                        + 2 * m64 * 64 * 4 + 4096 + 256 + 768)
    assert _lib.vsa_kmeans_workspace_size(shape, 0) == 0
    assert _lib.vsa_kmeans_workspace_size(shape, 257) == 0   # more clusters than rows
    assert _lib.vsa_kmeans_workspace_size(cube, 16) == 0
    km = lambda sh, C, it, wsb: lib.vsa_kmeans(FAKE, ctypes.byref(sh), C, it, FAKE, FAKE, FAKE, FAKE, FAKE, wsb,  # noqa
                                               FAKE, s)
    assert km(shape, 0, 1, 1 << 20) == _lib.VSA_ERR_INVALID_ARG
    assert km(shape, 1025, 1, 1 << 20) == _lib.VSA_ERR_INVALID_ARG
    assert km(shape, 16, 0, 1 << 20) == _lib.VSA_ERR_INVALID_ARG
    assert km(shape, 16, 3, 8) == _lib.VSA_ERR_WORKSPACE
    assert km(cube, 16, 3, 1 << 20) == _lib.VSA_ERR_UNSUPPORTED
    assert lib.vsa_kmeans(FAKE + 8, ctypes.byref(shape), 16, 3, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, FAKE,
                          s) == _lib.VSA_ERR_INVALID_ARG       # misaligned rows

    def mask(top_p, scale=0.0, cq=16, ck=16, wsb=1 << 20, max_kv=4):
        return lib.vsa_semantic_mask(FAKE, FAKE, FAKE, FAKE, cq, FAKE, FAKE, FAKE, FAKE, ck, ctypes.byref(shape),
                                     top_p, scale, FAKE, FAKE, FAKE, FAKE, max_kv, FAKE, wsb, FAKE, s)
    assert mask(0.0) == _lib.VSA_ERR_INVALID_ARG
    assert mask(1.5) == _lib.VSA_ERR_INVALID_ARG
    assert mask(0.5, scale=-1.0) == _lib.VSA_ERR_INVALID_ARG
    assert mask(0.5, ck=2000) == _lib.VSA_ERR_INVALID_ARG
    assert mask(0.5, max_kv=0) == _lib.VSA_ERR_INVALID_ARG
    assert mask(0.5, wsb=8) == _lib.VSA_ERR_WORKSPACE
    assert _lib.vsa_semantic_mask_workspace_size(shape) == 256   # 2 * B*H * nblk int2, 256-aligned
    assert lib.vsa_scatter_rows(FAKE, FAKE, FAKE, FAKE, None, ctypes.byref(shape), FAKE, s) == \
        _lib.VSA_ERR_INVALID_ARG                                    # LSE needs both buffers
    assert lib.vsa_gather_rows(FAKE, FAKE, FAKE, ctypes.byref(cube), FAKE, s) == _lib.VSA_ERR_UNSUPPORTED
    good = _lib.make_sem_params(16, 16, 3, 0.5)
    assert _lib.vsa_semantic_workspace_size(shape, good) > 0
    for bad in (_lib.make_sem_params(0, 16, 3, 0.5), _lib.make_sem_params(16, 16, 0, 0.5),
                _lib.make_sem_params(16, 16, 3, 0.0), _lib.make_sem_params(16, 16, 3, 0.5, -1.0)):
        assert _lib.vsa_semantic_workspace_size(shape, bad) == 0
    io = _lib.QKVO(FAKE, FAKE, FAKE, FAKE, None)
    assert lib.vsa_semantic_attention(ctypes.byref(io), ctypes.byref(shape), ctypes.byref(good), FAKE, 8, FAKE,
                                      s) == _lib.VSA_ERR_WORKSPACE
