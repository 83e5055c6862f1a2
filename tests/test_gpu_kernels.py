"""GPU parity of each kernel against the fp64 oracle, through the C ABI.

Permutations, masks and head choices must match bit for bit; attention outputs within
max-abs 2e-2 and relative L2 1e-2 (bf16 inputs, fp32 accumulation).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic
import validity
from parity_util import assert_close_attention, cuda_err, head_slots, keep_for_head, mse_close, to_f64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_31_b200 as vsa
    from block_sparse_attention_31_b200 import _lib
else:  # collected on CPU only to be skipped
    vsa = _lib = None

S_, T_, C_ = oracle.SPATIAL, oracle.TEMPORAL, oracle.CUBE


def _wl(F, Hl, Wl, d, block, H=3, cube=(4, 4, 8), topk=0):
    return synthetic.Workload(f"t{F}x{Hl}x{Wl}", 1, H, F, Hl, Wl, d, block, "bf16", "given", cube=cube, topk=topk)


def _shape(wl, cubes):
    return _lib.make_shape(wl.B, wl.H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block, wl.cube if cubes else None)


# ------------------------------------------------------------------------------------
# permutation
# ------------------------------------------------------------------------------------

@pytest.mark.parametrize("F,Hl,Wl,d,block,cubes,src", [
    (4, 8, 8, 64, 64, False, "f32"),          # tiny grid, fp32 -> bf16 conversion
    (5, 6, 10, 128, 128, False, "bf16"),      # ragged: N = 300
    (5, 5, 9, 128, 128, True, "bf16"),        # partial cubes
    (21, 30, 52, 128, 128, False, "bf16"),    # Wan2.1-1.3B grid
    (9, 7, 17, 64, 128, True, "f32"),
])
def test_permute_unpermute_bit_exact(F, Hl, Wl, d, block, cubes, src):
    wl = _wl(F, Hl, Wl, d, block)
    kinds_list = [S_, T_, C_] if cubes else [S_, T_, T_]
    shape = _shape(wl, cubes)
    R = _lib.vsa_layout_rows(shape)
    dt = torch.float32 if src == "f32" else torch.bfloat16
    x = synthetic.make_random((1, 3, wl.N, d), dt, seed=11)
    xd = x.cuda()
    kinds = torch.tensor(kinds_list, dtype=torch.uint8, device="cuda")
    err = cuda_err()
    sentinel = torch.full((1, 3, R, d), 7.0, dtype=torch.bfloat16, device="cuda")
    _lib.vsa_permute(xd, _lib.VSA_F32 if src == "f32" else _lib.VSA_BF16, sentinel, kinds, shape, err)
    assert _lib.vsa_get_device_error(err) == 0
    got = sentinel.cpu()
    xb = x.to(torch.bfloat16)  # torch's round-to-nearest-even conversion
    for h, kind in enumerate(kinds_list):
        if kind == S_ and src == "bf16":
            assert (got[0, h] == 7.0).all()          # spatial heads untouched
            continue
        slots = head_slots(kind, wl)
        want = torch.zeros(R, d, dtype=torch.bfloat16)
        want[torch.from_numpy(slots)] = xb[0, h]
        assert torch.equal(got[0, h].view(torch.int16), want.view(torch.int16)), (h, kind)
    # unpermute back (bf16 destination leaves spatial heads alone; fp32 converts all)
    lse_src = torch.arange(3 * R, dtype=torch.float32, device="cuda").view(1, 3, R)
    out_dt = torch.float32 if src == "f32" else torch.bfloat16
    back = torch.full((1, 3, wl.N, d), -3.0, dtype=out_dt, device="cuda")
    lse = torch.full((1, 3, wl.N), -5.0, dtype=torch.float32, device="cuda")
    _lib.vsa_unpermute(sentinel, lse_src, back, _lib.VSA_F32 if src == "f32" else _lib.VSA_BF16, lse, kinds, shape,
                       err)
    assert _lib.vsa_get_device_error(err) == 0
    back, lse = back.cpu(), lse.cpu()
    for h, kind in enumerate(kinds_list):
        if kind == S_ and src == "bf16":
            assert (back[0, h] == -3.0).all()
            continue
        assert torch.equal(back[0, h].to(torch.bfloat16).view(torch.int16), xb[0, h].view(torch.int16))
        slots = torch.from_numpy(head_slots(kind, wl))
        assert torch.equal(lse[0, h], (h * R + slots).to(torch.float32))


# ------------------------------------------------------------------------------------
# masks
# ------------------------------------------------------------------------------------

def _run_masks(wl, kinds_list, w_s, w_t, cubes, q=None, k=None):
    shape = _shape(wl, cubes)
    params = _lib.make_params(w_s, w_t, topk=wl.topk)
    nblk = _lib.vsa_num_blocks(shape)
    max_kv = _lib.vsa_max_kv(shape, params)
    H = len(kinds_list)
    nw = (nblk + 31) // 32
    bits = torch.full((1, H, nblk, nw), -7, dtype=torch.int32, device="cuda")
    idx = torch.full((1, H, nblk, max_kv), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((1, H, nblk), -7, dtype=torch.int32, device="cuda")
    kinds = torch.tensor(kinds_list, dtype=torch.uint8, device="cuda")
    err = cuda_err()
    qc = kc = None
    ws_bytes = _lib.vsa_mask_workspace_size(shape, params)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device="cuda")
    if cubes:
        R = _lib.vsa_layout_rows(shape)
        qc = torch.empty(1, H, R, wl.d, dtype=torch.bfloat16, device="cuda")
        kc = torch.empty_like(qc)
        _lib.vsa_permute(q.cuda(), _lib.VSA_BF16, qc, kinds, shape, err)
        _lib.vsa_permute(k.cuda(), _lib.VSA_BF16, kc, kinds, shape, err)
    _lib.vsa_build_mask(kinds, qc, kc, shape, params, bits, idx, cnt, max_kv, ws, ws_bytes, err)
    assert _lib.vsa_get_device_error(err) == 0
    return bits.cpu(), idx.cpu(), cnt.cpu(), max_kv, nblk


@pytest.mark.parametrize("F,Hl,Wl,block,w_s,w_t", [
    (4, 8, 8, 64, 0, 0), (21, 30, 52, 128, 2, 140), (33, 45, 80, 128, 3, 337), (7, 5, 9, 64, 1, 11),
    (21, 30, 52, 128, 20, 1548), (21, 30, 52, 128, 0, 31)])
def test_pattern_masks_bit_exact(F, Hl, Wl, block, w_s, w_t):
    wl = _wl(F, Hl, Wl, 128, block, H=2)
    bits, idx, cnt, max_kv, nblk = _run_masks(wl, [S_, T_], w_s, w_t, cubes=False)
    for h, kind in enumerate([S_, T_]):
        keep = keep_for_head(kind, wl, w_s, w_t)
        want_idx, want_cnt = oracle.keep_to_lists(keep, max_kv)
        assert np.array_equal(cnt[0, h].numpy(), want_cnt)
        assert np.array_equal(idx[0, h].numpy(), want_idx)
        assert np.array_equal(bits[0, h].numpy().view(np.uint32), oracle.keep_to_bits(keep))


def _bits_to_keep(words, n):
    w = np.asarray(words).view(np.uint32)
    b = (w[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1
    return b.reshape(w.shape[0], -1)[:, :n].astype(bool)


@pytest.mark.parametrize("F,Hl,Wl,topk", [(5, 5, 9, 3), (9, 9, 17, 4), (126, 30, 52, 32)])
def test_cube_masks_match_oracle(F, Hl, Wl, topk):
    """Each row keeps its own cube and the top-k cubes of the oracle's fp64 coarse scores
    (equal to the oracle's set, or a logged near-tie at the k-th score); the bitset, lists
    and counts are three exact encodings of that set."""
    wl = _wl(F, Hl, Wl, 128, 128, H=2, topk=topk)
    wl = wl.with_(H=2)
    q, k, _ = synthetic.make_qkv(wl.with_(dtype="bf16"))
    bits, idx, cnt, max_kv, nblk = _run_masks(wl, [C_, C_], 0, 0, cubes=True, q=q, k=k)
    for h in range(2):
        want, score = oracle.cube_topk_keep(q[0, h], k[0, h], F, Hl, Wl, topk, wl.cube, return_scores=True)
        got = _bits_to_keep(bits[0, h].numpy(), want.shape[0])
        validity.topk_rows_valid(got, want, score, topk, f"cubes {F}x{Hl}x{Wl} head {h}")
        got_idx, got_cnt = oracle.keep_to_lists(got, max_kv)
        assert np.array_equal(cnt[0, h].numpy(), got_cnt)
        assert np.array_equal(idx[0, h].numpy(), got_idx)


@pytest.mark.parametrize("F,Hl,Wl,topk,ties", [
    (8, 16, 32, 8, True),      # 32 cubes, every score of a row equal: candidates = whole row
    (64, 32, 64, 32, True),    # 1024 cubes, all equal: more candidates than the gather holds
    (16, 16, 32, 40, False),   # topk above 32: full scan every round
])
def test_cube_topk_paths_bit_exact(F, Hl, Wl, topk, ties):
    """The candidate filter, its overflow fallback and the full-scan path pick the same
    cubes as the oracle, including the smaller-index rule on ties."""
    wl = _wl(F, Hl, Wl, 128, 128, H=2, topk=topk)
    q, k, _ = synthetic.make_qkv(wl)
    if ties:  # K constant: within a row every coarse score is the same number
        k = torch.ones_like(k)
    bits, idx, cnt, max_kv, nblk = _run_masks(wl, [C_, C_], 0, 0, cubes=True, q=q, k=k)
    for h in range(2):
        keep = oracle.cube_topk_keep(q[0, h], k[0, h], F, Hl, Wl, topk, wl.cube)
        want_idx, want_cnt = oracle.keep_to_lists(keep, max_kv)
        assert np.array_equal(cnt[0, h].numpy(), want_cnt)
        assert np.array_equal(idx[0, h].numpy(), want_idx)
        if ties:
            C = keep.shape[0]
            assert keep[C - 1, :topk].all()      # the smallest indices win the ties


def test_mask_overflow_flag():
    wl = _wl(21, 30, 52, 128, 128, H=1)
    shape = _shape(wl, False)
    params = _lib.make_params(2, 140)
    nblk = _lib.vsa_num_blocks(shape)
    small = 8
    bits = torch.zeros(1, 1, nblk, (nblk + 31) // 32, dtype=torch.int32, device="cuda")
    idx = torch.zeros(1, 1, nblk, small, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, 1, nblk, dtype=torch.int32, device="cuda")
    kinds = torch.zeros(1, dtype=torch.uint8, device="cuda")
    err = cuda_err()
    _lib.vsa_build_mask(kinds, None, None, shape, params, bits, idx, cnt, small, None, 0, err)
    assert _lib.vsa_get_device_error(err) & _lib.VSA_DEVERR_OVERFLOW


# ------------------------------------------------------------------------------------
# sparse attention kernel (masks from the oracle, so the kernel is tested on its own)
# ------------------------------------------------------------------------------------

def _check_block_order(order, kinds_list, wl, idx, cnt, nblk):
    """The work order is, per head, the head's blocks sorted by (first kept block, index)."""
    for h, kind in enumerate(kinds_list):
        nb = -(-oracle.layout_rows(kind, wl.F, wl.Hl, wl.Wl, wl.cube) // wl.block)
        first = [int(idx[0, h, i, 0]) if cnt[0, h, i] > 0 else 1 << 20 for i in range(nb)]
        want = sorted(range(nb), key=lambda i: (first[i], i)) + list(range(nb, nblk))
        assert order[h].tolist() == want, f"head {h}"


def _attention_case(wl, kinds_list, keeps, q, k, v, perm, rows=None, lse_check=True, ordered=False):
    H = len(kinds_list)
    shape = _lib.make_shape(1, H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block, wl.cube if C_ in kinds_list else None)
    nblk = _lib.vsa_num_blocks(shape)
    R = _lib.vsa_layout_rows(shape)
    max_kv = max(int(kp.sum(axis=1).max()) for kp in keeps) if keeps else 1
    max_kv = max(max_kv, 1)
    idx = np.full((1, H, nblk, max_kv), -1, dtype=np.int32)
    cnt = np.zeros((1, H, nblk), dtype=np.int32)
    for h, kp in enumerate(keeps):
        i_, c_ = oracle.keep_to_lists(kp, max_kv)
        idx[0, h, :kp.shape[0]] = i_
        cnt[0, h, :kp.shape[0]] = c_
    kinds = torch.tensor(kinds_list, dtype=torch.uint8, device="cuda")
    err = cuda_err()
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.full_like(qd, 9.0)
    lse = torch.full((1, H, wl.N), 9.0, dtype=torch.float32, device="cuda")
    if perm:
        qp = torch.empty(1, H, R, wl.d, dtype=torch.bfloat16, device="cuda")
        kp_, vp, op = torch.empty_like(qp), torch.empty_like(qp), torch.empty_like(qp)
        lsep = torch.empty(1, H, R, dtype=torch.float32, device="cuda")
        for src, dst in ((qd, qp), (kd, kp_), (vd, vp)):
            _lib.vsa_permute(src, _lib.VSA_BF16, dst, kinds, shape, err)
        idx_d, cnt_d = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
        order = None
        if ordered:
            order = torch.full((H, nblk), -5, dtype=torch.int32, device="cuda")
            _lib.vsa_block_order(kinds, idx_d, cnt_d, max_kv, shape, order)
            _check_block_order(order.cpu(), kinds_list, wl, idx, cnt, nblk)
            # pairing changes no result: natural pairing gives the same bits
            op_nat, lsep_nat = torch.empty_like(op), torch.empty_like(lsep)
            _lib.vsa_sparse_attn_fwd(_lib.qkvo(qd, kd, vd, o, lse), _lib.qkvo(qp, kp_, vp, op_nat, lsep_nat), kinds,
                                     idx_d, cnt_d, max_kv, shape, 0.0, err)
        _lib.vsa_sparse_attn_fwd(_lib.qkvo(qd, kd, vd, o, lse), _lib.qkvo(qp, kp_, vp, op, lsep), kinds,
                                 idx_d, cnt_d, max_kv, shape, 0.0, err, order=order)
        if ordered:
            for h, kind in enumerate(kinds_list):
                if kind != S_:  # rows past a head's own layout are never written
                    r = oracle.layout_rows(kind, wl.F, wl.Hl, wl.Wl, wl.cube)
                    assert torch.equal(op[0, h, :r], op_nat[0, h, :r]), f"head {h}"
                    assert torch.equal(lsep[0, h, :r], lsep_nat[0, h, :r]), f"head {h}"
        _lib.vsa_unpermute(op, lsep, o, _lib.VSA_BF16, lse, kinds, shape, err)
    else:
        _lib.vsa_sparse_attn_fwd(_lib.qkvo(qd, kd, vd, o, lse), None, kinds, torch.from_numpy(idx).cuda(),
                                 torch.from_numpy(cnt).cuda(), max_kv, shape, 0.0, err)
    assert _lib.vsa_get_device_error(err) == 0
    o, lse = o.cpu(), lse.cpu()
    for h, kind in enumerate(kinds_list):
        rr = np.arange(wl.N) if rows is None else rows
        want, want_lse = oracle.attention_rows(q[0, h], k[0, h], v[0, h], head_slots(kind, wl), wl.block, keeps[h],
                                               rows=rr, scale=1.0 / math.sqrt(wl.d))
        assert_close_attention(to_f64(o[0, h])[rr], want, f"head {h} kind {kind}")
        if lse_check:
            g = to_f64(lse[0, h])[rr]
            fin = np.isfinite(want_lse)
            assert np.array_equal(np.isfinite(g), fin)
            assert np.abs(g[fin] - want_lse[fin]).max() < 2e-2


@pytest.mark.parametrize("d,block", [(128, 128), (64, 64), (64, 128), (128, 64)])
def test_attention_random_masks(d, block):
    """Random block masks (diagonal kept) on a ragged grid spanning several tiles."""
    wl = _wl(5, 6, 10, d, block, H=2)       # N = 300: ragged last block
    q, k, v = (synthetic.make_random((1, 2, wl.N, d), torch.bfloat16, seed=s) for s in (1, 2, 3))
    nb = -(-wl.N // block)
    rng = np.random.default_rng(5)
    keeps = []
    for _ in range(2):
        kp = rng.random((nb, nb)) < 0.5
        np.fill_diagonal(kp, True)
        keeps.append(kp)
    _attention_case(wl, [S_, S_], keeps, q, k, v, perm=False)


@pytest.mark.parametrize("d,block", [(128, 128), (64, 64)])
def test_attention_structured_perm_path(d, block):
    """Spatial head from natural buffers, temporal head through the frame-major buffers."""
    wl = synthetic.Workload("s", 1, 2, 6, 8, 16, d, block, "bf16", "given")
    q, k, v = synthetic.make_qkv(wl)
    keeps = [keep_for_head(S_, wl, 1, 0), keep_for_head(T_, wl, 0, 9)]
    _attention_case(wl, [S_, T_], keeps, q, k, v, perm=True)


def test_attention_empty_rows_and_dense():
    wl = _wl(4, 8, 8, 128, 64, H=2)        # 4 blocks of 64
    q, k, v = (synthetic.make_random((1, 2, wl.N, 128), torch.bfloat16, seed=s) for s in (4, 5, 6))
    empty = np.zeros((4, 4), dtype=bool)
    empty[1, :] = True                      # only q block 1 keeps anything
    dense = np.ones((4, 4), dtype=bool)
    _attention_case(wl, [S_, S_], [empty, dense], q, k, v, perm=False)


def test_attention_cube_padding():
    wl = _wl(5, 5, 9, 128, 128, H=1, topk=3)
    q, k, v = synthetic.make_qkv(wl.with_(H=1))
    C = oracle.num_cubes(5, 5, 9)
    rng = np.random.default_rng(3)
    kp = rng.random((C, C)) < 0.6
    np.fill_diagonal(kp, True)
    _attention_case(wl.with_(H=1), [C_], [kp], q, k, v, perm=True)


@pytest.mark.parametrize("F,Hl,Wl", [(9, 9, 17), (12, 16, 16)])
def test_attention_block_order(F, Hl, Wl):
    """Cube and pattern heads run in the locality order of vsa_block_order: the order is the
    documented sort, results equal natural pairing bit for bit and match the oracle."""
    wl = _wl(F, Hl, Wl, 128, 128, H=3, topk=4)
    q, k, v = synthetic.make_qkv(wl)
    C = oracle.num_cubes(F, Hl, Wl)
    rng = np.random.default_rng(F)
    kc = rng.random((C, C)) < 0.15
    kc[rng.random(C) < 0.1] = False           # a few query cubes with nothing kept
    keeps = [kc, keep_for_head(S_, wl, 1, 0), keep_for_head(T_, wl, 0, 20)]
    _attention_case(wl, [C_, S_, T_], keeps, q, k, v, perm=True, ordered=True)


@pytest.mark.parametrize("q_scale", [0.0, 1.0, 8.0])
def test_attention_weights_within_bf16_rounding(q_scale):
    """With V rows = 64 * unit vectors, O[i, j] = 64 * P[i, j] / l: the kernel's softmax weights
    seen directly.  Their error is bf16 rounding of P (half an ulp, 2^-8 relative) plus the
    bf16 rounding of the output (another 2^-8); Q = 0 gives equal weights, exactly."""
    d = N = 128
    shape = _lib.make_shape(1, 1, 1, 1, N, d, 128)
    g = torch.Generator().manual_seed(1)
    q = (torch.randn(1, 1, N, d, generator=g) * q_scale).to(torch.bfloat16)
    k = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    v = (torch.eye(N, d) * 64).reshape(1, 1, N, d).to(torch.bfloat16)
    o = torch.empty(1, 1, N, d, dtype=torch.bfloat16, device="cuda")
    kinds = torch.zeros(1, dtype=torch.uint8, device="cuda")
    idx = torch.zeros(1, 1, 1, 1, dtype=torch.int32, device="cuda")
    cnt = torch.ones(1, 1, 1, dtype=torch.int32, device="cuda")
    err = cuda_err()
    _lib.vsa_sparse_attn_fwd(_lib.qkvo(q.cuda(), k.cuda(), v.cuda(), o), None, kinds, idx, cnt, 1, shape, 0.0, err)
    assert _lib.vsa_get_device_error(err) == 0
    s = (q[0, 0].double() @ k[0, 0].double().T) / math.sqrt(d)
    want = torch.softmax(s, dim=1) * 64
    got = o[0, 0].cpu().double()
    if q_scale == 0.0:
        assert torch.equal(got, torch.full_like(got, 0.5))
        return
    big = want > 1e-3
    rel = ((got - want).abs() / want)[big]
    assert rel.max() <= 2.0 ** -7 * 1.01, rel.max()


def test_attention_large_scores_stable():
    """Inputs scaled x8: logits up to a few hundred must not overflow the online softmax."""
    wl = _wl(3, 8, 16, 128, 128, H=1)
    q, k, v = (synthetic.make_random((1, 1, wl.N, 128), torch.bfloat16, seed=s, scale=sc)
               for s, sc in ((7, 8.0), (8, 8.0), (9, 1.0)))
    nb = -(-wl.N // 128)
    _attention_case(wl.with_(H=1), [S_], [np.ones((nb, nb), dtype=bool)], q, k, v, perm=False)


def test_attention_bad_lists_flag_error():
    wl = _wl(4, 8, 8, 64, 64, H=1)
    shape = _lib.make_shape(1, 1, 4, 8, 8, 64, 64)
    q = synthetic.make_random((1, 1, wl.N, 64), torch.bfloat16, seed=1).cuda()
    o = torch.empty_like(q)
    kinds = torch.zeros(1, dtype=torch.uint8, device="cuda")
    idx = torch.tensor([[[[0, 1], [1, 9], [2, -1], [3, -1]]]], dtype=torch.int32, device="cuda")  # 9 out of range
    cnt = torch.tensor([[[2, 2, 1, 3]]], dtype=torch.int32, device="cuda")                        # 3 > max_kv
    err = cuda_err()
    _lib.vsa_sparse_attn_fwd(_lib.qkvo(q, q, q, o), None, kinds, idx, cnt, 2, shape, 0.0, err)
    e = _lib.vsa_get_device_error(err)
    assert e & _lib.VSA_DEVERR_KV_RANGE
    o = o.cpu().float()
    assert (o[0, 0, 64:128] == 0).all() and (o[0, 0, 192:256] == 0).all()   # rejected rows are zero
    assert torch.isfinite(o).all()
    # a host address anywhere is refused before any launch
    o_host = torch.empty(1, 1, wl.N, 64, dtype=torch.bfloat16)
    with pytest.raises(_lib.VsaError) as ex:
        _lib.vsa_sparse_attn_fwd(_lib.qkvo(q, q, q, o_host), None, kinds, idx, cnt, 2, shape, 0.0, err)
    assert ex.value.status == _lib.VSA_ERR_INVALID_ARG
    # a work order that is not a permutation of the head's blocks
    o = torch.empty_like(q)
    good = torch.tensor([[[[0, -1], [1, -1], [2, -1], [3, -1]]]], dtype=torch.int32, device="cuda")
    ones = torch.ones(1, 1, 4, dtype=torch.int32, device="cuda")
    for bad in ([0, 0, 1, 2], [0, 1, 2, 7], [-1, 1, 2, 3]):
        err.zero_()
        order = torch.tensor(bad, dtype=torch.int32, device="cuda")
        _lib.vsa_sparse_attn_fwd(_lib.qkvo(q, q, q, o), None, kinds, good, ones, 2, shape, 0.0, err, order=order)
        assert _lib.vsa_get_device_error(err) & _lib.VSA_DEVERR_KV_RANGE, bad
    # a bad kind byte: the head's natural-order output rows are zero and its LSE is -inf
    err.zero_()
    kinds.fill_(9)
    o = torch.full_like(q, 5.0)
    lse = torch.full((1, 1, wl.N), 5.0, dtype=torch.float32, device="cuda")
    _lib.vsa_sparse_attn_fwd(_lib.qkvo(q, q, q, o, lse), None, kinds, idx, cnt, 2, shape, 0.0, err)
    assert _lib.vsa_get_device_error(err) & _lib.VSA_DEVERR_KIND
    assert (o == 0).all()
    assert torch.isneginf(lse).all()


# ------------------------------------------------------------------------------------
# profiling
# ------------------------------------------------------------------------------------

def _profile_gpu(q, k, v, wl, w_s, w_t, frac, static=False):
    shape = _lib.make_shape(wl.B, wl.H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block)
    params = _lib.make_params(w_s, w_t, profile_frac=frac)
    kinds = torch.full((wl.H,), 7, dtype=torch.uint8, device="cuda")
    mse = torch.zeros(wl.H * 2, dtype=torch.float32, device="cuda")
    err = cuda_err()
    if static:
        _lib.vsa_profile_heads_static(q.cuda(), k.cuda(), v.cuda(), shape, params, kinds, mse, err)
    else:
        ws_bytes = _lib.vsa_profile_workspace_size(shape, params)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        _lib.vsa_profile_heads(q.cuda(), k.cuda(), v.cuda(), shape, params, kinds, mse, ws, ws_bytes, err)
    assert _lib.vsa_get_device_error(err) == 0
    return kinds.cpu().numpy(), mse.cpu().numpy().reshape(-1, 2)


def _check_profile(q, k, v, wl, w_s, w_t, frac, kinds, mse, planted=True):
    """Kinds equal the oracle's (or a logged near-tie); both MSEs within the profiling
    tolerance of parity_util.mse_close."""
    for h in range(wl.H):
        kind, want, rows = oracle.profile_head(q[0, h], k[0, h], v[0, h], wl.F, wl.Hl, wl.Wl, wl.block, w_s, w_t,
                                               frac)
        validity.kind_valid(int(kinds[h]), kind, want, f"{wl.name} head {h}")
        if planted:
            assert kind == (S_ if h % 2 == 0 else T_)     # the planted structure
        nb = -(-wl.N // wl.block)
        dense, _ = oracle.attention_rows(q[0, h], k[0, h], v[0, h], np.arange(wl.N), wl.block,
                                         np.ones((nb, nb), dtype=bool), rows=rows, scale=1.0 / math.sqrt(wl.d))
        for j in range(2):
            mse_close(float(mse[h, j]), float(want[j]), dense, f"{wl.name} head {h} variant {j}")


@pytest.mark.parametrize("wl,w_s,w_t,frac", [
    (synthetic.Workload("p1", 1, 4, 6, 8, 16, 128, 128, "bf16", "profiled"), 1, 40, 0.05),
    (synthetic.Workload("p2", 1, 2, 6, 8, 16, 64, 64, "bf16", "profiled"), 1, 20, 0.05),
    (synthetic.WAN, 2, 140, 0.01),
])
def test_profile_matches_oracle(wl, w_s, w_t, frac):
    q, k, v = synthetic.make_qkv(wl)
    kinds, mse = _profile_gpu(q, k, v, wl, w_s, w_t, frac)
    _check_profile(q, k, v, wl, w_s, w_t, frac, kinds, mse)


def _far_below_inputs(wl, seed=21):
    """Every query carries 32 on dimension 0; the keys of frame 0 at positions 112-127 carry
    35.25 there (bf16-exact), the rest only N(0,1) noise.  Those 16 keys score about 100
    (natural log; 144 in base 2) above every other key, so a sampled row outside frame 0 has
    all its spatially allowed keys, and a row outside positions 112-127 all its temporally
    allowed keys, far below the row's dense maximum -- beyond the 2^-126 range of fp32."""
    q = synthetic.make_random((1, wl.H, wl.N, wl.d), torch.float32, seed=seed)
    k = synthetic.make_random((1, wl.H, wl.N, wl.d), torch.float32, seed=seed + 1)
    v = synthetic.make_random((1, wl.H, wl.N, wl.d), torch.float32, seed=seed + 2)
    q[..., 0] = 32.0
    k[:, :, 112:128, 0] = 35.25
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


@pytest.mark.parametrize("static", [False, True])
def test_profile_masked_variants_far_below_dense_max(static):
    """A masked variant whose every allowed key sits far below the dense maximum is computed
    with its own maximum (the kernel marks it and recomputes the row), so both MSEs and the
    kind match the oracle instead of collapsing to a zero output."""
    wl = synthetic.Workload("far-below", 1, 2, 4, 8, 16, 128, 64, "bf16", "profiled")
    q, k, v = _far_below_inputs(wl)
    w_s, w_t, frac = 0, 0, 0.05
    kinds, mse = _profile_gpu(q, k, v, wl, w_s, w_t, frac, static=static)
    _check_profile(q, k, v, wl, w_s, w_t, frac, kinds, mse, planted=False)
    for h in range(wl.H):
        _, want, rows = oracle.profile_head(q[0, h], k[0, h], v[0, h], wl.F, wl.Hl, wl.Wl, wl.block, w_s, w_t, frac)
        # the planted keys dominate the dense rows: the variants that miss them differ a lot
        assert want.min() > 0.05
        assert np.any((rows // wl.S) != 0) and np.any((rows % wl.S) // 16 != 7)


# ------------------------------------------------------------------------------------
# in-kernel layout: temporal heads gathered through the frame-major map
# ------------------------------------------------------------------------------------

@pytest.mark.parametrize("F,Hl,Wl,d,block,w_t", [(6, 8, 16, 128, 128, 9), (5, 6, 10, 128, 128, 7),
                                                 (7, 5, 9, 64, 64, 11), (21, 30, 52, 128, 128, 140)])
def test_attention_natural_layout_matches_permuted(F, Hl, Wl, d, block, w_t):
    """vsa_sparse_attn_fwd_natural (rows gathered in-kernel, ragged tails zero-filled) gives the
    permute -> attention -> unpermute result bit for bit, and matches the oracle."""
    wl = synthetic.Workload("nat", 1, 2, F, Hl, Wl, d, block, "bf16", "given")
    q, k, v = synthetic.make_qkv(wl)
    kinds_list = [S_, T_]
    keeps = [keep_for_head(S_, wl, 1, 0), keep_for_head(T_, wl, 0, w_t)]
    shape = _lib.make_shape(1, 2, F, Hl, Wl, d, block)
    nblk = _lib.vsa_num_blocks(shape)
    max_kv = max(int(kp.sum(axis=1).max()) for kp in keeps)
    idx = np.full((1, 2, nblk, max_kv), -1, dtype=np.int32)
    cnt = np.zeros((1, 2, nblk), dtype=np.int32)
    for h, kp in enumerate(keeps):
        i_, c_ = oracle.keep_to_lists(kp, max_kv)
        idx[0, h, :kp.shape[0]] = i_
        cnt[0, h, :kp.shape[0]] = c_
    idx_d, cnt_d = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
    kinds = torch.tensor(kinds_list, dtype=torch.uint8, device="cuda")
    err = cuda_err()
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    # permuted path
    o_p = torch.full_like(qd, 9.0)
    lse_p = torch.full((1, 2, wl.N), 9.0, dtype=torch.float32, device="cuda")
    qp, kp_, vp, op = (torch.empty_like(qd) for _ in range(4))
    lsep = torch.empty(1, 2, wl.N, dtype=torch.float32, device="cuda")
    for src, dst in ((qd, qp), (kd, kp_), (vd, vp)):
        _lib.vsa_permute(src, _lib.VSA_BF16, dst, kinds, shape, err)
    _lib.vsa_sparse_attn_fwd(_lib.qkvo(qd, kd, vd, o_p, lse_p), _lib.qkvo(qp, kp_, vp, op, lsep), kinds, idx_d,
                             cnt_d, max_kv, shape, 0.0, err)
    _lib.vsa_unpermute(op, lsep, o_p, _lib.VSA_BF16, lse_p, kinds, shape, err)
    # in-kernel layout
    o_n = torch.full_like(qd, 9.0)
    lse_n = torch.full((1, 2, wl.N), 9.0, dtype=torch.float32, device="cuda")
    _lib.vsa_sparse_attn_fwd_natural(_lib.qkvo(qd, kd, vd, o_n, lse_n), kinds, idx_d, cnt_d, max_kv, shape, 0.0, err)
    assert _lib.vsa_get_device_error(err) == 0
    assert torch.equal(o_n, o_p) and torch.equal(lse_n, lse_p)
    o_n = o_n.cpu()
    for h, kind in enumerate(kinds_list):
        want, _ = oracle.attention_rows(q[0, h], k[0, h], v[0, h], head_slots(kind, wl), wl.block, keeps[h],
                                        rows=np.arange(wl.N), scale=1.0 / math.sqrt(wl.d))
        assert_close_attention(to_f64(o_n[0, h]), want, f"head {h}")


def test_attention_natural_layout_rejects_cubes():
    shape = _lib.make_shape(1, 1, 8, 8, 8, 128, 128, (4, 4, 8))
    q = torch.zeros(1, 1, 512, 128, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(1, 1, 4, 1, dtype=torch.int32, device="cuda")
    cnt = torch.ones(1, 1, 4, dtype=torch.int32, device="cuda")
    kinds = torch.full((1,), 2, dtype=torch.uint8, device="cuda")
    with pytest.raises(_lib.VsaError) as ex:
        _lib.vsa_sparse_attn_fwd_natural(_lib.qkvo(q, q, q, q), kinds, idx, cnt, 1, shape, 0.0, cuda_err())
    assert ex.value.status == _lib.VSA_ERR_UNSUPPORTED
    # a cube kind byte on a shape without cubes is flagged on the device
    shape = _lib.make_shape(1, 1, 8, 8, 8, 128, 128)
    err = cuda_err()
    o = torch.empty_like(q)
    _lib.vsa_sparse_attn_fwd_natural(_lib.qkvo(q, q, q, o), kinds, idx, cnt, 1, shape, 0.0, err)
    assert _lib.vsa_get_device_error(err) & _lib.VSA_DEVERR_KIND
