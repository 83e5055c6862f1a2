"""FP8 Q.K^T ("Sparse Video-Gen" summary page, "Measured effects": FP8 quantisation added to
the sparse attention) through the C ABI.

The per-block e4m3 codes and scale exponents equal the oracle's quantiser bit for bit (an
integer result: both sides scale by a power of two exactly and round to nearest even), and
the attention outputs are within the attention tolerance (max-abs 2e-2, relative L2 1e-2) of
the oracle run on the dequantised Q and K -- the values the kernel multiplies -- with V in
bf16, under the masks the kernels executed."""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic
import validity
from parity_util import assert_close_attention, cuda_err, head_slots, keep_for_head, to_f64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_31_b200 as vsa
    from block_sparse_attention_31_b200 import _lib
else:
    vsa = _lib = None

S_, T_, C_ = oracle.SPATIAL, oracle.TEMPORAL, oracle.CUBE


def _layout_rows(x_head, kind, wl):
    """A head's rows in its layout ([R, d], padding zero) as fp64."""
    slots = head_slots(kind, wl)
    R = oracle.layout_rows(kind, wl.F, wl.Hl, wl.Wl, wl.cube)
    out = np.zeros((R, x_head.shape[-1]))
    out[slots] = to_f64(x_head)
    return out


def _dequantised(x_head, kind, wl):
    """The natural-order values the kernel multiplies: quantise the head's layout rows per block,
    dequantise, and map back to tokens."""
    rows = _layout_rows(x_head, kind, wl)
    code, exp = oracle.quantize_e4m3(rows, wl.block)
    return oracle.dequantize_e4m3(code, exp, wl.block)[head_slots(kind, wl)]


@pytest.mark.parametrize("F,Hl,Wl,cubes", [(5, 6, 10, False), (21, 30, 52, False), (9, 9, 17, True)])
def test_quantize_fp8_matches_oracle(F, Hl, Wl, cubes):
    wl = synthetic.Workload("q8", 1, 3, F, Hl, Wl, 128, 128, "bf16", "given")
    kinds_list = [S_, T_, C_] if cubes else [S_, T_, T_]
    shape = _lib.make_shape(1, 3, F, Hl, Wl, 128, 128, wl.cube if cubes else None)
    R = _lib.vsa_layout_rows(shape)
    nblk = _lib.vsa_num_blocks(shape)
    q, k, _ = synthetic.make_qkv(wl)
    kinds = torch.tensor(kinds_list, dtype=torch.uint8, device="cuda")
    err = cuda_err()
    for x in (q, k):
        xd = x.cuda()
        perm = torch.zeros(1, 3, R, 128, dtype=torch.bfloat16, device="cuda")
        _lib.vsa_permute(xd, _lib.VSA_BF16, perm, kinds, shape, err)
        dst = torch.full((1, 3, R, 128), 0x55, dtype=torch.uint8, device="cuda")
        exps = torch.full((3, nblk), -999, dtype=torch.int32, device="cuda")
        _lib.vsa_quantize_fp8(xd, perm, kinds, shape, dst, exps, err)
        assert _lib.vsa_get_device_error(err) == 0
        dst, exps = dst.cpu().numpy(), exps.cpu().numpy()
        for h, kind in enumerate(kinds_list):
            rows = _layout_rows(x[0, h], kind, wl)
            code, exp = oracle.quantize_e4m3(rows, 128)
            n = rows.shape[0]
            assert np.array_equal(dst[0, h, :n], code), (h, kind)
            assert not dst[0, h, n:].any()
            assert np.array_equal(exps[h, :exp.size], exp), (h, kind)
            assert not exps[h, exp.size:].any()


def _run_fp8(wl, select, kinds=None, rows_per_head=None, heads=None, blocks=None, **kw):
    q, k, v = synthetic.make_qkv(wl)
    plan = vsa.SparseAttention(wl.B, wl.H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block, select=select, qk_fp8=True,
                               with_lse=True, **kw)
    kd = None if kinds is None else torch.tensor(kinds, dtype=torch.uint8, device="cuda")
    o, lse = plan(q.cuda(), k.cuda(), v.cuda(), kinds=kd)
    assert plan.device_error() == 0
    o, lse = o.cpu(), lse.cpu()
    got_kinds = plan.kinds.cpu().numpy()
    for h in (range(wl.H) if heads is None else heads):
        what = f"{wl.name} fp8 head {h}"
        kind = int(got_kinds[h])
        if select == "profile":
            want_kind, mse, _ = oracle.profile_head(q[0, h], k[0, h], v[0, h], wl.F, wl.Hl, wl.Wl, wl.block,
                                                    plan.w_s, plan.w_t, wl.profile_frac)
            validity.kind_valid(kind, want_kind, mse, what)
        if kind == C_:
            want_keep, score = oracle.cube_topk_keep(q[0, h], k[0, h], wl.F, wl.Hl, wl.Wl, wl.topk, wl.cube,
                                                     return_scores=True)
        else:
            want_keep = keep_for_head(kind, wl, plan.w_s, plan.w_t)
        nb = want_keep.shape[0]
        cnt = plan.kv_cnt[0, h, :nb].cpu().numpy()
        idx = plan.kv_idx[0, h, :nb].cpu().numpy()
        keep = np.zeros((nb, nb), dtype=bool)
        for i in range(nb):
            keep[i, idx[i, :cnt[i]]] = True
        if kind == C_:
            validity.topk_rows_valid(keep, want_keep, score, wl.topk, what)
        else:
            assert np.array_equal(keep, want_keep), what
        if rows_per_head is None:
            rows = np.arange(wl.N)
        else:
            rows = synthetic.sample_indices(wl.N, rows_per_head, seed=h).numpy()
            if blocks is not None:
                slots = head_slots(kind, wl)
                rows = np.union1d(rows, np.nonzero(np.isin(slots // wl.block, blocks(nb)))[0])
        qd, kq = _dequantised(q[0, h], kind, wl), _dequantised(k[0, h], kind, wl)
        want, want_lse = oracle.attention_rows(qd, kq, v[0, h], head_slots(kind, wl), wl.block, keep, rows=rows,
                                               scale=1.0 / math.sqrt(wl.d))
        assert_close_attention(to_f64(o[0, h])[rows], want, what)
        assert np.abs(to_f64(lse[0, h])[rows] - want_lse).max() < 2e-2


def test_fp8qk_given_kinds_full():
    wl = synthetic.Workload("fp8 small", 1, 3, 8, 12, 20, 128, 128, "bf16", "given")
    _run_fp8(wl, "given", kinds=[S_, T_, T_], w_s=1, w_t=30)


def test_fp8qk_cubes_full():
    wl = synthetic.Workload("fp8 cubes", 1, 2, 16, 16, 32, 128, 128, "bf16", "cube", topk=8)
    _run_fp8(wl, "cube", cube=wl.cube, topk=wl.topk)


def _ends(nb):
    return [0, nb // 2 + 1, nb - 1]


def test_fp8qk_wan_profiled_sampled_rows():
    wl = synthetic.WAN
    _run_fp8(wl, "profile", rows_per_head=32, heads=[0, 1, 6, 11], blocks=_ends, target=wl.target,
             profile_frac=wl.profile_frac)


def test_fp8qk_hunyuan_profiled_sampled_rows():
    wl = synthetic.HUNYUAN
    _run_fp8(wl, "profile", rows_per_head=8, heads=[0, 1, 22, 23], blocks=_ends, target=wl.target,
             profile_frac=wl.profile_frac)


def test_fp8qk_equals_entry_points():
    """The whole call equals quantise -> vsa_sparse_attn_fwd_fp8qk run stage by stage."""
    wl = synthetic.Workload("fp8 stages", 1, 2, 6, 8, 16, 128, 128, "bf16", "given")
    q, k, v = (t.cuda() for t in synthetic.make_qkv(wl))
    plan = vsa.SparseAttention(1, 2, wl.F, wl.Hl, wl.Wl, 128, 128, select="given", w_s=1, w_t=20, qk_fp8=True)
    kinds = torch.tensor([S_, T_], dtype=torch.uint8, device="cuda")
    o = plan(q, k, v, kinds=kinds)
    shape = plan.shape
    R = _lib.vsa_layout_rows(shape)
    nblk = _lib.vsa_num_blocks(shape)
    err = cuda_err()
    perm = [torch.zeros(1, 2, R, 128, dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    for src, dst in zip((q, k, v), perm[:3]):
        _lib.vsa_permute(src, _lib.VSA_BF16, dst, kinds, shape, err)
    q8 = torch.empty(1, 2, R, 128, dtype=torch.uint8, device="cuda")
    k8 = torch.empty_like(q8)
    qe = torch.empty(2, nblk, dtype=torch.int32, device="cuda")
    ke = torch.empty_like(qe)
    _lib.vsa_quantize_fp8(q, perm[0], kinds, shape, q8, qe, err)
    _lib.vsa_quantize_fp8(k, perm[1], kinds, shape, k8, ke, err)
    o2 = torch.empty_like(q)
    _lib.vsa_sparse_attn_fwd_fp8qk(_lib.qkvo(q, k, v, o2), _lib.qkvo(*perm), q8, qe, k8, ke, kinds, plan.kv_idx,
                                   plan.kv_cnt, plan.max_kv, shape, 0.0, err)
    _lib.vsa_unpermute(perm[3], None, o2, _lib.VSA_BF16, None, kinds, shape, err)
    assert _lib.vsa_get_device_error(err) == 0
    assert torch.equal(o, o2)


def test_fp8qk_rejects_unsupported_shapes():
    for d, block in ((64, 128), (128, 64)):
        with pytest.raises(_lib.VsaError) as ex:
            vsa.SparseAttention(1, 2, 4, 8, 16, d, block, select="given", w_s=1, w_t=4, qk_fp8=True)
        assert ex.value.status in (_lib.VSA_ERR_UNSUPPORTED, _lib.VSA_ERR_INVALID_ARG)
