"""End-to-end parity of vsa_attention on the workload configurations.

Small cases compare every output row with the oracle; full-size cases (the launch
configuration the benchmark times) compare the head kinds and masks and, per head, whole
128-row blocks of the head's layout (the first, the last -- the ragged tail or a partial
cube -- and interior ones) plus a seeded sample of rows, which the oracle computes one by one.
Head kinds and top-k cube sets equal the oracle's or are logged near-ties (tests/validity.py);
the attention is then checked under the masks the kernels executed.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import validity
from parity_util import assert_close_attention, head_slots, keep_for_head, oracle_rows, to_f64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_31_b200 as vsa
else:
    vsa = None


def _plan(wl):
    kw = dict(dtype=torch.float32 if wl.dtype == "f32" else torch.bfloat16, with_lse=True)
    if wl.mode == "fixed":
        return vsa.SparseAttention(wl.B, wl.H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block, select="given", w_s=wl.w_s,
                                   w_t=wl.w_t, **kw)
    if wl.mode == "cube":
        return vsa.SparseAttention(wl.B, wl.H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block, select="cube", cube=wl.cube,
                                   topk=wl.topk, **kw)
    return vsa.SparseAttention(wl.B, wl.H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block, select="profile", target=wl.target,
                               profile_frac=wl.profile_frac, **kw)


def _executed_keep(plan, b, h, nb):
    """The block mask the kernels ran for one head, from its kept-block lists."""
    cnt = plan.kv_cnt[b, h, :nb].cpu().numpy()
    idx = plan.kv_idx[b, h, :nb].cpu().numpy()
    keep = np.zeros((nb, nb), dtype=bool)
    for i in range(nb):
        cols = idx[i, :cnt[i]]
        assert np.all(cols[1:] > cols[:-1]) and (cols.size == 0 or (cols[0] >= 0 and cols[-1] < nb))
        keep[i, cols] = True
    return keep


def _block_rows(wl, kind, blocks):
    """Natural tokens whose slot in the head's layout falls in the given blocks."""
    slots = head_slots(kind, wl)
    return np.nonzero(np.isin(slots // wl.block, blocks))[0]


def _run(wl, rows_per_head=None, seed_rows=0, heads=None, blocks=None):
    q, k, v = synthetic.make_qkv(wl)
    plan = _plan(wl)
    kinds = None
    if wl.mode == "fixed":
        kinds = torch.tensor(list(wl.fixed_kinds), dtype=torch.uint8, device="cuda")
    o, lse = plan(q.cuda(), k.cuda(), v.cuda(), kinds=kinds)
    assert plan.device_error() == 0
    o, lse = o.cpu(), lse.cpu()
    got_kinds = plan.kinds.cpu().numpy()  # [B*H]
    heads = range(wl.H) if heads is None else heads
    for b in range(wl.B):
        for h in heads:
            what = f"{wl.name} batch {b} head {h}"
            kind = int(got_kinds[b * wl.H + h])
            if wl.mode == "profiled":
                want_kind, mse, _ = oracle.profile_head(q[b, h], k[b, h], v[b, h], wl.F, wl.Hl, wl.Wl, wl.block,
                                                        plan.w_s, plan.w_t, wl.profile_frac)
                validity.kind_valid(kind, want_kind, mse, what)   # equal, or a logged near-tie
            # the masks the kernels executed: equal to the oracle's for the kind the GPU chose
            if kind == oracle.CUBE:
                want_keep, score = oracle.cube_topk_keep(q[b, h], k[b, h], wl.F, wl.Hl, wl.Wl, wl.topk, wl.cube,
                                                         return_scores=True)
            else:
                want_keep = keep_for_head(kind, wl, plan.w_s, plan.w_t)
            nb = want_keep.shape[0]
            keep = _executed_keep(plan, b, h, nb)
            if kind == oracle.CUBE:
                validity.topk_rows_valid(keep, want_keep, score, wl.topk, what)
            else:
                assert np.array_equal(keep, want_keep), what
            if rows_per_head is None:
                rows = np.arange(wl.N)
            else:
                rows = synthetic.sample_indices(wl.N, rows_per_head, seed_rows + b * wl.H + h).numpy()
                if blocks is not None:
                    rows = np.union1d(rows, _block_rows(wl, kind, blocks(kind, nb)))
            want, want_lse = oracle_rows(q[b, h], k[b, h], v[b, h], kind, wl, keep, rows)
            assert_close_attention(to_f64(o[b, h])[rows], want, what)
            assert np.abs(to_f64(lse[b, h])[rows] - want_lse).max() < 2e-2
    return plan


def _ends_and_middle(kind, nb):
    """The first block, the last block (ragged tail) and one interior block."""
    return [0, nb // 2 + 1, nb - 1]


def test_tiny_fixed_masks_full():
    plan = _run(synthetic.TINY)
    assert plan.kinds.cpu().tolist() == [0, 1]
    # both fixed w=0 masks on this grid are the 4x4 identity
    assert plan.kv_cnt.cpu().flatten().tolist() == [1] * 8


def test_small_profiled_full():
    wl = synthetic.Workload("small profiled", 1, 4, 8, 12, 20, 128, 128, "bf16", "profiled", target=0.3,
                            profile_frac=0.05)
    _run(wl)


def test_batched_profiled_full():
    """B = 2: every (batch, head) is profiled, masked and attended on its own."""
    wl = synthetic.Workload("batched profiled", 2, 3, 7, 10, 18, 128, 128, "bf16", "profiled", target=0.3,
                            profile_frac=0.05)
    _run(wl)


def test_batched_cube_full():
    wl = synthetic.Workload("batched cubes", 2, 2, 16, 16, 32, 128, 128, "bf16", "cube", cube=(4, 4, 8), topk=32)
    _run(wl)


def test_wan_profiled_sampled_rows():
    _run(synthetic.WAN, rows_per_head=48, blocks=_ends_and_middle)


@pytest.mark.parametrize("target", [1.0, 0.35, 0.13, 0.05])
def test_sweep_sampled_rows(target):
    """Every sweep point other than 0.18 (the Wan test): windows (20, 1548), (4, 298),
    (1, 98) and (0, 31)."""
    _run(synthetic.sweep(target), rows_per_head=24, heads=[0, 1, 6, 11], blocks=_ends_and_middle)


def test_hunyuan_profiled_sampled_rows():
    """118800 = 928 * 128 + 16: the last block of a spatial head holds 16 tokens."""
    _run(synthetic.HUNYUAN, rows_per_head=12, heads=[0, 1, 2, 3, 22, 23], blocks=_ends_and_middle)


def _cube_blocks(kind, nb):
    """Wan 6x cubes (32 x 8 x 7 of 4x4x8 tokens on 126x30x52): the first cube, a cube cut at
    the width edge (52 = 6 * 8 + 4), one cut at the height edge (30 = 7 * 4 + 2) and the last,
    cut in all three dimensions (126 = 31 * 4 + 2)."""
    return [0, 6, 7 * 7, nb - 1]


def test_wan_6x_cube_sampled_rows():
    _run(synthetic.WAN_6X, rows_per_head=16, heads=[0, 1, 5, 11], blocks=_cube_blocks)


def test_repeated_calls_identical():
    wl = synthetic.Workload("rep", 1, 2, 6, 8, 16, 128, 128, "bf16", "profiled", target=0.3, profile_frac=0.05)
    q, k, v = (t.cuda() for t in synthetic.make_qkv(wl))
    plan = _plan(wl)
    o1, l1 = plan(q, k, v)
    o1, l1 = o1.clone(), l1.clone()
    o2, l2 = plan(q, k, v)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert plan.device_error() == 0


def test_run_host_overlapped_matches_single_calls():
    """run_host (uploads, compute and downloads of consecutive calls overlapped on three
    streams) returns exactly what one call per batch returns."""
    wl = synthetic.Workload("host", 1, 4, 6, 8, 16, 128, 128, "bf16", "profiled", target=0.3, profile_frac=0.05)
    plan = _plan(wl)
    batches = [tuple(t.pin_memory() for t in synthetic.make_qkv(wl, seed=s)) for s in range(5)]
    outs = plan.run_host(batches)
    assert plan.device_error() == 0
    for (q, k, v), got in zip(batches, outs):
        want = plan(q.cuda(), k.cuda(), v.cuda())
        want = want[0] if isinstance(want, tuple) else want
        assert torch.equal(got, want.cpu())


@pytest.mark.parametrize("wl", [
    synthetic.Workload("small profiled", 1, 4, 8, 12, 20, 128, 128, "bf16", "profiled", target=0.3, profile_frac=0.05),
    synthetic.WAN])
def test_layout_in_kernel_same_result(wl):
    """The whole call with temporal heads gathered in-kernel equals the call with permuted
    copies bit for bit (same kinds, masks, outputs and LSE)."""
    q, k, v = (t.cuda() for t in synthetic.make_qkv(wl))
    outs = []
    for fused in (False, True):
        plan = vsa.SparseAttention(wl.B, wl.H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block, select="profile", target=wl.target,
                                   profile_frac=wl.profile_frac, with_lse=True, layout_in_kernel=fused)
        o, lse = plan(q, k, v)
        assert plan.device_error() == 0
        outs.append((o, lse, plan.kinds.clone(), plan.kv_idx.clone()))
    (o0, l0, k0, i0), (o1, l1, k1, i1) = outs
    assert torch.equal(k0, k1) and torch.equal(i0, i1)
    assert torch.equal(o0, o1) and torch.equal(l0, l1)
