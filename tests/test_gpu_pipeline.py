"""End-to-end parity of vsa_attention on the workload configurations.

Small cases compare every output row with the oracle; full-size cases (the launch
configuration the benchmark times) compare the head kinds and masks exactly and a seeded
sample of output rows that the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from parity_util import assert_close_attention, keep_for_head, oracle_rows, to_f64

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


def _run(wl, rows_per_head=None, seed_rows=0, heads=None):
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
            kind = int(got_kinds[b * wl.H + h])
            if wl.mode == "profiled":
                want_kind, _, _ = oracle.profile_head(q[b, h], k[b, h], v[b, h], wl.F, wl.Hl, wl.Wl, wl.block,
                                                      plan.w_s, plan.w_t, wl.profile_frac)
                assert kind == want_kind, (b, h)
            keep = keep_for_head(kind, wl, plan.w_s, plan.w_t, q[b, h], k[b, h])
            # the masks the kernels executed
            nb = keep.shape[0]
            want_idx, want_cnt = oracle.keep_to_lists(keep, plan.max_kv)
            assert np.array_equal(plan.kv_cnt[b, h, :nb].cpu().numpy(), want_cnt)
            assert np.array_equal(plan.kv_idx[b, h, :nb].cpu().numpy(), want_idx)
            rows = (np.arange(wl.N) if rows_per_head is None else
                    synthetic.sample_indices(wl.N, rows_per_head, seed_rows + b * wl.H + h).numpy())
            want, want_lse = oracle_rows(q[b, h], k[b, h], v[b, h], kind, wl, keep, rows)
            assert_close_attention(to_f64(o[b, h])[rows], want, f"{wl.name} batch {b} head {h}")
            assert np.abs(to_f64(lse[b, h])[rows] - want_lse).max() < 2e-2
    return plan


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
    _run(synthetic.WAN, rows_per_head=48)


@pytest.mark.parametrize("target", [1.0, 0.05])
def test_sweep_endpoints_sampled_rows(target):
    _run(synthetic.sweep(target), rows_per_head=24, heads=[0, 1, 6, 11])


def test_hunyuan_profiled_sampled_rows():
    _run(synthetic.HUNYUAN, rows_per_head=12, heads=[0, 1, 2, 3, 22, 23])


def test_wan_6x_cube_sampled_rows():
    _run(synthetic.WAN_6X, rows_per_head=16, heads=[0, 1, 5, 11])


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
