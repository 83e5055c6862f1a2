"""GPU parity of the semantic-aware permutation (Sparse VideoGen2 page, abstract) through
the C ABI: k-means centroids, labels, counts and cluster-major orders bit for bit; the
top-p cluster mask and the block mask and lists bit for bit; row gather/scatter exactly;
attention outputs within the attention tolerance of the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from parity_util import assert_close_attention, cuda_err, to_f64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import block_sparse_attention_31_b200 as vsa
    from block_sparse_attention_31_b200 import _lib
else:
    vsa = _lib = None


def _wl(F, Hl, Wl, d, block=128, H=2):
    return synthetic.WAN.with_(name="semantic test", H=H, F=F, Hl=Hl, Wl=Wl, d=d, block=block, mode="semantic")


def _kmeans_gpu(x, shape, C, iters):
    BH, N, d = x.shape[0] * x.shape[1], x.shape[2], x.shape[3]
    cent = torch.full((BH, C, d), 7.0, dtype=torch.float32, device="cuda")
    label = torch.full((BH, N), -9, dtype=torch.int32, device="cuda")
    count = torch.full((BH, C), -9, dtype=torch.int32, device="cuda")
    perm = torch.full((BH, N), -9, dtype=torch.int32, device="cuda")
    wsb = _lib.vsa_kmeans_workspace_size(shape, C)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    err = cuda_err()
    _lib.vsa_kmeans(x, shape, C, iters, cent, label, count, perm, ws, wsb, err)
    assert _lib.vsa_get_device_error(err) == 0
    return cent, label, count, perm


@pytest.mark.parametrize("F,Hl,Wl,d,C,iters", [(5, 7, 13, 64, 16, 3), (5, 7, 13, 128, 200, 2),
                                               (3, 10, 20, 128, 1, 1), (4, 8, 16, 64, 512, 2)])
def test_kmeans_matches_oracle(F, Hl, Wl, d, C, iters):
    """Centroids, labels, counts and order equal the oracle's bit for bit (ragged N, one and
    several centroid tiles, a single cluster)."""
    wl = _wl(F, Hl, Wl, d)
    q, k, _ = synthetic.make_qkv(wl)
    shape = _lib.make_shape(1, wl.H, F, Hl, Wl, d, 128)
    for x in (q, k):
        cent, label, count, perm = _kmeans_gpu(x.cuda(), shape, C, iters)
        for h in range(wl.H):
            oc, ol, on = oracle.kmeans(x[0, h], C, iters)
            op, _ = oracle.cluster_perm(ol, C)
            assert np.array_equal(label[h].cpu().numpy(), ol), f"labels head {h}"
            assert np.array_equal(count[h].cpu().numpy(), on), f"counts head {h}"
            assert np.array_equal(perm[h].cpu().numpy(), op), f"order head {h}"
            assert np.array_equal(cent[h].cpu().numpy().view(np.uint32), oc.view(np.uint32)), f"centroids head {h}"


def test_kmeans_wan_heads_match_oracle():
    """The Wan grid at the benchmark's cluster counts: one spatial- and one
    temporal-structured head."""
    wl = synthetic.WAN_SEMANTIC
    q, k, _ = synthetic.make_qkv(wl, heads=[0, 1])
    shape = _lib.make_shape(1, 2, wl.F, wl.Hl, wl.Wl, wl.d, wl.block)
    C, iters = wl.clusters[0], wl.kmeans_iters
    cent, label, count, perm = _kmeans_gpu(q.cuda(), shape, C, iters)
    for h in range(2):
        oc, ol, on = oracle.kmeans(q[0, h], C, iters)
        assert np.array_equal(label[h].cpu().numpy(), ol)
        assert np.array_equal(cent[h].cpu().numpy().view(np.uint32), oc.view(np.uint32))
        assert np.array_equal(perm[h].cpu().numpy(), oracle.cluster_perm(ol, C)[0])


@pytest.mark.parametrize("block,top_p,cq,ck", [(128, 0.6, 24, 40), (64, 0.3, 40, 24), (128, 1.0, 16, 16),
                                               (64, 0.95, 100, 130)])
def test_semantic_mask_matches_oracle(block, top_p, cq, ck):
    """Kept cluster pairs, block bitset, lists and counts equal the oracle's bit for bit."""
    wl = _wl(6, 9, 17, 128, block=block)
    q, k, _ = synthetic.make_qkv(wl)
    shape = _lib.make_shape(1, wl.H, wl.F, wl.Hl, wl.Wl, wl.d, block)
    gq = _kmeans_gpu(q.cuda(), shape, cq, 3)
    gk = _kmeans_gpu(k.cuda(), shape, ck, 3)
    nblk = -(-wl.N // block)
    kw, bw = -(-ck // 32), -(-nblk // 32)
    keep = torch.zeros(wl.H, cq, kw, dtype=torch.int32, device="cuda")
    bits = torch.zeros(wl.H, nblk, bw, dtype=torch.int32, device="cuda")
    idx = torch.full((wl.H, nblk, nblk), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((wl.H, nblk), -1, dtype=torch.int32, device="cuda")
    wsb = _lib.vsa_semantic_mask_workspace_size(shape)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    err = cuda_err()
    _lib.vsa_semantic_mask(gq[0], gq[2], gq[1], gq[3], cq, gk[0], gk[2], gk[1], gk[3], ck, shape, top_p, 0.0, keep,
                           bits, idx, cnt, nblk, ws, wsb, err)
    assert _lib.vsa_get_device_error(err) == 0
    kept_any = False
    for h in range(wl.H):
        res = oracle.semantic_head(q[0, h], k[0, h], None, cq, ck, 3, top_p, block, attention=False)
        want_keep = oracle.keep_to_bits(res["keep_clusters"])
        assert np.array_equal(keep[h].cpu().numpy().view(np.uint32), want_keep), f"cluster mask head {h}"
        kb = res["keep_blocks"]
        assert np.array_equal(bits[h].cpu().numpy().view(np.uint32), oracle.keep_to_bits(kb)), f"bits head {h}"
        want_idx, want_cnt = oracle.keep_to_lists(kb, nblk)
        got_cnt = cnt[h].cpu().numpy()
        assert np.array_equal(got_cnt, want_cnt), f"counts head {h}"
        got_idx = idx[h].cpu().numpy()
        for i in range(nblk):
            assert np.array_equal(got_idx[i, :got_cnt[i]], want_idx[i, :want_cnt[i]])
        kept_any |= bool((kb.mean() < 1.0))
    if top_p < 1.0:
        assert kept_any, "the budget should drop some block pairs"


def test_gather_scatter_rows_exact():
    """gather then scatter through a random per-head order is the identity; gather equals
    indexing and scatter moves the LSE with its row."""
    shape = _lib.make_shape(2, 3, 3, 7, 11, 64, 64)
    N = 3 * 7 * 11
    x = synthetic.make_random((2, 3, N, 64), seed=4).cuda()
    g = torch.Generator().manual_seed(3)
    perm = torch.stack([torch.randperm(N, generator=g) for _ in range(6)]).to(torch.int32).cuda()
    y = torch.empty_like(x)
    err = cuda_err()
    _lib.vsa_gather_rows(x, perm, y, shape, err)
    want = torch.stack([x.view(6, N, 64)[i, perm[i].long()] for i in range(6)]).view_as(x)
    assert torch.equal(y, want)
    lse = torch.randn(2, 3, N, device="cuda")
    back = torch.empty_like(x)
    lse_back = torch.empty_like(lse)
    _lib.vsa_scatter_rows(y, lse, perm, back, lse_back, shape, err)
    assert torch.equal(back, x)
    want_lse = torch.empty_like(lse).view(6, N)
    for i in range(6):
        want_lse[i, perm[i].long()] = lse.view(6, N)[i]
    assert torch.equal(lse_back.view(6, N), want_lse)
    assert _lib.vsa_get_device_error(err) == 0


@pytest.mark.parametrize("F,Hl,Wl,d,block,cq,ck,top_p", [(6, 9, 17, 128, 128, 24, 40, 0.6),
                                                         (5, 8, 12, 64, 64, 30, 20, 0.4),
                                                         (4, 10, 16, 128, 128, 16, 16, 1.0)])
def test_semantic_attention_matches_oracle(F, Hl, Wl, d, block, cq, ck, top_p):
    """The whole call: every output row within the attention tolerance of the oracle, LSE
    within 2e-2."""
    wl = _wl(F, Hl, Wl, d, block=block)
    q, k, v = synthetic.make_qkv(wl)
    plan = vsa.SemanticAttention(1, wl.H, F, Hl, Wl, d, block, cq=cq, ck=ck, iters=3, top_p=top_p, with_lse=True)
    o, lse = plan(q.cuda(), k.cuda(), v.cuda())
    assert plan.device_error() == 0
    for h in range(wl.H):
        res = oracle.semantic_head(q[0, h], k[0, h], v[0, h], cq, ck, 3, top_p, block)
        assert_close_attention(to_f64(o[0, h]), res["out"], f"head {h}")
        assert np.abs(to_f64(lse[0, h]) - res["lse"]).max() < 2e-2


def test_semantic_attention_wan_sampled_rows():
    """The benchmark's configuration (Wan grid, 128/128 clusters, 4 rounds, top-p 0.6): a
    seeded sample of rows of two heads against the oracle."""
    wl = synthetic.WAN_SEMANTIC
    heads = [0, 1]
    q, k, v = synthetic.make_qkv(wl, heads=heads)
    plan = vsa.SemanticAttention(1, len(heads), wl.F, wl.Hl, wl.Wl, wl.d, wl.block, cq=wl.clusters[0],
                                 ck=wl.clusters[1], iters=wl.kmeans_iters, top_p=wl.top_p)
    o = plan(q.cuda(), k.cuda(), v.cuda())
    assert plan.device_error() == 0
    rows = synthetic.sample_indices(wl.N, 48, seed=5).numpy()
    for h in range(len(heads)):
        res = oracle.semantic_head(q[0, h], k[0, h], v[0, h], wl.clusters[0], wl.clusters[1], wl.kmeans_iters,
                                   wl.top_p, wl.block, rows=rows)
        assert_close_attention(to_f64(o[0, h])[rows], res["out"], f"head {h}")
