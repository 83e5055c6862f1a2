"""GPU parity of the semantic-aware permutation (Sparse VideoGen2 page, abstract) through
the C ABI.

The oracle decides every k-means label, top-p set and block on exact fp64 values; the
kernels decide the labels in fp32.  Each stage is therefore checked from the GPU's own
previous stage: per round, the GPU's labels against the oracle's assignment from the GPU's
previous centroids (equal, or a near-tie within the kernel's fp32 error bound, logged), then
the GPU's centroids, counts and cluster-major order bit for bit against the oracle's update
of those labels; the top-p cluster sets against the oracle's from the GPU's centroids (equal,
or a near-tie, logged); the block mask and lists bit for bit against the oracle's from the
GPU's labels and cluster sets; attention outputs within the attention tolerance of the
oracle under the GPU's block mask.  k-means is deterministic, so the run with T rounds
repeats the first T-1 rounds of the run with T-1 rounds: each round is read from its own run.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic
import validity
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


def _unpack_bits(words, n):
    """[rows, ceil(n/32)] uint32 bitset -> bool [rows, n]."""
    w = np.asarray(words).view(np.uint32)
    bits = (w[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1
    return bits.reshape(w.shape[0], -1)[:, :n].astype(bool)


def _check_kmeans_rounds(x_head, runs, h, C, what):
    """Every round of one head: labels valid from the GPU's previous centroids, then the
    update, counts and order bit for bit from those labels.  Returns the near-ties."""
    x = x_head.float().numpy()
    prev = oracle.kmeans_init(x, C)
    ties = 0
    for T, (cent, label, count, perm) in enumerate(runs, 1):
        lab = label[h].cpu().numpy()
        ties += validity.labels_valid(x, prev, lab, f"{what} round {T}")
        want_c, want_n = oracle.kmeans_update(x, lab, prev)
        assert np.array_equal(count[h].cpu().numpy(), want_n), f"{what} round {T}: counts"
        got_c = cent[h].cpu().numpy()
        assert np.array_equal(got_c.view(np.uint32), want_c.view(np.uint32)), f"{what} round {T}: centroids"
        assert np.array_equal(perm[h].cpu().numpy(), oracle.cluster_perm(lab, C)[0]), f"{what} round {T}: order"
        prev = got_c
    return ties


@pytest.mark.parametrize("F,Hl,Wl,d,C,iters", [(5, 7, 13, 64, 16, 3), (5, 7, 13, 128, 200, 2),
                                               (3, 10, 20, 128, 1, 1), (4, 8, 16, 64, 512, 2),
                                               (4, 8, 16, 64, 250, 2), (5, 7, 13, 128, 300, 1)])
def test_kmeans_matches_oracle(F, Hl, Wl, d, C, iters):
    """Every round's labels (valid nearest centroids), centroids, counts and order (ragged N,
    a single cluster; one or two resident centroid tiles (C <= 256) and streamed tiles above
    that, for d = 64 and 128)."""
    wl = _wl(F, Hl, Wl, d)
    q, k, _ = synthetic.make_qkv(wl)
    shape = _lib.make_shape(1, wl.H, F, Hl, Wl, d, 128)
    for name, x in (("q", q), ("k", k)):
        xd = x.cuda()
        runs = [_kmeans_gpu(xd, shape, C, T) for T in range(1, iters + 1)]
        for h in range(wl.H):
            _check_kmeans_rounds(x[0, h], runs, h, C, f"{name} head {h}")


def test_kmeans_update_wide_range_exact():
    """Member values of one dimension spanning more than 53 binades (2^-60 next to values of
    order 1): the update's parallel sums are not provably exact there, so both of its fallbacks
    run (a thread's fp32 sums redone in fp64, and the cluster's ordered token-order sum); the
    centroids must still equal the oracle's token-order fp64 update bit for bit."""
    F, Hl, Wl, d, C = 4, 8, 16, 64, 8
    N = F * Hl * Wl
    g = torch.Generator().manual_seed(31)
    x = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    x[0, 0, ::3, 5] = 2.0 ** -60
    x[0, 0, 1::7, 9] = -3 * 2.0 ** -60
    assert float(x[0, 0, 0, 5]) == 2.0 ** -60       # exact in bf16
    shape = _lib.make_shape(1, 1, F, Hl, Wl, d, 128)
    xd = x.cuda()
    runs = [_kmeans_gpu(xd, shape, C, T) for T in range(1, 3)]
    _check_kmeans_rounds(x[0, 0], runs, 0, C, "wide-range head")


def test_kmeans_wan_heads_match_oracle():
    """The Wan grid at the benchmark's cluster counts and rounds: one spatial- and one
    temporal-structured head, every round."""
    wl = synthetic.WAN_SEMANTIC
    q, k, _ = synthetic.make_qkv(wl, heads=[0, 1])
    shape = _lib.make_shape(1, 2, wl.F, wl.Hl, wl.Wl, wl.d, wl.block)
    C, iters = wl.clusters[0], wl.kmeans_iters
    for name, x in (("q", q), ("k", k)):
        xd = x.cuda()
        runs = [_kmeans_gpu(xd, shape, C, T) for T in range(1, iters + 1)]
        for h in range(2):
            _check_kmeans_rounds(x[0, h], runs, h, C, f"wan {name} head {h}")


def _check_semantic_mask(gq, gk, h, cq, ck, d, block, top_p, keep_words, bits, idx, cnt, what):
    """Top-p sets from the GPU's centroids, then the block mask from the GPU's labels and sets.
    Returns the block mask (bool [nb, nb]) the attention must have run."""
    cent_q, lab_q, cnt_q, perm_q = (t[h].cpu().numpy() for t in gq)
    cent_k, lab_k, cnt_k, perm_k = (t[h].cpu().numpy() for t in gk)
    sc = oracle.semantic_scale(d)
    w = oracle.semantic_weights(cent_q, cnt_q, cent_k, cnt_k, sc)
    keep_o = oracle.semantic_keep(cent_q, cnt_q, cent_k, cnt_k, sc, top_p)
    keep_g = _unpack_bits(keep_words, ck)
    validity.topp_rows_valid(keep_g, keep_o, w, top_p, what)
    kb = oracle.semantic_block_keep(lab_q, perm_q, lab_k, perm_k, keep_g, block)
    nblk = kb.shape[0]
    assert np.array_equal(np.asarray(bits).view(np.uint32), oracle.keep_to_bits(kb)), f"{what}: bits"
    want_idx, want_cnt = oracle.keep_to_lists(kb, nblk)
    got_cnt = np.asarray(cnt)
    assert np.array_equal(got_cnt, want_cnt), f"{what}: counts"
    got_idx = np.asarray(idx)
    for i in range(nblk):
        assert np.array_equal(got_idx[i, :got_cnt[i]], want_idx[i, :want_cnt[i]]), f"{what}: list {i}"
    return kb


@pytest.mark.parametrize("block,top_p,cq,ck", [(128, 0.6, 24, 40), (64, 0.3, 40, 24), (128, 1.0, 16, 16),
                                               (64, 0.95, 100, 130)])
def test_semantic_mask_matches_oracle(block, top_p, cq, ck):
    """Kept cluster pairs (equal, or a logged near-tie) and the block bitset, lists and counts
    bit for bit, from the GPU's k-means results."""
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
    gq4 = (gq[0], gq[1], gq[2], gq[3])
    gk4 = (gk[0], gk[1], gk[2], gk[3])
    kept_any = False
    for h in range(wl.H):
        kb = _check_semantic_mask(gq4, gk4, h, cq, ck, wl.d, block, top_p, keep[h].cpu().numpy(),
                                  bits[h].cpu().numpy(), idx[h].cpu().numpy(), cnt[h].cpu().numpy(), f"head {h}")
        kept_any |= bool(kb.mean() < 1.0)
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


def _semantic_stages(q, k, v, shape, N, d, block, cq, ck, iters, top_p):
    """The semantic call stage by stage through the C ABI (the launches vsa_semantic_attention
    makes), keeping every intermediate result."""
    BH = q.shape[0] * q.shape[1]
    gq = _kmeans_gpu(q, shape, cq, iters)
    gk = _kmeans_gpu(k, shape, ck, iters)
    err = cuda_err()
    qp, kp, vp, op = (torch.empty_like(q) for _ in range(4))
    _lib.vsa_gather_rows(q, gq[3], qp, shape, err)
    _lib.vsa_gather_rows(k, gk[3], kp, shape, err)
    _lib.vsa_gather_rows(v, gk[3], vp, shape, err)
    nblk = -(-N // block)
    keep = torch.zeros(BH, cq, -(-ck // 32), dtype=torch.int32, device="cuda")
    bits = torch.zeros(q.shape[0], q.shape[1], nblk, -(-nblk // 32), dtype=torch.int32, device="cuda")
    idx = torch.full((q.shape[0], q.shape[1], nblk, nblk), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(q.shape[0], q.shape[1], nblk, dtype=torch.int32, device="cuda")
    wsb = _lib.vsa_semantic_mask_workspace_size(shape)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    _lib.vsa_semantic_mask(gq[0], gq[2], gq[1], gq[3], cq, gk[0], gk[2], gk[1], gk[3], ck, shape, top_p, 0.0, keep,
                           bits, idx, cnt, nblk, ws, wsb, err)
    kinds = torch.full((BH,), _lib.VSA_TEMPORAL, dtype=torch.uint8, device="cuda")
    lsep = torch.empty(q.shape[0], q.shape[1], N, dtype=torch.float32, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty_like(lsep)
    _lib.vsa_sparse_attn_fwd(_lib.qkvo(q, k, v, o, lse), _lib.qkvo(qp, kp, vp, op, lsep), kinds, idx, cnt, nblk,
                             shape, 0.0, err)
    _lib.vsa_scatter_rows(op, lsep, gq[3], o, lse, shape, err)
    assert _lib.vsa_get_device_error(err) == 0
    return dict(gq=gq, gk=gk, keep=keep, bits=bits, idx=idx, cnt=cnt, o=o, lse=lse)


def _check_semantic_call(wl, heads, q, k, v, cq, ck, iters, top_p, rows_of):
    """The whole call equals the stage-by-stage run bit for bit; every stage of the latter is
    valid against the oracle; sampled output rows are within tolerance of the oracle's
    attention under the GPU's block mask."""
    H = len(heads)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    plan = vsa.SemanticAttention(1, H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block, cq=cq, ck=ck, iters=iters, top_p=top_p,
                                 with_lse=True)
    o, lse = plan(qd, kd, vd)
    assert plan.device_error() == 0
    shape = _lib.make_shape(1, H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block)
    st = _semantic_stages(qd, kd, vd, shape, wl.N, wl.d, wl.block, cq, ck, iters, top_p)
    assert torch.equal(o, st["o"]) and torch.equal(lse, st["lse"])
    runs_q = [_kmeans_gpu(qd, shape, cq, T) for T in range(1, iters + 1)]
    runs_k = [_kmeans_gpu(kd, shape, ck, T) for T in range(1, iters + 1)]
    o, lse = o.cpu(), lse.cpu()
    for h in range(H):
        _check_kmeans_rounds(q[0, h], runs_q, h, cq, f"q head {h}")
        _check_kmeans_rounds(k[0, h], runs_k, h, ck, f"k head {h}")
        kb = _check_semantic_mask(st["gq"], st["gk"], h, cq, ck, wl.d, wl.block, top_p, st["keep"][h].cpu().numpy(),
                                  st["bits"][0, h].cpu().numpy(), st["idx"][0, h].cpu().numpy(),
                                  st["cnt"][0, h].cpu().numpy(), f"head {h}")
        perm_q, perm_k = st["gq"][3][h].cpu().numpy(), st["gk"][3][h].cpu().numpy()
        qslot = np.empty(wl.N, dtype=np.int64)
        qslot[perm_q] = np.arange(wl.N)
        kslot = np.empty(wl.N, dtype=np.int64)
        kslot[perm_k] = np.arange(wl.N)
        rows = rows_of(qslot)
        want, want_lse = oracle.attention_rows(q[0, h], k[0, h], v[0, h], qslot, wl.block, kb, rows=rows,
                                               kslots=kslot, scale=1.0 / math.sqrt(wl.d))
        assert_close_attention(to_f64(o[0, h])[rows], want, f"head {h}")
        assert np.abs(to_f64(lse[0, h])[rows] - want_lse).max() < 2e-2


@pytest.mark.parametrize("F,Hl,Wl,d,block,cq,ck,top_p", [(6, 9, 17, 128, 128, 24, 40, 0.6),
                                                         (5, 8, 12, 64, 64, 30, 20, 0.4),
                                                         (4, 10, 16, 128, 128, 16, 16, 1.0)])
def test_semantic_attention_matches_oracle(F, Hl, Wl, d, block, cq, ck, top_p):
    """The whole call on small grids: every output row within the attention tolerance, LSE
    within 2e-2."""
    wl = _wl(F, Hl, Wl, d, block=block)
    q, k, v = synthetic.make_qkv(wl)
    _check_semantic_call(wl, list(range(wl.H)), q, k, v, cq, ck, 3, top_p, lambda qslot: np.arange(wl.N))


def test_semantic_attention_wan_sampled_rows():
    """The benchmark's configuration (Wan grid, 128/128 clusters, 4 rounds, top-p 0.6) on two
    heads: the first, the last (ragged) and an interior 128-row block of the query layout,
    plus a seeded sample of rows."""
    wl = synthetic.WAN_SEMANTIC
    heads = [0, 1]
    q, k, v = synthetic.make_qkv(wl, heads=heads)
    sample = synthetic.sample_indices(wl.N, 48, seed=5).numpy()
    nb = -(-wl.N // wl.block)

    def rows_of(qslot):
        perm = np.argsort(qslot)       # token at each slot of the query layout
        slots = np.concatenate([np.arange(0, wl.block), np.arange((nb - 1) * wl.block, wl.N),
                                np.arange(100 * wl.block, 101 * wl.block)])
        return np.unique(np.concatenate([perm[slots], sample]))

    _check_semantic_call(wl, heads, q, k, v, wl.clusters[0], wl.clusters[1], wl.kmeans_iters, wl.top_p, rows_of)
