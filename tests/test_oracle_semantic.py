"""Pins of the oracle's semantic-aware permutation (Sparse VideoGen2 page, abstract:
k-means clustering of tokens, cluster-major reordering, top-p budget over clusters).

The checks take routes other than the oracle's own loops:
- planted blobs whose clustering is known in closed form;
- scipy's cdist distances and numpy means for the assignment and update;
- a hand-built case that only exact (fp64) distances resolve;
- bincount/argsort for the order;
- numpy weights for the top-p prefix;
- membership-matrix products for the block mask;
- torch fp64 SDPA and a token-level numpy softmax for the attention.
"""
import math

import numpy as np
import pytest
import torch

import oracle


# ------------------------------------------------------------------------------------
# k-means
# ------------------------------------------------------------------------------------

def _blobs(N, C, d, seed=0, spread=10.0, noise=0.1):
    """Token t belongs to blob t*C//N; centres far apart, small noise."""
    rng = np.random.default_rng(seed)
    centres = rng.standard_normal((C, d)) * spread
    blob = (np.arange(N) * C) // N
    x = centres[blob] + rng.standard_normal((N, d)) * noise
    return x.astype(np.float32), blob


def _fp32_mean(rows):
    return np.float32(np.mean(rows.astype(np.float64), axis=0))


@pytest.mark.parametrize("N,C,d", [(300, 7, 16), (1000, 16, 64)])
def test_kmeans_recovers_planted_blobs(N, C, d):
    """The initial rows floor((2j+1)N/2C) fall one in each contiguous blob, so one round
    already gives the blob partition; centroids are the blob means."""
    x, blob = _blobs(N, C, d)
    for iters in (1, 3):
        cent, label, count = oracle.kmeans(x, C, iters)
        assert np.array_equal(label, blob)
        assert np.array_equal(count, np.bincount(blob, minlength=C))
        for j in range(C):
            np.testing.assert_array_max_ulp(cent[j], _fp32_mean(x[blob == j]), maxulp=1)


def test_kmeans_assignment_and_update_rules():
    """Round T assigns each row to the nearest centroid of round T-1 (scipy's Euclidean
    distances), and round T's centroids are the fp32 means of those members; the single
    steps compose into the whole k-means."""
    from scipy.spatial.distance import cdist
    rng = np.random.default_rng(3)
    x = rng.standard_normal((800, 32)).astype(np.float32)
    C = 12
    prev, _, _ = oracle.kmeans(x, C, 2)
    cent, label, count = oracle.kmeans(x, C, 3)
    dist = cdist(x.astype(np.float64), prev.astype(np.float64))
    assert np.array_equal(label, np.argmin(dist, axis=1))
    assert np.array_equal(count, np.bincount(label, minlength=C))
    for j in range(C):
        if count[j]:
            np.testing.assert_array_max_ulp(cent[j], _fp32_mean(x[label == j]), maxulp=1)
        else:
            assert np.array_equal(cent[j], prev[j])
    # the exposed steps: assign against round 2's centroids, update from those labels
    lab, gap = oracle.kmeans_assign(x, prev)
    assert np.array_equal(lab, label)
    srt = np.sort(dist ** 2, axis=1)
    np.testing.assert_allclose(gap, srt[:, 1] - srt[:, 0], rtol=1e-9, atol=1e-12)
    c2, n2 = oracle.kmeans_update(x, lab, prev)
    assert np.array_equal(c2.view(np.uint32), cent.view(np.uint32)) and np.array_equal(n2, count)
    c0 = oracle.kmeans_init(x, C)
    assert np.array_equal(c0, x[[(2 * j + 1) * 800 // (2 * C) for j in range(C)]])


def test_kmeans_assignment_is_exact():
    """Centroids 1 and 1 + 2^-21 and the row 1 + 3*2^-23 (all exact in fp32): the second
    centroid is nearer (2^-23 against 3*2^-23), a gap that fp32's |c|^2 - 2 x.c form rounds
    to a tie (which would pick the first); the oracle's fp64 distances resolve it."""
    x = np.array([[1.0 + 3 * 2.0 ** -23], [1.0], [5.0], [1.0 + 2.0 ** -21]], dtype=np.float32)
    assert float(x[0, 0]) == 1.0 + 3 * 2.0 ** -23 and float(x[3, 0]) == 1.0 + 2.0 ** -21
    # the fp32 form of the distance ties
    c = x[[1, 3], 0]
    two = np.float32(2.0)
    d32 = [np.float32(cj * cj) - np.float32(two * np.float32(x[0, 0] * cj)) for cj in c]
    assert d32[0] == d32[1]
    cent, label, count = oracle.kmeans(x, 2, 1)      # initial centroids: rows 1 and 3
    assert label[0] == 1 and label[1] == 0 and label[3] == 1 and label[2] == 1


def test_kmeans_ties_and_empty_clusters():
    """Two equal initial centroids: in the first round every row goes to the smaller index
    (ties), so the other cluster is empty and keeps its centroid."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((64, 8)).astype(np.float32)
    x[24] = x[8]                         # initial rows of clusters 0 and 1 (C = 4)
    cent, label, count = oracle.kmeans(x, 4, 1)
    assert count[1] == 0 and not np.any(label == 1) and count[0] > 0
    assert np.array_equal(cent[1], x[8])
    assert not np.array_equal(cent[0], x[8])


def test_kmeans_one_and_all_clusters():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((20, 8)).astype(np.float32)
    cent, label, count = oracle.kmeans(x, 1, 2)
    assert np.all(label == 0) and count[0] == 20
    np.testing.assert_array_max_ulp(cent[0], _fp32_mean(x), maxulp=1)
    cent, label, count = oracle.kmeans(x, 20, 1)      # every row its own seed
    assert np.array_equal(label, np.arange(20)) and np.all(count == 1)
    with pytest.raises(ValueError):
        oracle.kmeans(x, 21, 1)


# ------------------------------------------------------------------------------------
# cluster-major order
# ------------------------------------------------------------------------------------

def test_cluster_perm_is_stable_sort():
    rng = np.random.default_rng(7)
    label = rng.integers(0, 9, size=500).astype(np.int32)
    label[label == 4] = 5                # an empty cluster
    perm, offset = oracle.cluster_perm(label, 9)
    assert np.array_equal(perm, np.argsort(label, kind="stable"))
    assert np.array_equal(offset, np.concatenate([[0], np.cumsum(np.bincount(label, minlength=9))]))


# ------------------------------------------------------------------------------------
# top-p budget
# ------------------------------------------------------------------------------------

def _weights(cq, ck, nk, scale):
    s = scale * cq.astype(np.float64) @ ck.astype(np.float64).T
    s[:, nk == 0] = -np.inf
    w = nk[None, :] * np.exp(s - s.max(axis=1, keepdims=True))
    return w


def _centroids(seed, Cq=9, Ck=13, d=16):
    rng = np.random.default_rng(seed)
    cq = rng.standard_normal((Cq, d)).astype(np.float32)
    ck = rng.standard_normal((Ck, d)).astype(np.float32)
    nq = rng.integers(1, 50, size=Cq).astype(np.int32)
    nk = rng.integers(1, 50, size=Ck).astype(np.int32)
    nq[2] = 0
    nk[5] = 0
    return cq, nq, ck, nk


@pytest.mark.parametrize("top_p", [0.3, 0.6, 0.9, 0.99])
def test_topp_is_the_shortest_heaviest_prefix(top_p):
    """Kept clusters: the heaviest ones, and the fewest whose weight reaches top_p of the
    row (numpy weights, relative slack 1e-12)."""
    cq, nq, ck, nk = _centroids(8)
    scale = 0.5
    keep = oracle.semantic_keep(cq, nq, ck, nk, scale, top_p)
    w = _weights(cq, ck, nk, scale)
    assert not keep[2].any() and not keep[:, 5].any()
    for i in np.nonzero(nq)[0]:
        kept, rest = w[i, keep[i]], w[i, ~keep[i] & (nk > 0)]
        total = w[i, nk > 0].sum()
        assert kept.size >= 1
        assert rest.size == 0 or kept.min() >= rest.max()
        assert kept.sum() >= top_p * total * (1 - 1e-12)
        assert kept.sum() - kept.min() < top_p * total * (1 + 1e-12)


def test_topp_limits_and_monotone():
    cq, nq, ck, nk = _centroids(9)
    full = oracle.semantic_keep(cq, nq, ck, nk, 0.5, 1.0)
    assert np.array_equal(full, (nq[:, None] > 0) & (nk[None, :] > 0))
    one = oracle.semantic_keep(cq, nq, ck, nk, 0.5, 1e-9)
    w = _weights(cq, ck, nk, 0.5)
    for i in np.nonzero(nq)[0]:
        assert np.array_equal(np.nonzero(one[i])[0], [int(np.argmax(w[i]))])
    prev = one
    for p in (0.2, 0.5, 0.8, 1.0):
        cur = oracle.semantic_keep(cq, nq, ck, nk, 0.5, p)
        assert np.all(cur >= prev)
        prev = cur


def test_topp_weights_by_cluster_size():
    """Two key clusters with the same centroid: their weights are in proportion to their
    sizes, so at top_p = 0.5 only the large one is kept; ties go to the smaller index."""
    d = 8
    cq = np.ones((1, d), dtype=np.float32)
    ck = np.ones((3, d), dtype=np.float32)
    ck[2] = -1.0
    keep = oracle.semantic_keep(cq, np.array([5], np.int32), ck, np.array([1, 99, 1], np.int32), 0.3, 0.5)
    assert np.array_equal(keep[0], [False, True, False])
    keep = oracle.semantic_keep(cq, np.array([5], np.int32), ck, np.array([7, 7, 1], np.int32), 0.3, 0.4)
    assert np.array_equal(keep[0], [True, False, False])


# ------------------------------------------------------------------------------------
# block mask over the two cluster-major layouts
# ------------------------------------------------------------------------------------

def _membership(label, perm, block):
    ls = np.asarray(label)[np.asarray(perm)]
    nb = -(-ls.size // block)
    m = np.zeros((nb, int(ls.max()) + 1))
    m[np.arange(ls.size) // block, ls] = 1.0
    return m


def test_block_keep_equals_membership_product():
    rng = np.random.default_rng(10)
    N, block, Cq, Ck = 333, 32, 11, 7
    lq = rng.integers(0, Cq, size=N).astype(np.int32)
    lk = rng.integers(0, Ck, size=N).astype(np.int32)
    pq, _ = oracle.cluster_perm(lq, Cq)
    pk, _ = oracle.cluster_perm(lk, Ck)
    keep = rng.random((Cq, Ck)) < 0.15
    got = oracle.semantic_block_keep(lq, pq, lk, pk, keep, block)
    mq, mk = _membership(lq, pq, block), _membership(lk, pk, block)
    want = (mq[:, :Cq] @ keep[:mq.shape[1]].astype(float) @ mk.T[:Ck]) > 0
    assert np.array_equal(got, want)


def test_block_keep_closed_forms():
    """One cluster per block: the cluster mask is the block mask."""
    block, C = 16, 6
    label = (np.arange(C * block) // block).astype(np.int32)
    perm, _ = oracle.cluster_perm(label, C)
    assert np.array_equal(perm, np.arange(C * block))
    eye = np.eye(C, dtype=bool)
    assert np.array_equal(oracle.semantic_block_keep(label, perm, label, perm, eye, block), eye)
    shift = np.roll(eye, 1, axis=1)
    assert np.array_equal(oracle.semantic_block_keep(label, perm, label, perm, shift, block), shift)
    ones = np.ones((C, C), dtype=bool)
    assert oracle.semantic_block_keep(label, perm, label, perm, ones, block).all()


# ------------------------------------------------------------------------------------
# the whole head
# ------------------------------------------------------------------------------------

def test_semantic_head_full_budget_is_dense_attention():
    """top_p = 1 keeps every cluster pair, so every block pair: dense softmax attention."""
    g = torch.Generator().manual_seed(11)
    N, d = 300, 32
    q, k, v = (torch.randn(N, d, generator=g, dtype=torch.float64) for _ in range(3))
    res = oracle.semantic_head(q, k, v, 8, 6, 2, 1.0, 64)
    assert res["keep_blocks"].all()
    want = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None])[0].numpy()
    np.testing.assert_allclose(res["out"], want, atol=1e-12, rtol=0)


def test_semantic_head_token_level_brute_force():
    """A sparse budget: each output row equals a numpy softmax over the keys whose
    cluster-major block pair is kept (separate query and key layouts)."""
    g = torch.Generator().manual_seed(12)
    N, d, block = 200, 16, 32
    q, k, v = (torch.randn(N, d, generator=g, dtype=torch.float64) for _ in range(3))
    res = oracle.semantic_head(q, k, v, 10, 12, 3, 0.5, block)
    kb = res["keep_blocks"]
    assert 0 < kb.mean() < 1
    qslot = np.argsort(res["perm_q"])
    kslot = np.argsort(res["perm_k"])
    allowed = kb[qslot[:, None] // block, kslot[None, :] // block]
    s = (q.numpy() @ k.numpy().T) / math.sqrt(d)
    s[~allowed] = -np.inf
    p = np.exp(s - s.max(axis=1, keepdims=True))
    want = (p / p.sum(axis=1, keepdims=True)) @ v.numpy()
    np.testing.assert_allclose(res["out"], want, atol=1e-12, rtol=0)


def test_semantic_weights_match_numpy():
    """The exposed criticality weights equal numpy's n_j exp(s_ij - max_j s_ij); empty
    clusters are marked -1; the top-p rows are built from these weights."""
    cq, nq, ck, nk = _centroids(13)
    w = oracle.semantic_weights(cq, nq, ck, nk, 0.5)
    want = _weights(cq, ck, nk, 0.5)
    live = (nq[:, None] > 0) & (nk[None, :] > 0)
    np.testing.assert_allclose(w[live], want[live], rtol=1e-13, atol=0)
    assert np.all(w[~live] == -1.0)
