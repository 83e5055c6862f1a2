"""Pins of the fp64 CPU oracle against what the pages and the mathematics fix.

Every check here uses a route other than the oracle's own formula: hand-computed
fixtures (tests/golden), numpy reshapes/transposes for the layouts, token-level brute
force for the block masks, torch's fp64 scaled_dot_product_attention and scipy's
logsumexp as independent library routines, closed forms (Q = 0, constant V, one
dominant key) and invariants (convex combination, symmetry, monotonicity).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
KIND = {"spatial": oracle.SPATIAL, "temporal": oracle.TEMPORAL, "cube": oracle.CUBE}


# ------------------------------------------------------------------------------------
# independent derivations used by several pins
# ------------------------------------------------------------------------------------

def frame_major_order(F, Hl, Wl):
    """Natural token sitting at each frame-major slot: transpose of the [F, S] grid."""
    return np.arange(F * Hl * Wl).reshape(F, Hl * Wl).T.ravel()


def cube_major_order(F, Hl, Wl, cube):
    """Natural token (or -1 for padding) at each cube-major slot, via pad/reshape/transpose."""
    cf, ch, cw = cube
    nf, nh, nw = -(-F // cf), -(-Hl // ch), -(-Wl // cw)
    grid = -np.ones((nf * cf, nh * ch, nw * cw), dtype=np.int64)
    grid[:F, :Hl, :Wl] = np.arange(F * Hl * Wl).reshape(F, Hl, Wl)
    blocks = grid.reshape(nf, cf, nh, ch, nw, cw).transpose(0, 2, 4, 1, 3, 5)
    return blocks.ravel()


def brute_force_keep(kind, F, Hl, Wl, block, w):
    """Block mask from the token-level rule: some query of block i and key of block j have
    frame distance <= w (spatial, natural order) or position distance <= w (temporal,
    frame-major order)."""
    N, S = F * Hl * Wl, Hl * Wl
    order = np.arange(N) if kind == oracle.SPATIAL else frame_major_order(F, Hl, Wl)
    coord = order // S if kind == oracle.SPATIAL else order % S
    nb = -(-N // block)
    keep = np.zeros((nb, nb), dtype=bool)
    for i in range(nb):
        ci = coord[i * block:(i + 1) * block]
        for j in range(nb):
            cj = coord[j * block:(j + 1) * block]
            keep[i, j] = bool((np.abs(ci[:, None] - cj[None, :]) <= w).any())
    return keep


def softmax_rows_python(q, k, v, allowed, scale):
    """Pure-Python masked softmax attention (tiny sizes only)."""
    N, d = q.shape
    out = np.zeros((N, d))
    lse = np.full(N, -np.inf)
    for t in range(N):
        scores = [(u, scale * sum(q[t, x] * k[u, x] for x in range(d))) for u in range(N) if allowed[t, u]]
        if not scores:
            continue
        m = max(s for _, s in scores)
        tot = sum(math.exp(s - m) for _, s in scores)
        for u, s in scores:
            out[t] += math.exp(s - m) / tot * v[u]
        lse[t] = m + math.log(tot)
    return out, lse


def token_allowed(slots, block, keep):
    b = slots // block
    return keep[b[:, None], b[None, :]]


# ------------------------------------------------------------------------------------
# layouts
# ------------------------------------------------------------------------------------

def test_layout_golden_values():
    n = 0
    with open(os.path.join(GOLDEN, "layout_slots.txt")) as fh:
        for line in fh:
            line = line.split("#")[0].strip()
            if not line:
                continue
            kind, F, Hl, Wl, cf, ch, cw, t, want = line.split()
            F, Hl, Wl, cf, ch, cw, t, want = map(int, (F, Hl, Wl, cf, ch, cw, t, want))
            slots = oracle.layout_slots(KIND[kind], F, Hl, Wl, (cf, ch, cw))
            assert slots[t] == want, (kind, t)
            n += 1
    assert n >= 15


@pytest.mark.parametrize("F,Hl,Wl", [(4, 8, 8), (3, 2, 5), (21, 30, 52), (7, 3, 11)])
def test_temporal_layout_is_transpose(F, Hl, Wl):
    slots = oracle.layout_slots(oracle.TEMPORAL, F, Hl, Wl)
    N = F * Hl * Wl
    assert np.array_equal(np.sort(slots), np.arange(N))          # bijection
    inv = frame_major_order(F, Hl, Wl)                             # token at each slot
    assert np.array_equal(slots[inv], np.arange(N))                # pi o pi^-1 = id
    assert np.array_equal(inv[slots], np.arange(N))                # pi^-1 o pi = id


@pytest.mark.parametrize("F,Hl,Wl,cube", [(5, 5, 9, (4, 4, 8)), (126, 30, 52, (4, 4, 8)), (8, 8, 16, (4, 4, 8)),
                                          (3, 7, 5, (2, 3, 2))])
def test_cube_layout_matches_reshape(F, Hl, Wl, cube):
    slots = oracle.layout_slots(oracle.CUBE, F, Hl, Wl, cube)
    order = cube_major_order(F, Hl, Wl, cube)
    rows = oracle.layout_rows(oracle.CUBE, F, Hl, Wl, cube)
    assert rows == len(order)
    real = order >= 0
    assert np.array_equal(slots[order[real]], np.nonzero(real)[0])
    assert len(np.unique(slots)) == F * Hl * Wl


def test_identity_layout():
    assert np.array_equal(oracle.layout_slots(oracle.SPATIAL, 3, 4, 5), np.arange(60))


# ------------------------------------------------------------------------------------
# pattern masks and windows
# ------------------------------------------------------------------------------------

def _golden_masks():
    out, cur = [], None
    with open(os.path.join(GOLDEN, "pattern_masks.txt")) as fh:
        for line in fh:
            line = line.split("#")[0].strip()
            if not line:
                continue
            if line.startswith("mask"):
                _, kind, F, Hl, Wl, block, w = line.split()
                cur = (KIND[kind], int(F), int(Hl), int(Wl), int(block), int(w), [])
                out.append(cur)
            else:
                cur[6].append([int(x) for x in line.split()])
    return out


def test_pattern_mask_golden():
    masks = _golden_masks()
    assert len(masks) == 5
    for kind, F, Hl, Wl, block, w, rows in masks:
        got = oracle.pattern_keep(kind, F, Hl, Wl, block, w)
        assert np.array_equal(got, np.array(rows, dtype=bool)), (kind, F, Hl, Wl, block, w)


@pytest.mark.parametrize("kind", [oracle.SPATIAL, oracle.TEMPORAL])
@pytest.mark.parametrize("F,Hl,Wl,block", [(4, 8, 8, 64), (3, 2, 5, 8), (5, 3, 7, 16), (6, 5, 4, 32), (7, 4, 9, 24)])
def test_pattern_mask_brute_force(kind, F, Hl, Wl, block):
    wmax = F if kind == oracle.SPATIAL else Hl * Wl
    for w in range(0, wmax + 1):
        want = brute_force_keep(kind, F, Hl, Wl, block, w)
        got = oracle.pattern_keep(kind, F, Hl, Wl, block, w)
        assert np.array_equal(got, want), w


@pytest.mark.parametrize("kind", [oracle.SPATIAL, oracle.TEMPORAL])
def test_pattern_mask_invariants(kind):
    F, Hl, Wl, block = 7, 6, 10, 32
    prev = None
    wmax = F - 1 if kind == oracle.SPATIAL else Hl * Wl - 1
    for w in range(0, wmax + 1, max(1, wmax // 12)):
        keep = oracle.pattern_keep(kind, F, Hl, Wl, block, w)
        assert np.array_equal(keep, keep.T)                      # symmetric
        assert keep.diagonal().all()                             # own block always kept
        if prev is not None:
            assert (keep | ~prev).all() and keep.sum() >= prev.sum()   # monotone in w
        prev = keep
    assert oracle.pattern_keep(kind, F, Hl, Wl, block, wmax).all()     # widest window = dense


@pytest.mark.parametrize("kind", [oracle.SPATIAL, oracle.TEMPORAL])
@pytest.mark.parametrize("target", [1.0, 0.35, 0.18, 0.13, 0.05])
def test_window_for_target_is_smallest(kind, target):
    F, Hl, Wl, block = 21, 30, 52, 128
    w = oracle.window_for_target(kind, F, Hl, Wl, block, target)
    nb = -(-(F * Hl * Wl) // block)
    kept = brute = oracle.pattern_keep(kind, F, Hl, Wl, block, w).sum() / nb ** 2
    assert kept >= target
    if w > 0:
        below = oracle.pattern_keep(kind, F, Hl, Wl, block, w - 1).sum() / nb ** 2
        assert below < target
    assert abs(oracle.kept_fraction(kind, F, Hl, Wl, block, w) - brute) < 1e-15


def test_profile_rows_count():
    # ceil(1% of N): 327.6 -> 328 and 1188 exactly (hand arithmetic).
    assert oracle.profile_rows(32760, 0.01) == 328
    assert oracle.profile_rows(118800, 0.01) == 1188
    assert oracle.profile_rows(256, 0.01) == 3
    assert oracle.profile_rows(10, 1e-9) == 1


# ------------------------------------------------------------------------------------
# attention
# ------------------------------------------------------------------------------------

def _rand(shape, seed, scale=1.0):
    return synthetic.make_random(shape, torch.float64, seed=seed, scale=scale).numpy()


def test_all_ones_mask_equals_sdpa():
    N, d, block = 200, 16, 32
    q, k, v = _rand((N, d), 1), _rand((N, d), 2), _rand((N, d), 3)
    nb = -(-N // block)
    keep = np.ones((nb, nb), dtype=bool)
    out, lse = oracle.attention_rows(q, k, v, np.arange(N), block, keep)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None], torch.from_numpy(v)[None, None])[0, 0]
    assert np.abs(out - ref.numpy()).max() < 1e-12
    from scipy.special import logsumexp
    want_lse = logsumexp(q @ k.T / math.sqrt(d), axis=1)
    assert np.abs(lse - want_lse).max() < 1e-12


def test_masked_attention_equals_sdpa_with_token_mask():
    F, Hl, Wl, d, block = 3, 4, 6, 8, 16
    N = F * Hl * Wl
    q, k, v = _rand((N, d), 4), _rand((N, d), 5), _rand((N, d), 6)
    slots = oracle.layout_slots(oracle.TEMPORAL, F, Hl, Wl)
    keep = brute_force_keep(oracle.TEMPORAL, F, Hl, Wl, block, 2)
    allowed = token_allowed(slots, block, keep)
    out, _ = oracle.attention_rows(q, k, v, slots, block, keep)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
        attn_mask=torch.from_numpy(allowed)[None])[0]
    assert np.abs(out - ref.numpy()).max() < 1e-12


def test_brute_force_python_tiny():
    N, d, block = 40, 6, 8
    rng = np.random.default_rng(7)
    q, k, v = rng.standard_normal((N, d)), rng.standard_normal((N, d)), rng.standard_normal((N, d))
    slots = rng.permutation(N)
    nb = N // block
    keep = rng.random((nb, nb)) < 0.4
    keep[0, :] = False                          # a q block with no kept key block at all
    out, lse = oracle.attention_rows(q, k, v, slots, block, keep)
    want, want_lse = softmax_rows_python(q, k, v, token_allowed(slots, block, keep), 1 / math.sqrt(d))
    assert np.abs(out - want).max() < 1e-12
    fin = np.isfinite(want_lse)
    assert np.array_equal(np.isfinite(lse), fin)
    assert np.abs(lse[fin] - want_lse[fin]).max() < 1e-12
    empty = slots // block == 0
    assert (out[empty] == 0).all() and np.isneginf(lse[empty]).all()


def test_closed_forms():
    F, Hl, Wl, d, block = 4, 4, 4, 8, 16
    N = F * Hl * Wl
    slots = oracle.layout_slots(oracle.SPATIAL, F, Hl, Wl)
    keep = oracle.pattern_keep(oracle.SPATIAL, F, Hl, Wl, block, 1)
    allowed = token_allowed(slots, block, keep)
    k, v = _rand((N, d), 8), _rand((N, d), 9)
    # Q = 0: uniform weights, output = mean of the allowed V rows
    out, lse = oracle.attention_rows(np.zeros((N, d)), k, v, slots, block, keep)
    for t in range(N):
        assert np.abs(out[t] - v[allowed[t]].mean(axis=0)).max() < 1e-13
        assert abs(lse[t] - math.log(allowed[t].sum())) < 1e-13
    # constant V: output = that constant
    q = _rand((N, d), 10)
    cv = np.tile(np.linspace(-2, 3, d), (N, 1))
    out, _ = oracle.attention_rows(q, k, cv, slots, block, keep)
    assert np.abs(out - cv).max() < 1e-13
    # one dominant allowed key: output = its V row
    kd = k.copy()
    kd[5] = 40.0 * q[0] / np.linalg.norm(q[0])
    out, _ = oracle.attention_rows(q, kd, v, slots, block, keep, rows=[0])
    assert allowed[0, 5]
    assert np.abs(out[0] - v[5]).max() < 1e-9


def test_convex_combination():
    F, Hl, Wl, d, block = 5, 4, 6, 16, 32
    N = F * Hl * Wl
    q, k, v = _rand((N, d), 11, 3.0), _rand((N, d), 12, 3.0), _rand((N, d), 13)
    slots = oracle.layout_slots(oracle.TEMPORAL, F, Hl, Wl)
    keep = oracle.pattern_keep(oracle.TEMPORAL, F, Hl, Wl, block, 3)
    allowed = token_allowed(slots, block, keep)
    out, _ = oracle.attention_rows(q, k, v, slots, block, keep)
    for t in range(N):
        vs = v[allowed[t]]
        assert (out[t] >= vs.min(axis=0) - 1e-12).all() and (out[t] <= vs.max(axis=0) + 1e-12).all()
    # weights sum to one: attention of an all-ones V column returns exactly 1
    out1, _ = oracle.attention_rows(q, k, np.ones((N, d)), slots, block, keep)
    assert np.abs(out1 - 1).max() < 1e-12


def test_row_subset_equals_full():
    F, Hl, Wl, d, block = 3, 5, 7, 8, 16
    N = F * Hl * Wl
    q, k, v = _rand((N, d), 14), _rand((N, d), 15), _rand((N, d), 16)
    slots = oracle.layout_slots(oracle.TEMPORAL, F, Hl, Wl)
    keep = oracle.pattern_keep(oracle.TEMPORAL, F, Hl, Wl, block, 4)
    full, lse_full = oracle.attention_rows(q, k, v, slots, block, keep)
    rows = np.array([0, 17, 55, N - 1])
    sub, lse_sub = oracle.attention_rows(q, k, v, slots, block, keep, rows=rows)
    assert np.array_equal(sub, full[rows]) and np.array_equal(lse_sub, lse_full[rows])


# ------------------------------------------------------------------------------------
# cube top-k
# ------------------------------------------------------------------------------------

def _pooled_scores_numpy(q, k, F, Hl, Wl, cube):
    order = cube_major_order(F, Hl, Wl, cube)
    vol = cube[0] * cube[1] * cube[2]
    C = len(order) // vol
    qb, kb = np.zeros((C, q.shape[1])), np.zeros((C, q.shape[1]))
    for c in range(C):
        toks = order[c * vol:(c + 1) * vol]
        toks = toks[toks >= 0]
        qb[c], kb[c] = q[toks].mean(axis=0), k[toks].mean(axis=0)
    return qb @ kb.T


def test_cube_scores_and_rank_rule():
    F, Hl, Wl, d, cube, topk = 6, 7, 10, 16, (4, 4, 8), 3
    N = F * Hl * Wl
    q, k = _rand((N, d), 20), _rand((N, d), 21)
    keep, score = oracle.cube_topk_keep(q, k, F, Hl, Wl, topk, cube, return_scores=True)
    want = _pooled_scores_numpy(q, k, F, Hl, Wl, cube)
    assert np.abs(score - want).max() < 1e-12
    C = score.shape[0]
    for c in range(C):
        for c2 in range(C):
            better = (score[c] > score[c, c2]) | ((score[c] == score[c, c2]) & (np.arange(C) < c2))
            in_topk = better.sum() < topk
            assert keep[c, c2] == (in_topk or c2 == c)
        assert keep[c].sum() in (topk, topk + 1)


def test_cube_topk_ties_go_to_smaller_index():
    F, Hl, Wl, d, cube = 8, 4, 16, 4, (4, 4, 8)     # 2 x 1 x 2 = 4 cubes
    N = F * Hl * Wl
    q = np.ones((N, d))
    k = np.ones((N, d))                             # every score identical
    keep = oracle.cube_topk_keep(q, k, F, Hl, Wl, 2, cube)
    C = keep.shape[0]
    assert C == 4
    for c in range(C):
        want = {0, 1, c}
        assert set(np.nonzero(keep[c])[0]) == want


def test_cube_topk_all_and_planted():
    F, Hl, Wl, d, cube = 9, 9, 17, 8, (4, 4, 8)
    N = F * Hl * Wl
    q, k = _rand((N, d), 22), _rand((N, d), 23)
    C = oracle.num_cubes(F, Hl, Wl, cube)
    assert oracle.cube_topk_keep(q, k, F, Hl, Wl, C, cube).all()
    # planted key cube: every query gets a positive component along dim 0 and the tokens
    # of one cube carry a huge key along it, so that cube must be selected by every row
    q2 = q.copy()
    q2[:, 0] = np.abs(q2[:, 0]) + 1.0
    k2 = k.copy()
    slots = oracle.layout_slots(oracle.CUBE, F, Hl, Wl, cube)
    planted = 5
    k2[slots // 128 == planted, 0] = 1000.0
    keep = oracle.cube_topk_keep(q2, k2, F, Hl, Wl, 2, cube)
    assert keep[:, planted].all()


# ------------------------------------------------------------------------------------
# profiling
# ------------------------------------------------------------------------------------

def test_profile_recovers_planted_kinds():
    wl = synthetic.Workload("profile-pin", 1, 4, 6, 8, 16, 32, 64, "f32", "profiled", target=0.2)
    q, k, v = synthetic.make_qkv(wl)
    w_s = oracle.window_for_target(oracle.SPATIAL, wl.F, wl.Hl, wl.Wl, wl.block, 0.2)
    w_t = oracle.window_for_target(oracle.TEMPORAL, wl.F, wl.Hl, wl.Wl, wl.block, 0.2)
    for h in range(wl.H):
        kind, mse, rows = oracle.profile_head(q[0, h], k[0, h], v[0, h], wl.F, wl.Hl, wl.Wl, wl.block,
                                              w_s, w_t, 0.05)
        assert kind == (oracle.SPATIAL if h % 2 == 0 else oracle.TEMPORAL)
        assert min(mse) * 20 < max(mse)


def test_profile_mse_definition_and_tie():
    F, Hl, Wl, d, block = 4, 6, 8, 16, 32
    N = F * Hl * Wl
    q, k, v = _rand((N, d), 30), _rand((N, d), 31), _rand((N, d), 32)
    w_s, w_t = 1, 9
    kind, mse, rows = oracle.profile_head(q, k, v, F, Hl, Wl, block, w_s, w_t, 0.1)
    assert len(rows) == math.ceil(0.1 * N)
    assert (np.diff(rows) > 0).all() and rows[0] >= 0 and rows[-1] < N
    # dense reference on the sampled rows from torch SDPA, masked ones from token masks
    qt, kt, vt = (torch.from_numpy(x)[None] for x in (q, k, v))
    dense = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0].numpy()[rows]
    es = []
    for kd, w in ((oracle.SPATIAL, w_s), (oracle.TEMPORAL, w_t)):
        slots = np.arange(N) if kd == oracle.SPATIAL else np.argsort(frame_major_order(F, Hl, Wl))
        allowed = torch.from_numpy(token_allowed(slots, block, brute_force_keep(kd, F, Hl, Wl, block, w)))
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=allowed[None])[0].numpy()
        es.append(((o[rows] - dense) ** 2).mean())
    assert np.allclose(mse, es, rtol=1e-9, atol=1e-15)
    assert kind == (oracle.TEMPORAL if es[1] < es[0] else oracle.SPATIAL)
    # both windows dense: identical candidates, tie goes to spatial
    kind, mse, _ = oracle.profile_head(q, k, v, F, Hl, Wl, block, F - 1, Hl * Wl - 1, 0.1)
    assert kind == oracle.SPATIAL and mse[0] == mse[1]


# ------------------------------------------------------------------------------------
# format conversion helpers
# ------------------------------------------------------------------------------------

def test_keep_to_lists_and_bits():
    keep = np.zeros((3, 40), dtype=bool)
    keep[0, [0, 31, 32, 39]] = True
    keep[2, 5] = True
    idx, cnt = oracle.keep_to_lists(keep, 5)
    assert cnt.tolist() == [4, 0, 1]
    assert idx[0].tolist() == [0, 31, 32, 39, -1] and idx[1].tolist() == [-1] * 5
    bits = oracle.keep_to_bits(keep)
    assert bits.shape == (3, 2)
    assert bits[0, 0] == (1 | (1 << 31)) and bits[0, 1] == (1 | (1 << 7)) and bits[2, 0] == 32
