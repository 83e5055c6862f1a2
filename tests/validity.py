"""Validity checks for GPU answers that may differ from the oracle's at near-ties.

Several steps of the path turn floating-point values into integers: a k-means label (an
argmin of distances), a top-p cluster set (a prefix of sorted weights), a top-k cube set (the
k largest coarse scores) and a head's kind (the smaller of two errors).  The oracle takes
each decision on exact (fp64) values; the kernels take it in their own precision.  Where the
oracle's deciding gap is below the bound stated with each check, both answers are correct:
the GPU's answer is accepted, logged here, and the downstream checks continue from it.
Everywhere else the GPU's answer must equal the oracle's.

The log is printed at the end of the test session (tests/conftest.py).
"""
from __future__ import annotations

import collections

import numpy as np

import oracle

NEAR_TIES = collections.Counter()
LOG = []

U32 = 2.0 ** -24        # unit roundoff of fp32
REL_TOPK = 1e-9          # top-k cubes: the k-th and (k+1)-th fp64 scores closer than this (relative)
REL_TOPP = 1e-9          # top-p: slack of the prefix conditions (relative)
REL_KIND = 1e-3          # head kind: the two MSEs closer than this (relative)


def _log(category: str, detail: str):
    NEAR_TIES[category] += 1
    LOG.append((category, detail))


def labels_valid(x, cent, lab_gpu, what: str = "") -> int:
    """k-means labels.  The kernel computes D_j = fl(|c_j|^2 - 2 s_j) with one rounding, where
    |c_j|^2 is an fp32 fused multiply-add chain of d terms (error <= gamma_d |c_j|^2) and
    s_j = x.c_hi + x.c_lo comes from the tensor cores: c_j = c_hi + c_lo + r with bf16 halves,
    |r_i| <= 2^-18 |c_ji|, every product exact, 2d of them accumulated in fp32.  Allowing each
    accumulation step an error of 2u (a truncating adder), |s_j - x.c_j| <= (gamma'_2d
    (1 + 2^-8) + 2^-18) sum_i |x_i c_ji| with gamma'_2d = 4du / (1 - 4du).  So the error of D_j
    is at most E_j = gamma_d |c_j|^2 + 2 (gamma'_2d (1 + 2^-8) + 2^-18) sum_i |x_i c_ji| + u |D_j|
    (gamma_d = du / (1 - du), u = 2^-24).  A label j_g other than the oracle's j_o is accepted
    when the fp64 distances satisfy dist(j_g) - dist(j_o) <= 2 (E_jg + E_jo).  Returns the
    number of accepted differences."""
    x = np.asarray(x, dtype=np.float32)
    cent = np.asarray(cent, dtype=np.float32)
    lab_gpu = np.asarray(lab_gpu)
    lab_o, _ = oracle.kmeans_assign(x, cent)
    diff = np.nonzero(lab_gpu != lab_o)[0]
    if diff.size == 0:
        return 0
    d = x.shape[1]
    gamma = d * U32 / (1 - d * U32)
    gamma_tc = 4 * d * U32 / (1 - 4 * d * U32)
    x64, c64 = x.astype(np.float64), cent.astype(np.float64)

    def err(t, j):
        c = c64[j]
        D = c @ c - 2.0 * (x64[t] @ c)
        dot = (gamma_tc * (1 + 2.0 ** -8) + 2.0 ** -18) * np.abs(x64[t] * c).sum()
        return gamma * (c @ c) + 2.0 * dot + U32 * abs(D)

    for t in diff:
        jg, jo = int(lab_gpu[t]), int(lab_o[t])
        assert 0 <= jg < cent.shape[0], f"{what}: label {jg} out of range at row {t}"
        dg = float(((x64[t] - c64[jg]) ** 2).sum())
        do = float(((x64[t] - c64[jo]) ** 2).sum())
        bound = 2.0 * (err(t, jg) + err(t, jo))
        assert dg - do <= bound, f"{what}: row {t} label {jg} (dist {dg!r}) vs oracle {jo} ({do!r}), bound {bound:.3e}"
        _log("kmeans label", f"{what} row {t}: {jg} vs {jo}, gap {dg - do:.3e} <= {bound:.3e}")
    return int(diff.size)


def topk_rows_valid(keep_gpu, keep_oracle, score, topk: int, what: str = "") -> int:
    """Top-k cube sets (own cube always kept).  A row that differs from the oracle's is
    accepted when it has as many members and every cube in the symmetric difference scores
    within REL_TOPK (1 + |s_k|) of the oracle's k-th largest score s_k of that row."""
    keep_gpu, keep_oracle = np.asarray(keep_gpu, bool), np.asarray(keep_oracle, bool)
    rows = np.nonzero((keep_gpu != keep_oracle).any(axis=1))[0]
    for c in rows:
        assert keep_gpu[c].sum() == keep_oracle[c].sum(), f"{what}: row {c} keeps {keep_gpu[c].sum()} cubes"
        assert keep_gpu[c, c], f"{what}: row {c} lost its own cube"
        s = score[c]
        sk = float(np.sort(s)[::-1][min(topk, s.size) - 1])
        tol = REL_TOPK * (1.0 + abs(sk))
        swapped = np.nonzero(keep_gpu[c] != keep_oracle[c])[0]
        assert np.all(np.abs(s[swapped] - sk) <= tol), \
            f"{what}: row {c} swaps cubes {swapped.tolist()} with scores {s[swapped]} far from s_k={sk!r}"
        _log("top-k cube", f"{what} row {c}: swapped {swapped.tolist()} at s_k={sk!r}")
    return int(rows.size)


def topp_rows_valid(keep_gpu, keep_oracle, w, top_p: float, what: str = "") -> int:
    """Top-p cluster sets.  w [Cq, Ck] are the oracle's fp64 weights (-1 = empty cluster).  A
    row that differs from the oracle's is accepted when it is still a shortest heaviest prefix
    reaching top_p within a relative slack REL_TOPP: every kept weight >= every dropped one,
    the kept sum reaches top_p of the total, and the kept sum without its lightest member
    does not."""
    keep_gpu, keep_oracle = np.asarray(keep_gpu, bool), np.asarray(keep_oracle, bool)
    rows = np.nonzero((keep_gpu != keep_oracle).any(axis=1))[0]
    eps = REL_TOPP
    for i in rows:
        live = w[i] >= 0
        assert not np.any(keep_gpu[i] & ~live), f"{what}: row {i} keeps an empty cluster"
        kept, rest = w[i, keep_gpu[i]], w[i, ~keep_gpu[i] & live]
        total = w[i, live].sum()
        assert kept.size >= 1, f"{what}: row {i} keeps nothing"
        assert rest.size == 0 or kept.min() >= rest.max() * (1 - eps), f"{what}: row {i} is not a heaviest set"
        assert kept.sum() >= top_p * total * (1 - eps), f"{what}: row {i} does not reach top_p"
        assert kept.sum() - kept.min() < top_p * total * (1 + eps), f"{what}: row {i} is not the shortest prefix"
        _log("top-p cluster", f"{what} row {i}: {np.nonzero(keep_gpu[i] != keep_oracle[i])[0].tolist()}")
    return int(rows.size)


def kind_valid(kind_gpu: int, kind_oracle: int, mse_oracle, what: str = "") -> bool:
    """Head kind.  A kind other than the oracle's is accepted when the oracle's two MSEs differ
    by less than REL_KIND of the larger one."""
    if int(kind_gpu) == int(kind_oracle):
        return False
    ms, mt = float(mse_oracle[0]), float(mse_oracle[1])
    gap = abs(ms - mt) / max(ms, mt, 1e-300)
    assert gap < REL_KIND, f"{what}: kind {kind_gpu} vs oracle {kind_oracle}, MSEs {ms!r} / {mt!r}"
    _log("head kind", f"{what}: {kind_gpu} vs {kind_oracle}, relative MSE gap {gap:.2e}")
    return True


def summary() -> str:
    if not NEAR_TIES:
        return "near-ties accepted: 0"
    parts = ", ".join(f"{k} {v}" for k, v in sorted(NEAR_TIES.items()))
    return f"near-ties accepted: {sum(NEAR_TIES.values())} ({parts})"
