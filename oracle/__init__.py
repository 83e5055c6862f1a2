"""fp64 CPU oracle for the spatial-temporal block-sparse attention path.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product package never imports
this module, and this module never imports the product package.

The arithmetic lives in ``vsa_oracle.c`` (plain C, fp64, OpenMP over rows); this file
only marshals numpy arrays in and out and converts the oracle's boolean block masks into
the list and bitset formats the GPU library emits, so that the two can be compared.
Each function names the passage of the pages it follows in the C source.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

SPATIAL, TEMPORAL, CUBE = 0, 1, 2

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "vsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-ffp-contract=off",
               _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i64, dbl, vp = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.or_num_cubes.restype = i64
        lib.or_num_cubes.argtypes = [i64] * 6
        lib.or_layout_rows.restype = i64
        lib.or_layout_rows.argtypes = [ctypes.c_int] + [i64] * 6
        lib.or_layout_slots.restype = None
        lib.or_layout_slots.argtypes = [ctypes.c_int] + [i64] * 6 + [vp]
        lib.or_pattern_keep.restype = None
        lib.or_pattern_keep.argtypes = [ctypes.c_int] + [i64] * 5 + [vp]
        lib.or_kept_fraction.restype = dbl
        lib.or_kept_fraction.argtypes = [ctypes.c_int] + [i64] * 5
        lib.or_window_for_target.restype = i64
        lib.or_window_for_target.argtypes = [ctypes.c_int] + [i64] * 4 + [dbl]
        lib.or_cube_topk_keep.restype = ctypes.c_int
        lib.or_cube_topk_keep.argtypes = [vp, vp] + [i64] * 8 + [vp, vp]
        lib.or_attention_rows.restype = None
        lib.or_attention_rows.argtypes = [vp, vp, vp, i64, i64, dbl, vp, i64, vp, i64, vp, i64, vp, vp]
        lib.or_attention_rows_qk.restype = None
        lib.or_attention_rows_qk.argtypes = [vp, vp, vp, i64, i64, dbl, vp, vp, i64, vp, i64, vp, i64, vp, vp]
        lib.or_kmeans_assign.restype = None
        lib.or_kmeans_assign.argtypes = [vp, i64, i64, vp, i64, vp, vp]
        lib.or_kmeans_update.restype = ctypes.c_int
        lib.or_kmeans_update.argtypes = [vp, i64, i64, vp, i64, vp, vp]
        lib.or_kmeans.restype = ctypes.c_int
        lib.or_kmeans.argtypes = [vp, i64, i64, i64, i64, vp, vp, vp]
        lib.or_cluster_perm.restype = None
        lib.or_cluster_perm.argtypes = [vp, i64, i64, vp, vp]
        lib.or_semantic_weights.restype = None
        lib.or_semantic_weights.argtypes = [vp, vp, i64, vp, vp, i64, i64, dbl, vp]
        lib.or_semantic_keep.restype = None
        lib.or_semantic_keep.argtypes = [vp, vp, i64, vp, vp, i64, i64, dbl, dbl, vp]
        lib.or_e4m3_value.restype = dbl
        lib.or_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.or_quantize_e4m3.restype = None
        lib.or_quantize_e4m3.argtypes = [vp, i64, i64, i64, vp, vp]
        lib.or_profile_rows.restype = i64
        lib.or_profile_rows.argtypes = [i64, dbl]
        lib.or_profile_head.restype = ctypes.c_int
        lib.or_profile_head.argtypes = [vp, vp, vp] + [i64] * 4 + [dbl] + [i64] * 3 + [dbl, vp, vp]
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f64(x) -> np.ndarray:
    """Widen a torch tensor or array to a C-contiguous fp64 numpy array."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def num_cubes(F, Hl, Wl, cube=(4, 4, 8)) -> int:
    return int(_load().or_num_cubes(F, Hl, Wl, *cube))


def layout_rows(kind, F, Hl, Wl, cube=(4, 4, 8)) -> int:
    return int(_load().or_layout_rows(kind, F, Hl, Wl, *cube))


def layout_slots(kind, F, Hl, Wl, cube=(4, 4, 8)) -> np.ndarray:
    """Slot of every natural token under a head's layout (int64 [N])."""
    out = np.empty(F * Hl * Wl, dtype=np.int64)
    _load().or_layout_slots(kind, F, Hl, Wl, *cube, _p(out))
    return out


def pattern_keep(kind, F, Hl, Wl, block, w) -> np.ndarray:
    """Boolean block mask [nblk, nblk] of a spatial or temporal head with window w."""
    nb = -(-(F * Hl * Wl) // block)
    out = np.empty((nb, nb), dtype=np.uint8)
    _load().or_pattern_keep(kind, F, Hl, Wl, block, w, _p(out))
    return out.astype(bool)


def kept_fraction(kind, F, Hl, Wl, block, w) -> float:
    return float(_load().or_kept_fraction(kind, F, Hl, Wl, block, w))


def window_for_target(kind, F, Hl, Wl, block, target) -> int:
    return int(_load().or_window_for_target(kind, F, Hl, Wl, block, float(target)))


def cube_topk_keep(q, k, F, Hl, Wl, topk, cube=(4, 4, 8), return_scores=False):
    """Cube mask [C, C] from pooled-QK^T top-k (one head, natural-order q, k [N, d])."""
    q, k = _f64(q), _f64(k)
    d = q.shape[-1]
    C = num_cubes(F, Hl, Wl, cube)
    keep = np.empty((C, C), dtype=np.uint8)
    score = np.empty((C, C), dtype=np.float64)
    rc = _load().or_cube_topk_keep(_p(q), _p(k), F, Hl, Wl, d, *cube, topk, _p(keep), _p(score))
    if rc != 0:
        raise MemoryError("oracle cube top-k allocation failed")
    return (keep.astype(bool), score) if return_scores else keep.astype(bool)


def attention_rows(q, k, v, slots, block, keep, rows=None, scale=None, kslots=None):
    """Masked softmax attention on natural-order rows of one head.

    ``slots`` maps tokens to slots of the queries' layout; ``kslots`` (default: the same)
    those of the keys' layout.  Returns (out [len(rows), d] fp64, lse [len(rows)] fp64,
    natural log).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    slots = np.ascontiguousarray(slots, dtype=np.int64)
    kslots = slots if kslots is None else np.ascontiguousarray(kslots, dtype=np.int64)
    keep8 = np.ascontiguousarray(keep, dtype=np.uint8)
    nb = keep8.shape[0]
    rows = np.arange(N, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    out = np.empty((len(rows), d), dtype=np.float64)
    lse = np.empty(len(rows), dtype=np.float64)
    _load().or_attention_rows_qk(_p(q), _p(k), _p(v), N, d, scale, _p(slots), _p(kslots), block, _p(keep8), nb,
                                 _p(rows), len(rows), _p(out), _p(lse))
    return out, lse


def profile_rows(N, frac) -> int:
    return int(_load().or_profile_rows(N, float(frac)))


def profile_head(q, k, v, F, Hl, Wl, block, w_s, w_t, frac=0.01, scale=None):
    """Profile one head: returns (kind, mse[2] = (spatial, temporal), sampled rows)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    r = profile_rows(N, frac)
    mse = np.empty(2, dtype=np.float64)
    rows = np.empty(r, dtype=np.int64)
    kind = _load().or_profile_head(_p(q), _p(k), _p(v), F, Hl, Wl, d, scale, block, w_s, w_t, float(frac),
                                   _p(mse), _p(rows))
    if kind < 0:
        raise MemoryError("oracle profiling allocation failed")
    return int(kind), mse, rows


# ---------------------------------------------------------------------------------------
# Semantic-aware permutation (Sparse VideoGen2 page, abstract); the readings are stated in
# vsa_oracle.c next to the C functions.
# ---------------------------------------------------------------------------------------

def _f32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def kmeans(x, C: int, iters: int):
    """k-means of one head's rows x [N, d]: (centroids [C, d] fp32, labels [N], counts [C])."""
    x = _f32(x)
    N, d = x.shape
    cent = np.empty((C, d), dtype=np.float32)
    label = np.empty(N, dtype=np.int32)
    count = np.empty(C, dtype=np.int32)
    if _load().or_kmeans(_p(x), N, d, C, iters, _p(cent), _p(label), _p(count)) != 0:
        raise ValueError("oracle k-means: bad arguments or allocation failure")
    return cent, label, count


def kmeans_assign(x, cent):
    """One assignment step: (labels [N] of the nearest centroid by fp64 squared distance, ties
    to the smaller index; gap [N] = second-nearest minus nearest distance)."""
    x, cent = _f32(x), _f32(cent)
    N, d = x.shape
    label = np.empty(N, dtype=np.int32)
    gap = np.empty(N, dtype=np.float64)
    _load().or_kmeans_assign(_p(x), N, d, _p(cent), cent.shape[0], _p(label), _p(gap))
    return label, gap


def kmeans_update(x, label, prev_cent):
    """One update step from given labels: (centroids [C, d] fp32, counts [C]); an empty
    cluster keeps its row of ``prev_cent``."""
    x = _f32(x)
    N, d = x.shape
    cent = np.array(_f32(prev_cent), copy=True)
    label = np.ascontiguousarray(label, dtype=np.int32)
    count = np.empty(cent.shape[0], dtype=np.int32)
    if _load().or_kmeans_update(_p(x), N, d, _p(label), cent.shape[0], _p(cent), _p(count)) != 0:
        raise MemoryError("oracle k-means update allocation failed")
    return cent, count


def kmeans_init(x, C: int):
    """Initial centroids: the rows floor((2j+1)N/(2C)) of x."""
    x = _f32(x)
    N = x.shape[0]
    rows = [((2 * j + 1) * N) // (2 * C) for j in range(C)]
    return np.ascontiguousarray(x[rows])


def cluster_perm(label, C: int):
    """Cluster-major order: (perm [N] slot -> token, offset [C + 1])."""
    label = np.ascontiguousarray(label, dtype=np.int32)
    perm = np.empty(label.size, dtype=np.int32)
    offset = np.empty(C + 1, dtype=np.int32)
    _load().or_cluster_perm(_p(label), label.size, C, _p(perm), _p(offset))
    return perm, offset


def semantic_keep(cq, nq, ck, nk, scale: float, top_p: float) -> np.ndarray:
    """Kept key clusters per query cluster: bool [Cq, Ck]."""
    cq, ck = _f32(cq), _f32(ck)
    nq = np.ascontiguousarray(nq, dtype=np.int32)
    nk = np.ascontiguousarray(nk, dtype=np.int32)
    Cq, d = cq.shape
    Ck = ck.shape[0]
    keep = np.empty((Cq, Ck), dtype=np.uint8)
    _load().or_semantic_keep(_p(cq), _p(nq), Cq, _p(ck), _p(nk), Ck, d, float(scale), float(top_p), _p(keep))
    return keep.astype(bool)


def semantic_weights(cq, nq, ck, nk, scale: float) -> np.ndarray:
    """Criticality weights [Cq, Ck] (fp64): n_j exp(s_ij - max_j s_ij); -1 where a cluster is
    empty."""
    cq, ck = _f32(cq), _f32(ck)
    nq = np.ascontiguousarray(nq, dtype=np.int32)
    nk = np.ascontiguousarray(nk, dtype=np.int32)
    Cq, d = cq.shape
    Ck = ck.shape[0]
    w = np.empty((Cq, Ck), dtype=np.float64)
    _load().or_semantic_weights(_p(cq), _p(nq), Cq, _p(ck), _p(nk), Ck, d, float(scale), _p(w))
    return w


def semantic_block_keep(label_q, perm_q, label_k, perm_k, keep, block: int) -> np.ndarray:
    """Block mask [nb, nb] over the two cluster-major layouts: block a of the queries and
    block b of the keys are kept when a kept cluster pair joins one of a's slots to one of
    b's slots."""
    lq = np.asarray(label_q)[np.asarray(perm_q)]        # cluster of each query slot
    lk = np.asarray(label_k)[np.asarray(perm_k)]
    N = lq.size
    nb = -(-N // block)
    keep = np.asarray(keep, dtype=bool)
    out = np.zeros((nb, nb), dtype=bool)
    for a in range(nb):
        qs = np.unique(lq[a * block:(a + 1) * block])
        row = keep[qs].any(axis=0)                      # key clusters reached from block a
        for b in range(nb):
            out[a, b] = row[np.unique(lk[b * block:(b + 1) * block])].any()
    return out


def semantic_scale(d: int, scale: float = 0.0) -> float:
    """Softmax scale of the criticality scores: the given one, else 1/sqrt(d) in fp64."""
    return float(scale) if scale > 0 else 1.0 / math.sqrt(d)


def semantic_head(q, k, v, cq: int, ck: int, iters: int, top_p: float, block: int, rows=None, scale: float = 0.0,
                  attention: bool = True):
    """The whole semantic path for one head (natural-order q, k, v [N, d]).

    Returns a dict with the k-means results of Q and K, both permutations, the cluster and
    block masks and, when ``attention``, the output rows (fp64) and their LSE.
    """
    d = q.shape[-1]
    cent_q, lab_q, cnt_q = kmeans(q, cq, iters)
    cent_k, lab_k, cnt_k = kmeans(k, ck, iters)
    perm_q, _ = cluster_perm(lab_q, cq)
    perm_k, _ = cluster_perm(lab_k, ck)
    sc = semantic_scale(d, scale)
    keep_c = semantic_keep(cent_q, cnt_q, cent_k, cnt_k, sc, top_p)
    keep_b = semantic_block_keep(lab_q, perm_q, lab_k, perm_k, keep_c, block)
    res = dict(cent_q=cent_q, label_q=lab_q, count_q=cnt_q, perm_q=perm_q, cent_k=cent_k, label_k=lab_k,
               count_k=cnt_k, perm_k=perm_k, keep_clusters=keep_c, keep_blocks=keep_b)
    if attention:
        N = lab_q.size
        qslot = np.empty(N, dtype=np.int64)
        qslot[perm_q] = np.arange(N)
        kslot = np.empty(N, dtype=np.int64)
        kslot[perm_k] = np.arange(N)
        out, lse = attention_rows(q, k, v, qslot, block, keep_b, rows=rows, kslots=kslot,
                                  scale=None if scale <= 0 else scale)
        res.update(out=out, lse=lse)
    return res


# ---------------------------------------------------------------------------------------
# FP8 Q and K (Sparse Video-Gen summary page, "Measured effects": FP8 quantisation); the
# readings are stated in vsa_oracle.c.
# ---------------------------------------------------------------------------------------

def quantize_e4m3(x, block: int):
    """Per-block e4m3 quantisation of one head's rows x [rows, d]: (codes uint8 [rows, d],
    scale exponents int32 [ceil(rows / block)])."""
    x = _f64(x)
    rows, d = x.shape
    code = np.empty((rows, d), dtype=np.uint8)
    exp = np.empty(-(-rows // block), dtype=np.int32)
    _load().or_quantize_e4m3(_p(x), rows, d, block, _p(code), _p(exp))
    return code, exp


_E4M3_TABLE = None


def e4m3_values(code) -> np.ndarray:
    """fp64 values of e4m3 codes."""
    global _E4M3_TABLE
    if _E4M3_TABLE is None:
        lib = _load()
        _E4M3_TABLE = np.array([lib.or_e4m3_value(c) for c in range(256)], dtype=np.float64)
    return _E4M3_TABLE[np.asarray(code, dtype=np.uint8)]


def dequantize_e4m3(code, exp, block: int) -> np.ndarray:
    """The values the codes stand for: e4m3(code) * 2^e of the row's block."""
    v = e4m3_values(code)
    rows = v.shape[0]
    e = np.repeat(np.asarray(exp, dtype=np.int64), block)[:rows]
    return np.ldexp(v, e[:, None])


# ---------------------------------------------------------------------------------------
# Format conversion of an oracle mask into the GPU library's output formats.
# ---------------------------------------------------------------------------------------

def keep_to_lists(keep: np.ndarray, max_kv: int):
    """Ascending kept-column list per row, padded with -1, and the per-row count."""
    nq = keep.shape[0]
    idx = np.full((nq, max_kv), -1, dtype=np.int32)
    cnt = np.zeros(nq, dtype=np.int32)
    for i in range(nq):
        cols = np.nonzero(keep[i])[0]
        cnt[i] = len(cols)
        idx[i, :min(len(cols), max_kv)] = cols[:max_kv]
    return idx, cnt


def keep_to_bits(keep: np.ndarray) -> np.ndarray:
    """Bitset [nq, ceil(nk/32)] uint32, bit (j % 32) of word j // 32 set when kept."""
    nq, nk = keep.shape
    nw = -(-nk // 32)
    padded = np.zeros((nq, nw * 32), dtype=np.uint64)
    padded[:, :nk] = keep
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    words = (padded.reshape(nq, nw, 32) * weights).sum(axis=2)
    return words.astype(np.uint32)
