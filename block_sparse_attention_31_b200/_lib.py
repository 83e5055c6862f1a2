"""ctypes binding of libvsa.so: one Python function per C entry point, same names.

Argument marshalling only -- every step of the attention path runs in the library's CUDA
kernels.  PyTorch provides device memory and streams.  There is no CPU fallback: if the
library cannot be loaded, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvsa.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "vsa.h")

VSA_OK, VSA_ERR_INVALID_ARG, VSA_ERR_UNSUPPORTED, VSA_ERR_WORKSPACE, VSA_ERR_CUDA, VSA_ERR_DEVICE, \
    VSA_ERR_TIMEOUT = range(7)
VSA_DEVERR_KV_RANGE, VSA_DEVERR_TIMEOUT, VSA_DEVERR_KIND, VSA_DEVERR_OVERFLOW = 0x1, 0x2, 0x4, 0x8
VSA_F32, VSA_BF16 = 0, 1
VSA_SPATIAL, VSA_TEMPORAL, VSA_CUBE = 0, 1, 2
VSA_SELECT_PROFILE, VSA_SELECT_GIVEN, VSA_SELECT_CUBE = 0, 1, 2


class VsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("F", ctypes.c_int), ("Hl", ctypes.c_int),
                ("Wl", ctypes.c_int), ("d", ctypes.c_int), ("block", ctypes.c_int), ("cube_f", ctypes.c_int),
                ("cube_h", ctypes.c_int), ("cube_w", ctypes.c_int)]


class Params(ctypes.Structure):
    _fields_ = [("w_s", ctypes.c_int), ("w_t", ctypes.c_int), ("profile_frac", ctypes.c_double),
                ("topk", ctypes.c_int), ("scale", ctypes.c_float), ("layout_in_kernel", ctypes.c_int),
                ("qk_fp8", ctypes.c_int)]


class SemParams(ctypes.Structure):
    _fields_ = [("cq", ctypes.c_int), ("ck", ctypes.c_int), ("iters", ctypes.c_int), ("top_p", ctypes.c_float),
                ("scale", ctypes.c_float)]


class HostBatch(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("o", ctypes.c_void_p)]


class QKVO(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("o", ctypes.c_void_p),
                ("lse", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libvsa.so is not built ({LIB_PATH}); run `python block_sparse_attention_31_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, vp, i32, i64, sz = ctypes.POINTER, ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    st = ctypes.c_int
    sig = {
        "vsa_status_string": (ctypes.c_char_p, [st]),
        "vsa_version": (i32, []),
        "vsa_layout_rows": (st, [P(Shape), P(i64)]),
        "vsa_num_blocks": (st, [P(Shape), P(i32)]),
        "vsa_pattern_window": (st, [P(Shape), i32, ctypes.c_double, P(i32), P(ctypes.c_double)]),
        "vsa_max_kv": (st, [P(Shape), P(Params), P(i32)]),
        "vsa_profile_rows": (st, [P(Shape), P(Params), P(i32)]),
        "vsa_profile_workspace_size": (sz, [P(Shape), P(Params)]),
        "vsa_mask_workspace_size": (sz, [P(Shape), P(Params)]),
        "vsa_attention_workspace_size": (sz, [P(Shape), P(Params), i32, i32]),
        "vsa_permute": (st, [vp, i32, vp, vp, P(Shape), vp, vp]),
        "vsa_unpermute": (st, [vp, vp, vp, i32, vp, vp, P(Shape), vp, vp]),
        "vsa_profile_heads": (st, [vp, vp, vp, P(Shape), P(Params), vp, vp, vp, sz, vp, vp]),
        "vsa_profile_static_scratch_bytes": (sz, []),
        "vsa_profile_heads_static": (st, [vp, vp, vp, P(Shape), P(Params), vp, vp, vp, vp]),
        "vsa_build_mask": (st, [vp, vp, vp, P(Shape), P(Params), vp, vp, vp, i32, vp, sz, vp, vp]),
        "vsa_block_order": (st, [vp, vp, vp, i32, P(Shape), vp, vp]),
        "vsa_sparse_attn_fwd": (st, [P(QKVO), P(QKVO), vp, vp, vp, i32, vp, P(Shape), ctypes.c_float, vp, vp]),
        "vsa_sparse_attn_fwd_natural": (st, [P(QKVO), vp, vp, vp, i32, vp, P(Shape), ctypes.c_float, vp, vp]),
        "vsa_quantize_fp8": (st, [vp, vp, vp, P(Shape), vp, vp, vp, vp]),
        "vsa_sparse_attn_fwd_fp8qk": (st, [P(QKVO), P(QKVO), vp, vp, vp, vp, vp, vp, vp, i32, vp, P(Shape),
                                           ctypes.c_float, vp, vp]),
        "vsa_attention": (st, [P(QKVO), i32, P(Shape), P(Params), i32, vp, vp, vp, sz, vp, vp]),
        "vsa_attention_host": (st, [P(HostBatch), i32, P(QKVO), i32, P(Shape), P(Params), i32, vp, vp, vp, sz, vp,
                                    vp, vp, vp]),
        "vsa_attention_workspace_layout": (st, [P(Shape), P(Params), i32, i32, P(sz), P(sz), P(sz), P(i32)]),
        "vsa_get_device_error": (st, [vp, vp, P(i32)]),
        "vsa_kmeans_workspace_size": (sz, [P(Shape), i32]),
        "vsa_kmeans": (st, [vp, P(Shape), i32, i32, vp, vp, vp, vp, vp, sz, vp, vp]),
        "vsa_semantic_mask_workspace_size": (sz, [P(Shape)]),
        "vsa_semantic_mask": (st, [vp, vp, vp, vp, i32, vp, vp, vp, vp, i32, P(Shape), ctypes.c_float,
                                   ctypes.c_float, vp, vp, vp, vp, i32, vp, sz, vp, vp]),
        "vsa_gather_rows": (st, [vp, vp, vp, P(Shape), vp, vp]),
        "vsa_scatter_rows": (st, [vp, vp, vp, vp, vp, P(Shape), vp, vp]),
        "vsa_semantic_workspace_size": (sz, [P(Shape), P(SemParams)]),
        "vsa_semantic_attention": (st, [P(QKVO), P(Shape), P(SemParams), vp, sz, vp, vp]),
        "vsa_selftest_exp2": (st, [vp, vp, vp, i32, vp]),
        "vsa_selftest_wait_timeout": (st, [vp, vp, vp]),
        "vsa_selftest_device_reset": (st, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def declared_symbols() -> list:
    """Names of every entry point declared in include/vsa.h."""
    with open(HEADER_PATH) as fh:
        text = fh.read()
    return sorted(set(re.findall(r"^VSA_API\s+[^;(]*?\b(vsa_\w+)\s*\(", text, flags=re.M)))


def status_string(status: int) -> str:
    return lib.vsa_status_string(status).decode()


def _check(status: int, where: str):
    if status != VSA_OK:
        raise VsaError(status, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(stream)


def make_shape(B, H, F, Hl, Wl, d, block, cube=None) -> Shape:
    cf, ch, cw = cube if cube else (0, 0, 0)
    return Shape(B, H, F, Hl, Wl, d, block, cf, ch, cw)


def make_params(w_s=0, w_t=0, profile_frac=0.01, topk=0, scale=0.0, layout_in_kernel=False, qk_fp8=False) -> Params:
    return Params(int(w_s), int(w_t), float(profile_frac), int(topk), float(scale), int(bool(layout_in_kernel)),
                  int(bool(qk_fp8)))


# ---------------------------------------------------------------------------------------
# planning helpers
# ---------------------------------------------------------------------------------------

def vsa_layout_rows(shape: Shape) -> int:
    out = ctypes.c_int64()
    _check(lib.vsa_layout_rows(ctypes.byref(shape), ctypes.byref(out)), "vsa_layout_rows")
    return out.value


def vsa_num_blocks(shape: Shape) -> int:
    out = ctypes.c_int()
    _check(lib.vsa_num_blocks(ctypes.byref(shape), ctypes.byref(out)), "vsa_num_blocks")
    return out.value


def vsa_pattern_window(shape: Shape, kind: int, target: float):
    w, kept = ctypes.c_int(), ctypes.c_double()
    _check(lib.vsa_pattern_window(ctypes.byref(shape), kind, float(target), ctypes.byref(w), ctypes.byref(kept)),
           "vsa_pattern_window")
    return w.value, kept.value


def vsa_max_kv(shape: Shape, params: Params) -> int:
    out = ctypes.c_int()
    _check(lib.vsa_max_kv(ctypes.byref(shape), ctypes.byref(params), ctypes.byref(out)), "vsa_max_kv")
    return out.value


def vsa_profile_rows(shape: Shape, params: Params) -> int:
    out = ctypes.c_int()
    _check(lib.vsa_profile_rows(ctypes.byref(shape), ctypes.byref(params), ctypes.byref(out)), "vsa_profile_rows")
    return out.value


def vsa_profile_workspace_size(shape: Shape, params: Params) -> int:
    return int(lib.vsa_profile_workspace_size(ctypes.byref(shape), ctypes.byref(params)))


def vsa_mask_workspace_size(shape: Shape, params: Params) -> int:
    return int(lib.vsa_mask_workspace_size(ctypes.byref(shape), ctypes.byref(params)))


def vsa_attention_workspace_size(shape: Shape, params: Params, dtype: int, select: int) -> int:
    return int(lib.vsa_attention_workspace_size(ctypes.byref(shape), ctypes.byref(params), dtype, select))


def vsa_attention_workspace_layout(shape: Shape, params: Params, dtype: int, select: int):
    ob, oi, oc, mk = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_int()
    _check(lib.vsa_attention_workspace_layout(ctypes.byref(shape), ctypes.byref(params), dtype, select,
                                              ctypes.byref(ob), ctypes.byref(oi), ctypes.byref(oc), ctypes.byref(mk)),
           "vsa_attention_workspace_layout")
    return ob.value, oi.value, oc.value, mk.value


# ---------------------------------------------------------------------------------------
# kernels
# ---------------------------------------------------------------------------------------

def vsa_permute(src, src_dtype, dst, kinds, shape: Shape, err, stream=None):
    _check(lib.vsa_permute(_ptr(src), src_dtype, _ptr(dst), _ptr(kinds), ctypes.byref(shape), _ptr(err),
                           _stream(stream)), "vsa_permute")


def vsa_unpermute(src, src_lse, dst, dst_dtype, dst_lse, kinds, shape: Shape, err, stream=None):
    _check(lib.vsa_unpermute(_ptr(src), _ptr(src_lse), _ptr(dst), dst_dtype, _ptr(dst_lse), _ptr(kinds),
                             ctypes.byref(shape), _ptr(err), _stream(stream)), "vsa_unpermute")


def vsa_profile_heads(q, k, v, shape: Shape, params: Params, kinds, mse, ws, ws_bytes, err, stream=None):
    _check(lib.vsa_profile_heads(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(shape), ctypes.byref(params), _ptr(kinds),
                                 _ptr(mse), _ptr(ws), int(ws_bytes), _ptr(err), _stream(stream)), "vsa_profile_heads")


def vsa_profile_static_scratch_bytes() -> int:
    return int(lib.vsa_profile_static_scratch_bytes())


def vsa_profile_heads_static(q, k, v, shape: Shape, params: Params, kinds, mse, err, stream=None):
    """vsa_profile_heads with the library's own fixed scratch (no workspace argument)."""
    _check(lib.vsa_profile_heads_static(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(shape), ctypes.byref(params),
                                        _ptr(kinds), _ptr(mse), _ptr(err), _stream(stream)),
           "vsa_profile_heads_static")


def vsa_build_mask(kinds, q_cube, k_cube, shape: Shape, params: Params, bits, kv_idx, kv_cnt, max_kv, ws, ws_bytes,
                   err, stream=None):
    _check(lib.vsa_build_mask(_ptr(kinds), _ptr(q_cube), _ptr(k_cube), ctypes.byref(shape), ctypes.byref(params),
                              _ptr(bits), _ptr(kv_idx), _ptr(kv_cnt), int(max_kv), _ptr(ws), int(ws_bytes), _ptr(err),
                              _stream(stream)), "vsa_build_mask")


def qkvo(q, k, v, o, lse=None) -> QKVO:
    return QKVO(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse))


def vsa_block_order(kinds, kv_idx, kv_cnt, max_kv, shape: Shape, order, stream=None):
    _check(lib.vsa_block_order(_ptr(kinds), _ptr(kv_idx), _ptr(kv_cnt), int(max_kv), ctypes.byref(shape),
                               _ptr(order), _stream(stream)), "vsa_block_order")


def vsa_sparse_attn_fwd(natural: QKVO, permuted, kinds, kv_idx, kv_cnt, max_kv, shape: Shape, scale, err,
                        stream=None, order=None):
    _check(lib.vsa_sparse_attn_fwd(ctypes.byref(natural), ctypes.byref(permuted) if permuted is not None else None,
                                   _ptr(kinds), _ptr(kv_idx), _ptr(kv_cnt), int(max_kv), _ptr(order),
                                   ctypes.byref(shape), float(scale), _ptr(err), _stream(stream)),
           "vsa_sparse_attn_fwd")


def vsa_quantize_fp8(natural, permuted, kinds, shape: Shape, dst, exps, err, stream=None):
    _check(lib.vsa_quantize_fp8(_ptr(natural), _ptr(permuted), _ptr(kinds), ctypes.byref(shape), _ptr(dst), _ptr(exps),
                                _ptr(err), _stream(stream)), "vsa_quantize_fp8")


def vsa_sparse_attn_fwd_fp8qk(natural: QKVO, permuted, q8, qexp, k8, kexp, kinds, kv_idx, kv_cnt, max_kv,
                              shape: Shape, scale, err, stream=None, order=None):
    _check(lib.vsa_sparse_attn_fwd_fp8qk(ctypes.byref(natural),
                                         ctypes.byref(permuted) if permuted is not None else None, _ptr(q8),
                                         _ptr(qexp), _ptr(k8), _ptr(kexp), _ptr(kinds), _ptr(kv_idx), _ptr(kv_cnt),
                                         int(max_kv), _ptr(order), ctypes.byref(shape), float(scale), _ptr(err),
                                         _stream(stream)), "vsa_sparse_attn_fwd_fp8qk")


def vsa_sparse_attn_fwd_natural(natural: QKVO, kinds, kv_idx, kv_cnt, max_kv, shape: Shape, scale, err, stream=None,
                                order=None):
    _check(lib.vsa_sparse_attn_fwd_natural(ctypes.byref(natural), _ptr(kinds), _ptr(kv_idx), _ptr(kv_cnt),
                                           int(max_kv), _ptr(order), ctypes.byref(shape), float(scale), _ptr(err),
                                           _stream(stream)), "vsa_sparse_attn_fwd_natural")


def vsa_attention_host(batches, sets, dtype: int, shape: Shape, params: Params, select: int, kinds, mse, ws,
                       ws_bytes, err, stream_up, stream_compute, stream_down):
    """batches: sequence of (q, k, v, o) host tensors (pinned); sets: two QKVO of device buffers."""
    arr = (HostBatch * len(batches))(*[HostBatch(_ptr(q), _ptr(k), _ptr(v), _ptr(o)) for q, k, v, o in batches])
    sarr = (QKVO * 2)(*sets)
    _check(lib.vsa_attention_host(arr, len(batches), sarr, dtype, ctypes.byref(shape), ctypes.byref(params), select,
                                  _ptr(kinds), _ptr(mse), _ptr(ws), int(ws_bytes), _ptr(err), _stream(stream_up),
                                  _stream(stream_compute), _stream(stream_down)), "vsa_attention_host")


def vsa_attention(io: QKVO, dtype: int, shape: Shape, params: Params, select: int, kinds, mse, ws, ws_bytes, err,
                  stream=None):
    _check(lib.vsa_attention(ctypes.byref(io), dtype, ctypes.byref(shape), ctypes.byref(params), select, _ptr(kinds),
                             _ptr(mse), _ptr(ws), int(ws_bytes), _ptr(err), _stream(stream)), "vsa_attention")


def vsa_get_device_error(err, stream=None) -> int:
    """Synchronises the stream and returns the device error word (0 when clean)."""
    h = ctypes.c_int()
    st = lib.vsa_get_device_error(_ptr(err), _stream(stream), ctypes.byref(h))
    if st not in (VSA_OK, VSA_ERR_DEVICE, VSA_ERR_TIMEOUT):
        raise VsaError(st, "vsa_get_device_error")
    return h.value


def vsa_selftest_exp2(x, y_poly, y_mufu, stream=None):
    _check(lib.vsa_selftest_exp2(_ptr(x), _ptr(y_poly), _ptr(y_mufu), int(x.numel()), _stream(stream)),
           "vsa_selftest_exp2")


def vsa_selftest_wait_timeout(err, waited, stream=None):
    _check(lib.vsa_selftest_wait_timeout(_ptr(err), _ptr(waited), _stream(stream)), "vsa_selftest_wait_timeout")


def vsa_selftest_device_reset():
    _check(lib.vsa_selftest_device_reset(), "vsa_selftest_device_reset")


# ---------------------------------------------------------------------------------------
# semantic-aware permutation
# ---------------------------------------------------------------------------------------

def make_sem_params(cq, ck, iters, top_p, scale=0.0) -> SemParams:
    return SemParams(int(cq), int(ck), int(iters), float(top_p), float(scale))


def vsa_kmeans_workspace_size(shape: Shape, n_clusters: int) -> int:
    return int(lib.vsa_kmeans_workspace_size(ctypes.byref(shape), int(n_clusters)))


def vsa_kmeans(x, shape: Shape, n_clusters, iters, centroids, labels, counts, perm, ws, ws_bytes, err, stream=None):
    _check(lib.vsa_kmeans(_ptr(x), ctypes.byref(shape), int(n_clusters), int(iters), _ptr(centroids), _ptr(labels),
                          _ptr(counts), _ptr(perm), _ptr(ws), int(ws_bytes), _ptr(err), _stream(stream)),
           "vsa_kmeans")


def vsa_semantic_mask_workspace_size(shape: Shape) -> int:
    return int(lib.vsa_semantic_mask_workspace_size(ctypes.byref(shape)))


def vsa_semantic_mask(cent_q, counts_q, labels_q, perm_q, cq, cent_k, counts_k, labels_k, perm_k, ck, shape: Shape,
                      top_p, scale, keep, bits, kv_idx, kv_cnt, max_kv, ws, ws_bytes, err, stream=None):
    _check(lib.vsa_semantic_mask(_ptr(cent_q), _ptr(counts_q), _ptr(labels_q), _ptr(perm_q), int(cq), _ptr(cent_k),
                                 _ptr(counts_k), _ptr(labels_k), _ptr(perm_k), int(ck), ctypes.byref(shape),
                                 float(top_p), float(scale), _ptr(keep), _ptr(bits), _ptr(kv_idx), _ptr(kv_cnt),
                                 int(max_kv), _ptr(ws), int(ws_bytes), _ptr(err), _stream(stream)),
           "vsa_semantic_mask")


def vsa_gather_rows(src, perm, dst, shape: Shape, err, stream=None):
    _check(lib.vsa_gather_rows(_ptr(src), _ptr(perm), _ptr(dst), ctypes.byref(shape), _ptr(err), _stream(stream)),
           "vsa_gather_rows")


def vsa_scatter_rows(src, src_lse, perm, dst, dst_lse, shape: Shape, err, stream=None):
    _check(lib.vsa_scatter_rows(_ptr(src), _ptr(src_lse), _ptr(perm), _ptr(dst), _ptr(dst_lse), ctypes.byref(shape),
                                _ptr(err), _stream(stream)), "vsa_scatter_rows")


def vsa_semantic_workspace_size(shape: Shape, params: SemParams) -> int:
    return int(lib.vsa_semantic_workspace_size(ctypes.byref(shape), ctypes.byref(params)))


def vsa_semantic_attention(io: QKVO, shape: Shape, params: SemParams, ws, ws_bytes, err, stream=None):
    _check(lib.vsa_semantic_attention(ctypes.byref(io), ctypes.byref(shape), ctypes.byref(params), _ptr(ws),
                                      int(ws_bytes), _ptr(err), _stream(stream)), "vsa_semantic_attention")
