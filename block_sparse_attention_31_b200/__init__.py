"""Spatial-temporal block-sparse self-attention for video diffusion transformers on B200.

The compute lives in ``libvsa.so`` (hand-written CUDA for sm_100a behind the C ABI in
``include/vsa.h``).  This package is its thin Python binding: ``_lib`` mirrors each C entry
point under the same name, and :class:`SparseAttention` owns the device buffers (from
PyTorch) of one configured call and invokes ``vsa_attention`` (``vsa_attention_host`` for
host batches).
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import _lib
from ._lib import (VSA_BF16, VSA_CUBE, VSA_F32, VSA_SELECT_CUBE, VSA_SELECT_GIVEN, VSA_SELECT_PROFILE, VSA_SPATIAL,
                   VSA_TEMPORAL, Params, QKVO, Shape, VsaError, make_params, make_shape, qkvo, vsa_attention,
                   vsa_attention_workspace_layout, vsa_attention_workspace_size, vsa_block_order,
                   vsa_build_mask, vsa_get_device_error, vsa_layout_rows, vsa_mask_workspace_size, vsa_max_kv, vsa_num_blocks,
                   vsa_pattern_window, vsa_permute, vsa_profile_heads, vsa_profile_rows, vsa_profile_workspace_size,
                   vsa_sparse_attn_fwd, vsa_sparse_attn_fwd_natural, vsa_unpermute, SemParams, make_sem_params,
                   vsa_quantize_fp8, vsa_sparse_attn_fwd_fp8qk,
                   vsa_gather_rows, vsa_kmeans, vsa_kmeans_workspace_size, vsa_scatter_rows, vsa_semantic_attention,
                   vsa_semantic_mask, vsa_semantic_mask_workspace_size, vsa_semantic_workspace_size)

_SELECT = {"profile": VSA_SELECT_PROFILE, "given": VSA_SELECT_GIVEN, "cube": VSA_SELECT_CUBE}
_DTYPE = {torch.float32: VSA_F32, torch.bfloat16: VSA_BF16}


class _HostPipelined:
    """run_host for a configured call: subclasses provide __call__(q, k, v, out=, kinds=, stream=)
    and the attributes B, H, N, d, dtype and device."""

    def run_host(self, batches, outs=None, kinds: Optional[torch.Tensor] = None, timing=None):
        """Run the call on a sequence of host batches with the transfers overlapped: while call i
        computes, the inputs of call i+1 upload and the output of call i-1 downloads (three
        streams, two device buffer sets).  ``batches`` is a list of (q, k, v) CPU tensors, which
        must be pinned for the copies to overlap; ``outs`` is a list of CPU output tensors
        (pinned ones are allocated when None).  Returns ``outs`` once every output has arrived.
        The log-sum-exp, when configured, stays on the device and is not returned.  ``timing``, a
        pair of timing-enabled CUDA events, is recorded before the first upload and after the
        last download."""
        n = len(batches)
        shape = (self.B, self.H, self.N, self.d)
        if outs is None:
            outs = [torch.empty(shape, dtype=self.dtype).pin_memory() for _ in range(n)]
        if len(outs) != n:
            raise ValueError("need one output tensor per batch")
        for (q, k, v), o in zip(batches, outs):
            for t in (q, k, v, o):
                if t.device.type != "cpu" or t.dtype != self.dtype or tuple(t.shape) != shape:
                    raise ValueError(f"host tensors of shape {shape} and dtype {self.dtype} expected")
        if not hasattr(self, "_host_bufs"):
            self._host_bufs = [[torch.empty(shape, dtype=self.dtype, device=self.device) for _ in range(4)]
                               for _ in range(2)]  # q, k, v, o per buffer set
            self._streams = [torch.cuda.Stream(self.device) for _ in range(3)]  # upload, compute, download
        up, comp, down = self._streams
        ev = lambda: torch.cuda.Event()  # noqa: E731
        up_done, comp_done, down_done = [], [], []
        up.wait_stream(torch.cuda.current_stream(self.device))
        if timing is not None:
            timing[0].record(up)
        for i, ((q, k, v), o) in enumerate(zip(batches, outs)):
            dq, dk, dv, do = self._host_bufs[i % 2]
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(comp_done[i - 2])  # call i-2 has read this buffer set
                dq.copy_(q, non_blocking=True)
                dk.copy_(k, non_blocking=True)
                dv.copy_(v, non_blocking=True)
                up_done.append(ev())
                up_done[i].record(up)
            with torch.cuda.stream(comp):
                comp.wait_event(up_done[i])
                if i >= 2:
                    comp.wait_event(down_done[i - 2])  # call i-2's output has left this buffer
                self(dq, dk, dv, out=do, kinds=kinds, stream=comp)
                comp_done.append(ev())
                comp_done[i].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(comp_done[i])
                o.copy_(do, non_blocking=True)
                down_done.append(ev())
                down_done[i].record(down)
        if timing is not None:
            timing[1].record(down)
        down.synchronize()
        return outs



class SparseAttention(_HostPipelined):
    """One configured attention call over a B x H x (F x Hl x Wl) x d problem.

    select:  "profile" (heads pick spatial/temporal by online profiling), "given" (kinds
             passed per call) or "cube" (own cube + top-k pooled cubes for every head).
    Windows: pass ``w_s``/``w_t`` directly, or ``target`` (a kept-block fraction) to use the
             smallest windows reaching it.
    layout_in_kernel: temporal heads are gathered through the frame-major map inside the
             attention kernel instead of being permuted into copies (bf16, no cube dims).
    qk_fp8:  Q.K^T on e4m3 codes with one power-of-two scale per block; P.V stays bf16
             (bf16, d = 128, block 128).
    """

    def __init__(self, B: int, H: int, F: int, Hl: int, Wl: int, d: int, block: int = 128, *,
                 dtype: torch.dtype = torch.bfloat16, select: str = "profile", w_s: Optional[int] = None,
                 w_t: Optional[int] = None, target: Optional[float] = None, topk: int = 0,
                 cube: Optional[Sequence[int]] = None, profile_frac: float = 0.01, scale: float = 0.0,
                 with_lse: bool = False, layout_in_kernel: bool = False, qk_fp8: bool = False, device="cuda"):
        if dtype not in _DTYPE:
            raise ValueError(f"unsupported dtype {dtype}")
        self.B, self.H, self.F, self.Hl, self.Wl, self.d, self.block = B, H, F, Hl, Wl, d, block
        self.N = F * Hl * Wl
        dev = torch.device(device)
        if dev.type == "cuda" and dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.dtype, self.select, self.device = dtype, _SELECT[select], dev
        self.shape = make_shape(B, H, F, Hl, Wl, d, block, tuple(cube) if cube else None)
        if target is not None:
            w_s_t, self.kept_s = vsa_pattern_window(self.shape, VSA_SPATIAL, target)
            w_t_t, self.kept_t = vsa_pattern_window(self.shape, VSA_TEMPORAL, target)
            w_s = w_s_t if w_s is None else w_s
            w_t = w_t_t if w_t is None else w_t
        self.w_s, self.w_t = int(w_s or 0), int(w_t or 0)
        self.params = make_params(self.w_s, self.w_t, profile_frac, topk, scale, layout_in_kernel, qk_fp8)
        self.ws_bytes = vsa_attention_workspace_size(self.shape, self.params, _DTYPE[dtype], self.select)
        if self.ws_bytes == 0:
            raise VsaError(_lib.VSA_ERR_INVALID_ARG, "vsa_attention_workspace_size")
        off_bits, off_idx, off_cnt, self.max_kv = vsa_attention_workspace_layout(self.shape, self.params,
                                                                                 _DTYPE[dtype], self.select)
        self.nblk = vsa_num_blocks(self.shape)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.device)
        nwords = (self.nblk + 31) // 32
        rows = B * H * self.nblk
        self.bits = self.ws[off_bits:off_bits + rows * nwords * 4].view(torch.int32).view(B, H, self.nblk, nwords)
        self.kv_idx = self.ws[off_idx:off_idx + rows * self.max_kv * 4].view(torch.int32).view(B, H, self.nblk,
                                                                                               self.max_kv)
        self.kv_cnt = self.ws[off_cnt:off_cnt + rows * 4].view(torch.int32).view(B, H, self.nblk)
        self.kinds = torch.zeros(B * H, dtype=torch.uint8, device=self.device)
        self.mse = torch.zeros(B * H * 2, dtype=torch.float32, device=self.device)
        self.err = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.with_lse = with_lse

    def __call__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None, kinds: Optional[torch.Tensor] = None, stream=None):
        for t in (q, k, v):
            if t.dtype != self.dtype or t.device != self.device or not t.is_contiguous():
                raise ValueError("q, k, v must be contiguous tensors of the configured dtype and device")
            if tuple(t.shape) != (self.B, self.H, self.N, self.d):
                raise ValueError(f"expected shape {(self.B, self.H, self.N, self.d)}, got {tuple(t.shape)}")
        if out is None:
            out = torch.empty_like(q)
        if self.with_lse and lse is None:
            lse = torch.empty(self.B, self.H, self.N, dtype=torch.float32, device=self.device)
        if self.select == VSA_SELECT_GIVEN:
            if kinds is None:
                raise ValueError("select='given' needs kinds")
            self.kinds.copy_(kinds.reshape(-1).to(torch.uint8))
        vsa_attention(qkvo(q, k, v, out, lse), _DTYPE[self.dtype], self.shape, self.params, self.select, self.kinds,
                      self.mse, self.ws, self.ws_bytes, self.err, stream)
        return (out, lse) if self.with_lse else out

    def device_error(self) -> int:
        return vsa_get_device_error(self.err)

    def clear_error(self):
        self.err.zero_()

    def run_host(self, batches, outs=None, kinds: Optional[torch.Tensor] = None, timing=None):
        """The call on a sequence of host batches through the library's vsa_attention_host: the
        uploads of batch i+1 and the download of batch i-1 overlap the compute of batch i (three
        streams, two device buffer sets owned here).  ``batches`` is a list of (q, k, v) CPU
        tensors, which must be pinned for the copies to overlap; ``outs`` a list of CPU output
        tensors (pinned ones are allocated when None).  Returns ``outs`` once every output has
        arrived.  ``timing``, a pair of timing-enabled CUDA events, is recorded before the first
        upload and after the last download."""
        n = len(batches)
        shape = (self.B, self.H, self.N, self.d)
        if outs is None:
            outs = [torch.empty(shape, dtype=self.dtype).pin_memory() for _ in range(n)]
        if len(outs) != n:
            raise ValueError("need one output tensor per batch")
        for (q, k, v), o in zip(batches, outs):
            for t in (q, k, v, o):
                if t.device.type != "cpu" or t.dtype != self.dtype or tuple(t.shape) != shape or not t.is_contiguous():
                    raise ValueError(f"contiguous host tensors of shape {shape} and dtype {self.dtype} expected")
        if self.select == VSA_SELECT_GIVEN:
            if kinds is None:
                raise ValueError("select='given' needs kinds")
            self.kinds.copy_(kinds.reshape(-1).to(torch.uint8))
        if not hasattr(self, "_host_bufs"):
            self._host_bufs = [[torch.empty(shape, dtype=self.dtype, device=self.device) for _ in range(4)]
                               for _ in range(2)]  # q, k, v, o per buffer set
            self._host_lse = ([torch.empty(self.B, self.H, self.N, dtype=torch.float32, device=self.device)
                               for _ in range(2)] if self.with_lse else [None, None])
            self._streams = [torch.cuda.Stream(self.device) for _ in range(3)]  # upload, compute, download
        up, comp, down = self._streams
        cur = torch.cuda.current_stream(self.device)
        up.wait_stream(cur)
        comp.wait_stream(cur)
        if timing is not None:
            timing[0].record(up)
        sets = [qkvo(b[0], b[1], b[2], b[3], lse) for b, lse in zip(self._host_bufs, self._host_lse)]
        _lib.vsa_attention_host([(q, k, v, o) for (q, k, v), o in zip(batches, outs)], sets, _DTYPE[self.dtype],
                                self.shape, self.params, self.select, self.kinds, self.mse, self.ws, self.ws_bytes,
                                self.err, up, comp, down)
        if timing is not None:
            timing[1].record(down)
        down.synchronize()
        return outs


class SemanticAttention(_HostPipelined):
    """Block-sparse attention with the semantic-aware permutation (Sparse VideoGen2 page,
    abstract): per-head k-means of Q (``cq`` clusters) and K (``ck``), cluster-major orders,
    a ``top_p`` budget over cluster pairs, then the same attention kernel.  bf16 only, no
    cube dims."""

    def __init__(self, B: int, H: int, F: int, Hl: int, Wl: int, d: int, block: int = 128, *, cq: int = 128,
                 ck: int = 128, iters: int = 4, top_p: float = 0.6, scale: float = 0.0, with_lse: bool = False,
                 device="cuda"):
        self.B, self.H, self.F, self.Hl, self.Wl, self.d, self.block = B, H, F, Hl, Wl, d, block
        self.N = F * Hl * Wl
        dev = torch.device(device)
        if dev.type == "cuda" and dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.device, self.dtype = dev, torch.bfloat16
        self.shape = make_shape(B, H, F, Hl, Wl, d, block)
        self.params = make_sem_params(cq, ck, iters, top_p, scale)
        self.ws_bytes = vsa_semantic_workspace_size(self.shape, self.params)
        if self.ws_bytes == 0:
            raise VsaError(_lib.VSA_ERR_INVALID_ARG, "vsa_semantic_workspace_size")
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.device)
        self.err = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.with_lse = with_lse

    def __call__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None, kinds=None, stream=None):
        if kinds is not None:
            raise ValueError("the semantic call chooses its blocks itself; kinds must be None")
        for t in (q, k, v):
            if t.dtype != torch.bfloat16 or t.device != self.device or not t.is_contiguous():
                raise ValueError("q, k, v must be contiguous bf16 tensors on the configured device")
            if tuple(t.shape) != (self.B, self.H, self.N, self.d):
                raise ValueError(f"expected shape {(self.B, self.H, self.N, self.d)}, got {tuple(t.shape)}")
        if out is None:
            out = torch.empty_like(q)
        if self.with_lse and lse is None:
            lse = torch.empty(self.B, self.H, self.N, dtype=torch.float32, device=self.device)
        vsa_semantic_attention(qkvo(q, k, v, out, lse), self.shape, self.params, self.ws, self.ws_bytes, self.err,
                               stream)
        return (out, lse) if self.with_lse else out

    def device_error(self) -> int:
        return vsa_get_device_error(self.err)


def attention(q, k, v, F: int, Hl: int, Wl: int, **kw):
    """Convenience wrapper: build a :class:`SparseAttention` for q's shape and run it once."""
    B, H, N, d = q.shape
    plan = SparseAttention(B, H, F, Hl, Wl, d, dtype=q.dtype, device=q.device, **kw)
    return plan(q, k, v)


__all__ = ["SparseAttention", "SemanticAttention", "attention", "SemParams", "make_sem_params", "vsa_gather_rows",
           "vsa_kmeans", "vsa_kmeans_workspace_size", "vsa_scatter_rows", "vsa_semantic_attention",
           "vsa_semantic_mask", "vsa_semantic_mask_workspace_size", "vsa_semantic_workspace_size", "VsaError", "Shape", "Params", "QKVO", "make_shape", "make_params", "qkvo",
           "vsa_attention", "vsa_attention_workspace_layout", "vsa_attention_workspace_size", "vsa_block_order", "vsa_build_mask",
           "vsa_get_device_error", "vsa_layout_rows", "vsa_mask_workspace_size", "vsa_max_kv", "vsa_num_blocks",
           "vsa_pattern_window", "vsa_permute", "vsa_profile_heads", "vsa_profile_rows",
           "vsa_profile_workspace_size", "vsa_sparse_attn_fwd", "vsa_sparse_attn_fwd_natural", "vsa_unpermute",
           "vsa_quantize_fp8", "vsa_sparse_attn_fwd_fp8qk", "VSA_SPATIAL", "VSA_TEMPORAL",
           "VSA_CUBE", "VSA_F32", "VSA_BF16", "VSA_SELECT_PROFILE", "VSA_SELECT_GIVEN", "VSA_SELECT_CUBE"]
