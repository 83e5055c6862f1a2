"""Benchmark of one spatial-temporal block-sparse attention call on B200.

One step = the whole hot path on one batch of synthetic input resident in HBM:
profiling -> frame-major permutation of Q/K/V -> block masks -> block-sparse attention
-> un-permutation of O, each through its C-ABI entry point on one stream, with CUDA events
between the stages for the per-kernel timing.  The default workload is the Wan2.1-1.3B
latent grid of HunyuanVideo-720p (B1 H24 33x45x80, d 128, block 128, kept fraction 0.18,
profiled heads), the largest single-GPU workload by work and bytes.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config hunyuan|wan|wan6x|sweep0.35|...]
    python bench.py --impl reference ...   (the fp64 CPU oracle timed on host cores)

Multi-GPU (torchrun, one rank per GPU): every rank runs its own independent attention call
(weak scaling); the timed region is bracketed by barriers and the reported time is the
maximum over ranks.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

METRIC = "ms/attention call and effective TFLOP/s (sparse & dense-equiv) vs bf16 peak"
# DRAM bytes (read + write) per launch of the attention kernel from one ncu capture of the current
# kernel on that workload (profiles/ has the command and the figures); absent -> null.
TRAFFIC = {"hunyuanvideo-720p: B1 H24 33x45x80 d128 block128 bf16": 2217364736 + 712276736}

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------------------
# work accounting
# ---------------------------------------------------------------------------------------

def block_valid_counts(wl, kind, nblk):
    """Real tokens in each block of a head's layout."""
    if kind == synthetic.CUBE:
        cf, ch, cw = wl.cube
        ncf, nch, ncw = -(-wl.F // cf), -(-wl.Hl // ch), -(-wl.Wl // cw)
        out = np.zeros(nblk, dtype=np.int64)
        for c in range(min(nblk, ncf * nch * ncw)):
            a, b, e = c // (nch * ncw), (c // ncw) % nch, c % ncw
            out[c] = min(cf, wl.F - a * cf) * min(ch, wl.Hl - b * ch) * min(cw, wl.Wl - e * cw)
        return out
    out = np.zeros(nblk, dtype=np.int64)
    nb = -(-wl.N // wl.block)
    out[:nb] = np.minimum(wl.block, wl.N - np.arange(nb) * wl.block)
    return out


def attention_work(wl, kinds, kv_idx, kv_cnt):
    """(algorithmic flops, executed flops, kept block pairs) of the masks."""
    B, H = kv_cnt.shape[:2]
    nblk = kv_cnt.shape[2]
    alg = exe = 0.0
    pairs = 0
    for b in range(B):
        for h in range(H):
            kind = int(kinds[b * H + h])
            valid = block_valid_counts(wl, kind, nblk)
            cnt = kv_cnt[b, h]
            for i in np.nonzero(cnt)[0]:
                js = kv_idx[b, h, i, :cnt[i]]
                alg += 4.0 * wl.d * valid[i] * valid[js].sum()
                exe += 4.0 * wl.d * 128 * wl.block * cnt[i]
                pairs += int(cnt[i])
    return alg, exe, pairs


def kept_block_run(i, n, block, group, w):
    """Kept key blocks [lo, hi] of query block i under the window rule: block j spans groups
    [a_j, b_j] = [j*block // group, (min(n, (j+1)*block) - 1) // group] and is kept when the
    two spans are at most w groups apart."""
    nb = -(-n // block)
    j = np.arange(nb)
    a = (j * block) // group
    b = (np.minimum(n, (j + 1) * block) - 1) // group
    keep = np.maximum(0, np.maximum(a - b[i], a[i] - b)) <= w
    idx = np.nonzero(keep)[0]
    return int(idx[0]), int(idx[-1])


def profile_allowed_keys(wl, r, w_s, w_t):
    """Sum over the r sampled rows rho_i = floor((2i+1)N/(2r)) of the keys each pattern allows
    (spatial: natural blocks, group = frame; temporal: frame-major blocks, group = position)."""
    N, B, F, S = wl.N, wl.block, wl.F, wl.S
    total = 0
    for i in range(r):
        t = ((2 * i + 1) * N) // (2 * r)
        lo, hi = kept_block_run(t // B, N, B, S, w_s)
        total += min(N, (hi + 1) * B) - lo * B
        p = (t % S) * F + t // S  # frame-major slot
        lo, hi = kept_block_run(p // B, N, B, F, w_t)
        total += min(N, (hi + 1) * B) - lo * B
    return float(total)


def stage_work(wl, kinds, pipe, pairs):
    """Algorithmic bytes (HBM stages) or executed flops (profiling) per call of each stage,
    and the number of exponentials the attention evaluates."""
    from block_sparse_attention_31_b200 import _lib
    N, d, row = wl.N, wl.d, wl.d * 2
    if wl.mode == "semantic":
        BH = wl.B * wl.H
        nwords = -(-pipe.nblk // 32)
        cq, ck = wl.clusters
        out = {
            # k-means: per round one dot product per (row, centroid) pair (2*d flops) for Q and
            # K, on the tensor cores as two bf16 halves of each centroid (executed twice that);
            # the update, order and the rest are lower-order
            "profile": {"flops": BH * wl.kmeans_iters * 2.0 * d * N * (cq + ck), "bound": "tensor",
                        "executed_flops": BH * wl.kmeans_iters * 4.0 * d * N * (cq + ck)},
            "permute": {"bytes": BH * 3.0 * 2 * N * row, "bound": "hbm"},
            "mask": {"bytes": BH * pipe.nblk * (nwords + pipe.max_kv + 1) * 4.0, "bound": "hbm"},
            "unpermute": {"bytes": BH * 2.0 * N * row, "bound": "hbm"},
        }
        return out, float(pairs) * 128 * wl.block
    R = _lib.vsa_layout_rows(pipe.shape)
    n_t = sum(1 for k in kinds if k == _lib.VSA_TEMPORAL)
    n_c = sum(1 for k in kinds if k == _lib.VSA_CUBE)
    BH = wl.B * wl.H
    # permute: temporal heads read and write N rows; cube heads read N real rows and write every
    # one of the R slots (padding zeroed); spatial bf16 heads are read in place (no copy)
    n_tc = 0 if pipe.in_kernel else n_t  # temporal heads copied (not gathered in the kernel)
    perm = 3.0 * (n_tc * 2 * N + n_c * (N + R)) * row
    if getattr(pipe, "qk_fp8", False):  # e4m3 codes of Q and K: read bf16 rows, write one byte each
        perm += 2.0 * BH * R * (row + d)
    unperm = (n_tc + n_c) * 2.0 * N * row
    nwords = -(-pipe.nblk // 32)
    mask = BH * pipe.nblk * (nwords + pipe.max_kv + 1) * 4.0
    if wl.mode == "cube":
        C = R // (wl.cube[0] * wl.cube[1] * wl.cube[2])
        mask += n_c * (2.0 * R * row + 2.0 * 2 * C * d * 8 + 2.0 * C * C * 8)  # pool reads, means, scores w+r
    out = {"permute": {"bytes": perm, "bound": "hbm"}, "unpermute": {"bytes": unperm, "bound": "hbm"},
           "mask": {"bytes": mask, "bound": "hbm"}}
    if wl.mode == "profiled":
        r = _lib.vsa_profile_rows(pipe.shape, pipe.params)
        # algorithmic work of profiling: per head the dense part (Q.K^T and P.V over all N keys,
        # 4*d*r*N) plus one P.V per pattern over the keys that pattern allows each sampled row
        allowed = profile_allowed_keys(wl, r, pipe.params.w_s, pipe.params.w_t)
        alg = BH * (4.0 * d * r * N + 2.0 * d * allowed)
        # executed: Q.K^T once and three full-width P.V (the masked ones lane-masked)
        out["profile"] = {"flops": alg, "executed_flops": BH * 8.0 * d * r * N, "bound": "tensor", "rows": r,
                          "allowed_keys_per_head": allowed}
    exp2 = float(pairs) * 128 * wl.block
    return out, exp2


def stage_roofline(work, stage_ms, hbm_gbs, tensor_tflops):
    out = {}
    for name, w in work.items():
        t = stage_ms[name] / 1e3
        if t <= 0 or w.get("bytes", 1) == 0:
            continue
        if w["bound"] == "hbm":
            gbs = w["bytes"] / t / 1e9
            out[name] = {"bound": "hbm", "bytes": w["bytes"], "achieved": gbs, "peak": hbm_gbs, "unit": "GB/s",
                         "frac": gbs / hbm_gbs}
        else:
            tf = w["flops"] / t / 1e12
            out[name] = {"bound": "tensor", "flops": w["flops"], "achieved": tf, "peak": tensor_tflops,
                         "unit": "TFLOP/s", "frac": tf / tensor_tflops}
            if "executed_flops" in w:
                out[name]["executed_flops"] = w["executed_flops"]
                out[name]["executed_frac"] = w["executed_flops"] / t / 1e12 / tensor_tflops
    return out


# ---------------------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------------------

def gpu_smi_id(device_index: int) -> str:
    """nvidia-smi's name for a torch device: its PCI address (indices differ when
    CUDA_VISIBLE_DEVICES reorders or hides GPUs)."""
    try:
        p = torch.cuda.get_device_properties(device_index)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except (AttributeError, RuntimeError):
        return str(device_index)


class ClockSampler:
    """nvidia-smi clock samples, each stamped with the host time it arrived; only samples
    inside mark_start()..mark_stop() are summarised (the neighbours of the window when none
    fall inside it, flagged "window": "nearest")."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, smi_id: str, period_ms: int = 20):
        self.idx, self.period = smi_id, period_ms
        self.proc, self.samples, self.t0, self.t1 = None, [], None, None

    def _reader(self):
        for ln in self.proc.stdout:
            if ln.strip():
                self.samples.append((time.monotonic(), ln))

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", str(self.period)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        self.thread = threading.Thread(target=self._reader, daemon=True)
        self.thread.start()
        deadline = time.monotonic() + 5.0
        while not self.samples and time.monotonic() < deadline:  # sampler running before timing starts
            time.sleep(0.01)
        return self

    def mark_start(self):
        self.t0 = time.monotonic()

    def mark_stop(self):
        self.t1 = time.monotonic()
        time.sleep(2.0 * self.period / 1000.0)  # let the sample after the window arrive

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)

    def summary(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        rows = []
        for t, ln in self.samples:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((t, float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        window = "inside"
        if self.t0 is not None and self.t1 is not None:
            inside = [r for r in rows if self.t0 <= r[0] <= self.t1]
            if not inside and rows:  # region shorter than the sampling period
                before = [r for r in rows if r[0] < self.t0][-1:]
                after = [r for r in rows if r[0] > self.t1][:1]
                inside, window = before + after, "nearest"
            rows = inside
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        reasons = set()
        for r in rows:
            for n, v in zip(names, r[3]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median([r[1] for r in rows]), "sm_max_mhz": rows[-1][2],
                "reasons": sorted(reasons), "samples": len(rows), "window": window,
                "period_ms": self.period}


# ---------------------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------------------

class Pipeline:
    """Buffers for the stage-by-stage path through the public entry points."""

    def __init__(self, wl, device, in_kernel=False, qk_fp8=False):
        import block_sparse_attention_31_b200 as vsa
        from block_sparse_attention_31_b200 import _lib
        self.vsa, self.lib, self.wl, self.dev = vsa, _lib, wl, device
        self.qk_fp8 = bool(qk_fp8)
        self.in_kernel = bool(in_kernel) and wl.mode != "cube"  # cube heads always use their copies
        cube = wl.cube if wl.mode == "cube" else None
        self.shape = _lib.make_shape(wl.B, wl.H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block, cube)
        if wl.mode == "profiled":
            w_s, _ = _lib.vsa_pattern_window(self.shape, _lib.VSA_SPATIAL, wl.target)
            w_t, _ = _lib.vsa_pattern_window(self.shape, _lib.VSA_TEMPORAL, wl.target)
        else:
            w_s, w_t = wl.w_s or 0, wl.w_t or 0
        self.params = _lib.make_params(w_s, w_t, wl.profile_frac, wl.topk)
        self.R = _lib.vsa_layout_rows(self.shape)
        self.nblk = _lib.vsa_num_blocks(self.shape)
        self.max_kv = _lib.vsa_max_kv(self.shape, self.params)
        BH = wl.B * wl.H
        bf = torch.bfloat16
        self.qp, self.kp, self.vp, self.op = (torch.zeros(wl.B, wl.H, self.R, wl.d, dtype=bf, device=device)
                                              for _ in range(4))
        self.bits = torch.zeros(wl.B, wl.H, self.nblk, (self.nblk + 31) // 32, dtype=torch.int32, device=device)
        self.kv_idx = torch.zeros(wl.B, wl.H, self.nblk, self.max_kv, dtype=torch.int32, device=device)
        self.kv_cnt = torch.zeros(wl.B, wl.H, self.nblk, dtype=torch.int32, device=device)
        self.kinds = torch.zeros(BH, dtype=torch.uint8, device=device)
        if wl.mode == "fixed":
            self.kinds.copy_(torch.tensor(list(wl.fixed_kinds), dtype=torch.uint8))
        elif wl.mode == "cube":
            self.kinds.fill_(synthetic.CUBE)
        self.mse = torch.zeros(BH * 2, dtype=torch.float32, device=device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        self.prof_bytes = _lib.vsa_profile_workspace_size(self.shape, self.params) if wl.mode == "profiled" else 0
        self.mask_bytes = _lib.vsa_mask_workspace_size(self.shape, self.params)
        self.prof_ws = torch.empty(max(self.prof_bytes, 256), dtype=torch.uint8, device=device)
        self.mask_ws = torch.empty(max(self.mask_bytes, 256), dtype=torch.uint8, device=device)
        # work order for cube heads, as the whole call builds it
        self.order = (torch.empty(wl.B * wl.H * self.nblk, dtype=torch.int32, device=device)
                      if wl.mode == "cube" else None)
        cube = wl.mode == "cube"
        if self.qk_fp8:  # e4m3 codes of Q and K in every head's layout, one exponent per block
            self.q8 = torch.empty(wl.B, wl.H, self.R, wl.d, dtype=torch.uint8, device=device)
            self.k8 = torch.empty_like(self.q8)
            self.qe = torch.empty(BH, self.nblk, dtype=torch.int32, device=device)
            self.ke = torch.empty_like(self.qe)
        self.launches = ((2 if self.qk_fp8 else 0)                          # quantise Q and K
                         + (4 if wl.mode == "profiled" else 0)                 # prep, attn3, row error, reduce
                         + (0 if self.in_kernel else 6 if cube else 3)        # permutes
                         + (5 if cube else 1)                                 # masks (+ pool, score, top-k, order)
                         + 1                                                  # attention
                         + (0 if self.in_kernel else 2 if cube else 1))       # unpermute

    def step(self, q, k, v, o, ev=None):
        L, s = self.lib, None
        if ev is not None:
            ev[0].record()
        if self.wl.mode == "profiled":
            L.vsa_profile_heads(q, k, v, self.shape, self.params, self.kinds, self.mse, self.prof_ws, self.prof_bytes,
                                self.err, s)
        if ev is not None:
            ev[1].record()
        if not self.in_kernel:
            for src, dst in ((q, self.qp), (k, self.kp), (v, self.vp)):
                L.vsa_permute(src, L.VSA_BF16, dst, self.kinds, self.shape, self.err, s)
        if self.qk_fp8:  # the e4m3 codes of Q and K count with the layouts
            L.vsa_quantize_fp8(q, self.qp, self.kinds, self.shape, self.q8, self.qe, self.err, s)
            L.vsa_quantize_fp8(k, self.kp, self.kinds, self.shape, self.k8, self.ke, self.err, s)
        if ev is not None:
            ev[2].record()
        L.vsa_build_mask(self.kinds, self.qp, self.kp, self.shape, self.params, self.bits, self.kv_idx, self.kv_cnt,
                         self.max_kv, self.mask_ws, self.mask_bytes, self.err, s)
        if self.order is not None:
            L.vsa_block_order(self.kinds, self.kv_idx, self.kv_cnt, self.max_kv, self.shape, self.order, s)
        if ev is not None:
            ev[3].record()
        if self.qk_fp8:
            L.vsa_sparse_attn_fwd_fp8qk(L.qkvo(q, k, v, o), L.qkvo(self.qp, self.kp, self.vp, self.op), self.q8,
                                        self.qe, self.k8, self.ke, self.kinds, self.kv_idx, self.kv_cnt, self.max_kv,
                                        self.shape, 0.0, self.err, s, order=self.order)
        elif self.in_kernel:  # temporal heads gathered through the frame-major map inside the kernel
            L.vsa_sparse_attn_fwd_natural(L.qkvo(q, k, v, o), self.kinds, self.kv_idx, self.kv_cnt, self.max_kv,
                                          self.shape, 0.0, self.err, s)
        else:
            L.vsa_sparse_attn_fwd(L.qkvo(q, k, v, o), L.qkvo(self.qp, self.kp, self.vp, self.op), self.kinds,
                                  self.kv_idx, self.kv_cnt, self.max_kv, self.shape, 0.0, self.err, s, order=self.order)
        if ev is not None:
            ev[4].record()
        if not self.in_kernel:
            L.vsa_unpermute(self.op, None, o, L.VSA_BF16, None, self.kinds, self.shape, self.err, s)
        if ev is not None:
            ev[5].record()


class SemanticPipeline:
    """The semantic-permutation call (Sparse VideoGen2 page, abstract), stage by stage through
    the C ABI.  Its stages fill the same five timing slots: k-means of Q and K ("profile"),
    row gathers into the cluster-major orders ("permute"), the top-p cluster budget and block
    mask ("mask"), the attention, and the scatter of O back to token order ("unpermute")."""

    def __init__(self, wl, device):
        from block_sparse_attention_31_b200 import _lib
        self.lib, self.wl, self.in_kernel, self.order = _lib, wl, False, None
        self.shape = _lib.make_shape(wl.B, wl.H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block)
        self.cq, self.ck = wl.clusters
        self.params = _lib.make_sem_params(self.cq, self.ck, wl.kmeans_iters, wl.top_p)
        BH, N, d = wl.B * wl.H, wl.N, wl.d
        self.nblk = -(-N // wl.block)
        self.max_kv = self.nblk
        i32, f32, bf = torch.int32, torch.float32, torch.bfloat16
        self.cent = [torch.empty(BH, c, d, dtype=f32, device=device) for c in (self.cq, self.ck)]
        self.label = [torch.empty(BH, N, dtype=i32, device=device) for _ in range(2)]
        self.count = [torch.empty(BH, c, dtype=i32, device=device) for c in (self.cq, self.ck)]
        self.perm = [torch.empty(BH, N, dtype=i32, device=device) for _ in range(2)]
        self.qp, self.kp, self.vp, self.op = (torch.empty(wl.B, wl.H, N, d, dtype=bf, device=device)
                                              for _ in range(4))
        self.keep = torch.empty(BH, self.cq, -(-self.ck // 32), dtype=i32, device=device)
        self.bits = torch.zeros(wl.B, wl.H, self.nblk, -(-self.nblk // 32), dtype=i32, device=device)
        self.kv_idx = torch.zeros(wl.B, wl.H, self.nblk, self.max_kv, dtype=i32, device=device)
        self.kv_cnt = torch.zeros(wl.B, wl.H, self.nblk, dtype=i32, device=device)
        # every head is read from the permuted rows (the kernel's VSA_TEMPORAL addressing)
        self.kinds = torch.full((BH,), _lib.VSA_TEMPORAL, dtype=torch.uint8, device=device)
        self.km_bytes = _lib.vsa_kmeans_workspace_size(self.shape, max(self.cq, self.ck))
        self.km_ws = torch.empty(self.km_bytes, dtype=torch.uint8, device=device)
        self.mask_bytes = _lib.vsa_semantic_mask_workspace_size(self.shape)
        self.mask_ws = torch.empty(self.mask_bytes, dtype=torch.uint8, device=device)
        self.err = torch.zeros(1, dtype=i32, device=device)
        self.launches = (2 * (1 + 3 * wl.kmeans_iters)  # k-means: init, then assign, sort, update per round
                         + 3 + 4 + 1 + 1)               # gathers, mask (keep, 2 ranges, blocks), attention, scatter

    def step(self, q, k, v, o, ev=None):
        L, s, wl = self.lib, None, self.wl
        if ev is not None:
            ev[0].record()
        for j, (x, C) in enumerate(((q, self.cq), (k, self.ck))):
            L.vsa_kmeans(x, self.shape, C, wl.kmeans_iters, self.cent[j], self.label[j], self.count[j], self.perm[j],
                         self.km_ws, self.km_bytes, self.err, s)
        if ev is not None:
            ev[1].record()
        L.vsa_gather_rows(q, self.perm[0], self.qp, self.shape, self.err, s)
        L.vsa_gather_rows(k, self.perm[1], self.kp, self.shape, self.err, s)
        L.vsa_gather_rows(v, self.perm[1], self.vp, self.shape, self.err, s)
        if ev is not None:
            ev[2].record()
        L.vsa_semantic_mask(self.cent[0], self.count[0], self.label[0], self.perm[0], self.cq, self.cent[1],
                            self.count[1], self.label[1], self.perm[1], self.ck, self.shape, wl.top_p, 0.0,
                            self.keep, self.bits, self.kv_idx, self.kv_cnt, self.max_kv, self.mask_ws,
                            self.mask_bytes, self.err, s)
        if ev is not None:
            ev[3].record()
        L.vsa_sparse_attn_fwd(L.qkvo(q, k, v, o), L.qkvo(self.qp, self.kp, self.vp, self.op), self.kinds,
                              self.kv_idx, self.kv_cnt, self.max_kv, self.shape, 0.0, self.err, s)
        if ev is not None:
            ev[4].record()
        L.vsa_scatter_rows(self.op, None, self.perm[0], o, None, self.shape, self.err, s)
        if ev is not None:
            ev[5].record()


def make_pipeline(wl, device, in_kernel=False, qk_fp8=False):
    if wl.mode == "semantic":
        return SemanticPipeline(wl, device)
    return Pipeline(wl, device, in_kernel=in_kernel, qk_fp8=qk_fp8)


STAGES = ("profile", "permute", "mask", "attention", "unpermute")


def max_over_ranks(x: float, device) -> float:
    """Maximum of a per-rank scalar over the process group (identity without one)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Each rank runs its own independent problem (weak scaling)."""
    return base + rank


def aggregate_tflops(flops_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job throughput: the work of all ranks over the slowest rank's time."""
    return world * flops_per_rank / (ms_max / 1e3) / 1e12


def gpu_arm(args, wl, rank, world, device):
    torch.cuda.set_device(device)
    q, k, v = synthetic.make_qkv(wl, seed=rank_seed(wl.seed, rank))
    qd, kd, vd = q.to(device), k.to(device), v.to(device)
    o = torch.empty_like(qd)
    pipe = make_pipeline(wl, device, in_kernel=args.layout == "kernel", qk_fp8=args.qk == "fp8")
    for _ in range(args.warmup):
        pipe.step(qd, kd, vd, o)
    torch.cuda.synchronize()
    if pipe.lib.vsa_get_device_error(pipe.err) != 0:
        raise RuntimeError(f"device error word {pipe.lib.vsa_get_device_error(pipe.err)} after warm-up")
    # work accounting from the executed masks
    alg, exe, pairs = attention_work(wl, pipe.kinds.cpu().numpy(), pipe.kv_idx.cpu().numpy(),
                                     pipe.kv_cnt.cpu().numpy())
    dense = synthetic.dense_flops(wl)
    swork, exp2 = stage_work(wl, pipe.kinds.cpu().tolist(), pipe, pairs)
    nb = -(-wl.N // wl.block)
    kept_frac = pairs / (wl.B * wl.H * float(pipe.nblk if wl.mode == "cube" else nb) ** 2)
    # timed region
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(gpu_smi_id(torch.cuda.current_device())) as clk:
        clk.mark_start()
        start.record()
        for i in range(args.steps):
            pipe.step(qd, kd, vd, o, evs[i])
        stop.record()
        torch.cuda.synchronize()
        clk.mark_stop()
    if world > 1:
        torch.distributed.barrier()
    total_ms = start.elapsed_time(stop)
    stage_ms = {n: float(np.mean([e[j].elapsed_time(e[j + 1]) for e in evs])) for j, n in enumerate(STAGES)}
    if pipe.lib.vsa_get_device_error(pipe.err) != 0:
        raise RuntimeError("device error word set during the timed region")
    total_ms = max_over_ranks(total_ms, device)
    ms = total_ms / args.steps
    # end to end through the public API: pinned host inputs -> device -> vsa_attention -> host O
    e2e = e2e_arm(args, wl, q, k, v, device)
    e2e["ms_per_step"] = max_over_ranks(e2e["ms_per_step"], device)
    return dict(ms=ms, stage_ms=stage_ms, alg=alg, exe=exe, dense=dense, pairs=pairs, kept=kept_frac,
                swork=swork, exp2=exp2,
                clocks=clk.summary(), launches=pipe.launches, e2e=e2e, w_s=getattr(pipe.params, "w_s", None),
                w_t=getattr(pipe.params, "w_t", None),
                kinds=pipe.kinds.cpu().tolist())


def e2e_arm(args, wl, q, k, v, device):
    import block_sparse_attention_31_b200 as vsa
    if wl.mode == "semantic":
        plan = vsa.SemanticAttention(wl.B, wl.H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block, cq=wl.clusters[0],
                                     ck=wl.clusters[1], iters=wl.kmeans_iters, top_p=wl.top_p, device=device)
        return _e2e_run(args, plan, q, k, v, None, "SemanticAttention.run_host")
    select = {"profiled": "profile", "fixed": "given", "cube": "cube"}[wl.mode]
    kw = dict(select=select, dtype=q.dtype, device=device, layout_in_kernel=args.layout == "kernel",
              qk_fp8=args.qk == "fp8")
    if wl.mode == "profiled":
        kw.update(target=wl.target, profile_frac=wl.profile_frac)
    elif wl.mode == "cube":
        kw.update(cube=wl.cube, topk=wl.topk)
    else:
        kw.update(w_s=wl.w_s, w_t=wl.w_t)
    plan = vsa.SparseAttention(wl.B, wl.H, wl.F, wl.Hl, wl.Wl, wl.d, wl.block, **kw)
    kinds = torch.tensor(list(wl.fixed_kinds), dtype=torch.uint8, device=device) if wl.mode == "fixed" else None
    return _e2e_run(args, plan, q, k, v, kinds, "vsa_attention_host (C ABI, host batches) via SparseAttention.run_host")


def _e2e_run(args, plan, q, k, v, kinds, api):
    hq, hk, hv = q.pin_memory(), k.pin_memory(), v.pin_memory()
    steps = max(2, min(args.steps, 10))
    # every step uploads its Q, K, V from pinned host memory and downloads its O; the public
    # run_host overlaps the uploads of step i+1 and the download of step i-1 with step i
    batches = [(hq, hk, hv)] * steps
    outs = [torch.empty_like(hq).pin_memory() for _ in range(steps)]
    plan.run_host(batches[:2], outs[:2], kinds=kinds)  # warm-up
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    plan.run_host(batches, outs, kinds=kinds, timing=(a, b))
    torch.cuda.synchronize()
    if plan.device_error() != 0:
        raise RuntimeError("device error word set in the end-to-end run")
    bpe = hq.element_size()
    return {"ms_per_step": a.elapsed_time(b) / steps, "h2d_bytes_per_step": 3 * hq.numel() * bpe,
            "d2h_bytes_per_step": outs[0].numel() * bpe, "steps": steps,
            "api": f"{api} (uploads, compute and downloads of consecutive steps overlap)"}


# ---------------------------------------------------------------------------------------
# the CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------------------

def oracle_sample(wl, seconds: float, seed: int = 0):
    """Time the oracle on a bounded sample of the workload; returns (flops/s, description)."""
    import oracle
    t_begin = time.perf_counter()
    q, k, v = synthetic.make_qkv(wl, seed=seed, heads=[0, 1] if wl.H > 1 else [0])
    heads = q.shape[1]
    kinds, keeps, kslots = [], [], []
    t0 = time.perf_counter()
    for h in range(heads):
        if wl.mode == "semantic":
            res = oracle.semantic_head(q[0, h], k[0, h], None, wl.clusters[0], wl.clusters[1], wl.kmeans_iters,
                                       wl.top_p, wl.block, attention=False)
            qs, ks = np.empty(wl.N, dtype=np.int64), np.empty(wl.N, dtype=np.int64)
            qs[res["perm_q"]] = np.arange(wl.N)
            ks[res["perm_k"]] = np.arange(wl.N)
            kinds.append(qs)
            kslots.append(ks)
            keeps.append(res["keep_blocks"])
            continue
        kslots.append(None)
        if wl.mode == "cube":
            kinds.append(oracle.CUBE)
            keeps.append(oracle.cube_topk_keep(q[0, h], k[0, h], wl.F, wl.Hl, wl.Wl, wl.topk, wl.cube))
        else:
            if wl.mode == "profiled":
                w_s = oracle.window_for_target(oracle.SPATIAL, wl.F, wl.Hl, wl.Wl, wl.block, wl.target)
                w_t = oracle.window_for_target(oracle.TEMPORAL, wl.F, wl.Hl, wl.Wl, wl.block, wl.target)
                kind, _, _ = oracle.profile_head(q[0, h], k[0, h], v[0, h], wl.F, wl.Hl, wl.Wl, wl.block, w_s, w_t,
                                                 wl.profile_frac) if seconds > 60 else (h % 2, None, None)
            else:
                w_s, w_t, kind = wl.w_s, wl.w_t, wl.fixed_kinds[h]
            kinds.append(kind)
            keeps.append(oracle.pattern_keep(kind, wl.F, wl.Hl, wl.Wl, wl.block, w_s if kind == 0 else w_t))
    mask_s = time.perf_counter() - t0
    # attention rows: grow the sample until the time budget is used
    flops = 0.0
    spent = 0.0
    rows_done = 0
    n = 8
    rng = np.random.default_rng(seed)
    while spent < seconds:
        for h in range(heads):
            # semantic heads: kinds[h] holds the query slots, kslots[h] the key slots
            slots = (kinds[h] if kslots[h] is not None
                     else oracle.layout_slots(kinds[h], wl.F, wl.Hl, wl.Wl, wl.cube))
            ks = slots if kslots[h] is None else kslots[h]
            rows = np.sort(rng.choice(wl.N, size=min(n, wl.N), replace=False))
            t1 = time.perf_counter()
            oracle.attention_rows(q[0, h], k[0, h], v[0, h], slots, wl.block, keeps[h], rows=rows, kslots=ks)
            spent += time.perf_counter() - t1
            allowed = keeps[h][(slots // wl.block)[rows]][:, ks // wl.block].sum()
            flops += 4.0 * wl.d * float(allowed)
            rows_done += len(rows)
        n = min(n * 2, 4096)
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    kinds_how = ("profiled by the oracle" if wl.mode == "profiled" and seconds > 60 else
                 "the planted kinds (even heads spatial, odd temporal: what profiling picks on these inputs)"
                 if wl.mode == "profiled" else "as the workload fixes them")
    desc = (f"attention rows only (the dominant step; profiling, permutation and masks are not in the timed "
            f"work): {rows_done} query rows of {heads} head(s) of {wl.name}, head kinds {kinds_how}, masks built "
            f"for those heads in {mask_s:.1f} s (excluded), attention rows timed for {spent:.1f} s")
    return flops / spent, desc, cores, time.perf_counter() - t_begin


def reference_arm(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per_step = max(1.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    vals = []
    desc = cores = None
    for i in range(args.warmup + args.steps):
        v, desc, cores, _ = oracle_sample(wl, per_step, seed=i)
        if i >= args.warmup:
            vals.append(v)
    tflops = float(np.mean(vals)) / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "sample": "bounded row sample per step"},
            "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="hunyuan")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--qk", default="bf16", choices=["bf16", "fp8"],
                    help="Q.K^T in bf16, or on e4m3 codes with one power-of-two scale per block (P.V stays bf16)")
    ap.add_argument("--layout", default="copies", choices=["copies", "kernel"],
                    help="temporal heads: permuted into copies (faster at these sizes), or gathered inside "
                         "the attention kernel")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    wl = synthetic.WORKLOADS[args.config]
    if args.impl != "reference" and wl.dtype != "bf16":
        raise SystemExit("the benchmark times bf16 workloads; the fp32 tiny case is a parity test")
    if args.impl == "reference":
        reference_arm(args, wl)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    res = gpu_arm(args, wl, rank, world, device)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    peaks, src = load_peaks()
    peak_sust = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    peak_burst = float(peaks["bf16_tflops"])
    attn_s = res["stage_ms"]["attention"] / 1e3
    achieved = res["alg"] / attn_s / 1e12
    # e4m3 Q.K^T: half the flops (Q.K^T) run at twice the bf16 rate (the nominal fp8 / bf16 ratio,
    # 4.5 / 2.25), the other half (P.V) at the bf16 rate, so the attention's peak is the bf16
    # peak / 0.75 (derived, not measured)
    fp8 = args.qk == "fp8"
    qk_factor = 1.0 / 0.75 if fp8 else 1.0
    attn_peak, attn_peak_sust = peak_burst * qk_factor, peak_sust * qk_factor
    attn_peak_src = (f"derived: {src} bf16_tflops (burst) / 0.75, Q.K^T at twice the bf16 rate (nominal "
                     "fp8/bf16 ratio 4.5/2.25), P.V at the bf16 rate" if fp8 else
                     f"{src} bf16_tflops (burst; the kernel runs at the maximum SM clock, see clocks)")
    value = aggregate_tflops(res["alg"], res["ms"], world)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": res["ms"], "ms_per_call": res["ms"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16, Q.K^T e4m3" if fp8 else "bf16", "data": "synthetic",
        "config": {"workload": wl.name + (", Q.K^T e4m3 per-block scales" if fp8 else ""), "B": wl.B, "H": wl.H,
                   "grid": [wl.F, wl.Hl, wl.Wl], "d": wl.d,
                   "block": wl.block, "mode": wl.mode, "w_s": res["w_s"], "w_t": res["w_t"],
                   "kept_block_fraction": res["kept"], "head_kinds": res["kinds"],
                   "layout": ("cluster-major copies (Q by its k-means clusters, K and V by theirs)"
                              if wl.mode == "semantic" else "temporal heads gathered in the attention kernel"
                              if args.layout == "kernel" and wl.mode != "cube" else "permuted copies"),
                   "l2": "inputs larger than L2 (Q,K,V = %.0f MB > 126 MB); no flush" %
                         (3 * wl.B * wl.H * wl.N * wl.d * 2 / 1e6)},
        **({"semantic": {"clusters_q": wl.clusters[0], "clusters_k": wl.clusters[1],
                         "kmeans_iters": wl.kmeans_iters, "top_p": wl.top_p,
                         "stage_slots": "profile = k-means of Q and K, permute = row gathers, mask = top-p "
                                        "budget and block mask, unpermute = scatter of O"}}
           if wl.mode == "semantic" else {}),
        "value_definition": "sparse-actual TFLOP/s of the whole call: algorithmic flops of the kept blocks "
                            "(4*d*valid_q*valid_k per kept pair) / ms per call, summed over ranks",
        "dense_equiv_tflops": aggregate_tflops(res["dense"], res["ms"], world),
        "stage_ms": res["stage_ms"],
        "roofline": {"kernel": "vsa_sparse_attn_fwd_fp8qk" if fp8 else "vsa_sparse_attn_fwd", "bound": "tensor",
                     "achieved": achieved, "peak": attn_peak, "unit": "TFLOP/s", "frac": achieved / attn_peak,
                     "peak_source": attn_peak_src,
                     "frac_of_sustained_peak": achieved / attn_peak_sust,
                     "executed_tflops": res["exe"] / attn_s / 1e12,
                     "executed_frac": res["exe"] / attn_s / 1e12 / attn_peak,
                     "traffic": None if fp8 else TRAFFIC.get(wl.name)},
        "stage_roofline": stage_roofline(res["swork"], res["stage_ms"], float(peaks["hbm_gbs"]), peak_burst),
        "softmax_exp2_per_call": res["exp2"],
        "gpu_launches": res["launches"] * args.steps,
        "clocks": res["clocks"],
        "e2e": {"value": aggregate_tflops(res["alg"], res["e2e"]["ms_per_step"], world), "unit": "TFLOP/s",
                "ms_per_step": res["e2e"]["ms_per_step"], "h2d_bytes_per_step": res["e2e"]["h2d_bytes_per_step"],
                "d2h_bytes_per_step": res["e2e"]["d2h_bytes_per_step"], "api": res["e2e"]["api"]},
    }
    if not args.no_cpu_baseline and world == 1:
        v, desc, cores, _ = oracle_sample(wl, args.cpu_seconds)
        line["cpu_baseline"] = {"value": v / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                "sample": desc}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
