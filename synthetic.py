"""Seeded synthetic workloads for the spatial-temporal block-sparse attention path.

This module is shared by the tests, the benchmark and the CPU oracle's callers.  It
holds workload shapes and seeded random draws only: no permutation, mask, softmax or
profiling arithmetic lives here, so neither side of a parity check can borrow the
other's logic through it.

Workload recipe (stand-ins for the latent grids of the video models the pages name;
no model, weights or videos are used):

* a latent grid of F frames x Hl x Wl tokens, token t = (f*Hl + h)*Wl + w, tensors laid
  out [B, H, N, d] with d fastest;
* draws from ``torch.Generator('cpu').manual_seed(seed)`` in this order:
  z_Q, z_K, V of shape [B, H, N, d], then u_frame [H, F, d], u_pos [H, Hl*Wl, d],
  all standard normal;
* even heads carry a shared per-frame vector (u = u_frame[h, f(t)]), odd heads a
  shared per-position vector (u = u_pos[h, s(t)]), so half of the heads favour
  intra-frame attention and half same-position attention across frames;
* Q = z_Q + 2*u, K = z_K + 2*u, V = noise; cast to bf16 with round-to-nearest-even
  except for the fp32 tiny case, whose Q/K/V are plain N(0,1) (no planted vector) with
  fixed head kinds.

The planted structure mirrors the two head families of the Sparse VideoGen summary page
("Approach": spatial heads attend within a frame, temporal heads to the same position
across frames).
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import torch

SPATIAL, TEMPORAL, CUBE = 0, 1, 2


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention call's shape and selection parameters."""

    name: str
    B: int
    H: int
    F: int
    Hl: int
    Wl: int
    d: int
    block: int
    dtype: str                       # "f32" or "bf16"
    mode: str                        # "fixed", "profiled", "cube" or "semantic"
    target: Optional[float] = None   # kept-block fraction the windows must reach
    w_s: Optional[int] = None        # fixed windows (mode "fixed")
    w_t: Optional[int] = None
    fixed_kinds: Optional[Sequence[int]] = None
    cube: tuple = (4, 4, 8)
    topk: int = 0
    profile_frac: float = 0.01
    structure_scale: float = 2.0
    seed: int = 0
    clusters: tuple = (128, 128)     # k-means clusters of Q and of K (mode "semantic")
    kmeans_iters: int = 4
    top_p: float = 0.6

    @property
    def S(self) -> int:
        return self.Hl * self.Wl

    @property
    def N(self) -> int:
        return self.F * self.Hl * self.Wl

    @property
    def nblk(self) -> int:
        return -(-self.N // self.block)

    @property
    def ncubes(self) -> int:
        cf, ch, cw = self.cube
        return (-(-self.F // cf)) * (-(-self.Hl // ch)) * (-(-self.Wl // cw))

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


TINY = Workload("tiny: B1 H2 4x8x8 d64 block64 fp32", 1, 2, 4, 8, 8, 64, 64, "f32", "fixed",
                w_s=0, w_t=0, fixed_kinds=(SPATIAL, TEMPORAL), structure_scale=0.0)  # plain N(0,1)
WAN = Workload("wan2.1-1.3b: B1 H12 21x30x52 d128 block128 bf16", 1, 12, 21, 30, 52, 128, 128,
               "bf16", "profiled", target=0.18)
HUNYUAN = Workload("hunyuanvideo-720p: B1 H24 33x45x80 d128 block128 bf16", 1, 24, 33, 45, 80, 128, 128,
                   "bf16", "profiled", target=0.18)
WAN_6X = Workload("wan2.1-1.3b 6x horizon: B1 H12 126x30x52 d128 cubes 4x4x8 top-32", 1, 12, 126, 30, 52,
                  128, 128, "bf16", "cube", topk=32)
WAN_SEMANTIC = Workload("wan2.1-1.3b semantic: B1 H12 21x30x52 d128 block128 bf16, k-means 128/128 x4, top-p 0.6",
                        1, 12, 21, 30, 52, 128, 128, "bf16", "semantic")
SWEEP_TARGETS = (1.0, 0.35, 0.18, 0.13, 0.05)


def sweep(target: float) -> Workload:
    return WAN.with_(name=f"sparsity sweep kept={target}: B1 H12 21x30x52 d128 block128 bf16", target=target)


WORKLOADS = {"tiny": TINY, "wan": WAN, "hunyuan": HUNYUAN, "wan6x": WAN_6X, "wan-semantic": WAN_SEMANTIC}
for _t in SWEEP_TARGETS:
    WORKLOADS[f"sweep{_t}"] = sweep(_t)


def make_qkv(wl: Workload, seed: Optional[int] = None, heads: Optional[Sequence[int]] = None):
    """Return (q, k, v) CPU tensors [B, H, N, d] in the workload's dtype.

    ``heads`` optionally restricts the returned tensors to a subset of heads; the draws
    are still made for all heads so that values do not depend on the subset.
    """
    seed = wl.seed if seed is None else seed
    g = torch.Generator("cpu").manual_seed(seed)
    B, H, N, d, F, S = wl.B, wl.H, wl.N, wl.d, wl.F, wl.S
    zq = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    zk = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    v = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    u_frame = torch.randn(H, F, d, generator=g, dtype=torch.float32)
    u_pos = torch.randn(H, S, d, generator=g, dtype=torch.float32)
    t = torch.arange(N)
    f_of_t = t // S
    s_of_t = t % S
    c = wl.structure_scale
    for h in range(H):
        u = u_frame[h, f_of_t] if h % 2 == 0 else u_pos[h, s_of_t]
        zq[:, h] += c * u
        zk[:, h] += c * u
    if heads is not None:
        idx = torch.as_tensor(list(heads), dtype=torch.long)
        zq, zk, v = zq[:, idx], zk[:, idx], v[:, idx]
    if wl.dtype == "bf16":
        return (zq.to(torch.bfloat16).contiguous(), zk.to(torch.bfloat16).contiguous(),
                v.to(torch.bfloat16).contiguous())
    return zq.contiguous(), zk.contiguous(), v.contiguous()


def make_random(shape, dtype=torch.bfloat16, seed: int = 0, scale: float = 1.0):
    """Plain seeded N(0, scale^2) tensor for edge-case tests."""
    g = torch.Generator("cpu").manual_seed(seed)
    return (torch.randn(*shape, generator=g, dtype=torch.float32) * scale).to(dtype)


def sample_indices(n: int, count: int, seed: int) -> torch.Tensor:
    """Seeded sorted sample of ``count`` distinct indices in [0, n)."""
    g = torch.Generator("cpu").manual_seed(seed)
    count = min(count, n)
    return torch.randperm(n, generator=g)[:count].sort().values


def dense_flops(wl: Workload) -> float:
    """4*N^2*d per head: the flop count of dense attention on the real tokens."""
    return 4.0 * wl.B * wl.H * float(wl.N) ** 2 * wl.d


def human(wl: Workload) -> str:
    return f"{wl.name} (N={wl.N})"


__all__ = ["Workload", "WORKLOADS", "TINY", "WAN", "HUNYUAN", "WAN_6X", "WAN_SEMANTIC", "SWEEP_TARGETS", "sweep",
           "make_qkv", "make_random", "sample_indices", "dense_flops", "SPATIAL", "TEMPORAL", "CUBE"]
