"""Helpers shared by the GPU parity tests: tolerance checks and oracle-side references."""
import math

import numpy as np
import torch

import oracle

# Attention output tolerance (bf16 inputs, fp32 accumulation): max-abs and relative L2.
ATOL_MAX = 2e-2
REL_L2 = 1e-2


def assert_close_attention(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    err = np.abs(got - want)
    mx = float(err.max()) if err.size else 0.0
    rel = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))
    assert mx <= ATOL_MAX, f"{what}: max-abs {mx:.3e} > {ATOL_MAX}"
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e} > {REL_L2}"
    return mx, rel


def head_slots(kind, wl):
    return oracle.layout_slots(kind, wl.F, wl.Hl, wl.Wl, wl.cube)


def keep_for_head(kind, wl, w_s, w_t, q=None, k=None):
    if kind == oracle.CUBE:
        return oracle.cube_topk_keep(q, k, wl.F, wl.Hl, wl.Wl, wl.topk, wl.cube)
    w = w_s if kind == oracle.SPATIAL else w_t
    return oracle.pattern_keep(kind, wl.F, wl.Hl, wl.Wl, wl.block, w)


def oracle_rows(q, k, v, kind, wl, keep, rows):
    """Oracle attention (natural order) for the given rows of one head."""
    slots = head_slots(kind, wl)
    return oracle.attention_rows(q, k, v, slots, wl.block, keep, rows=rows, scale=1.0 / math.sqrt(wl.d))


def to_f64(t):
    return t.detach().to("cpu").double().numpy()


def cuda_err():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


# Profiling MSE tolerance.  The kernel forms each variant's output with P rounded to bf16
# (relative error up to 2^-9 per probability) and fp32 accumulation, so an output element can
# be off by about 2^-9 times the size of the outputs, and the difference of two variants by
# twice that.  With eps = 2^-7 * max |O_dense| over the sampled outputs (a factor 2 of margin),
# an MSE m computed from differences off by at most eps is within 2 sqrt(m) eps + eps^2 of the
# exact one.
MSE_EPS_REL = 2.0 ** -7
MSE_LOG = []


def mse_close(got: float, want: float, dense_rows, what=""):
    eps = MSE_EPS_REL * float(np.abs(dense_rows).max())
    bound = 2.0 * math.sqrt(max(want, 0.0)) * eps + eps * eps
    MSE_LOG.append((what, got, want, abs(got - want) / max(bound, 1e-300)))
    assert abs(got - want) <= bound, f"{what}: MSE {got!r} vs oracle {want!r}, bound {bound:.3e}"
