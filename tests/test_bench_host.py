"""Host logic of bench.py that needs no GPU: the clock sampler's window filter."""
import pytest

import bench


def _line(sm, reasons=("Not Active",) * 4):
    return ", ".join(["0", str(sm), "1965", "700.5", "0x0", *reasons])


def _sampler(samples, t0, t1):
    c = bench.ClockSampler("0")
    c.samples = samples
    c.t0, c.t1 = t0, t1
    return c


def test_clock_summary_keeps_only_the_timed_window():
    s = [(0.9, _line(900)), (1.05, _line(1900)), (1.10, _line(1800)), (1.15, _line(1700)), (1.3, _line(100))]
    out = _sampler(s, 1.0, 1.2).summary()
    assert out["samples"] == 3 and out["sm_mhz"] == 1800 and out["window"] == "inside"
    assert out["sm_max_mhz"] == 1965 and out["reasons"] == []


def test_clock_summary_short_window_takes_the_neighbours():
    s = [(0.9, _line(1950)), (1.5, _line(1930)), (2.0, _line(100))]
    out = _sampler(s, 1.0, 1.01).summary()
    assert out["window"] == "nearest" and out["samples"] == 2 and out["sm_mhz"] == 1940


def test_clock_summary_reports_throttle_reasons():
    active = ("Not Active", "Not Active", "Not Active", "Active")
    s = [(1.05, _line(1800, active)), (1.1, _line(1850))]
    out = _sampler(s, 1.0, 1.2).summary()
    assert out["reasons"] == ["sw_power_cap"]


def test_clock_summary_without_samples():
    out = _sampler([], 1.0, 2.0).summary()
    assert out["samples"] == 0 and out["sm_mhz"] is None and out["reasons"] == ["unavailable"]


# ---------------------------------------------------------------------------------------
# work accounting: the figures the bench divides by time
# ---------------------------------------------------------------------------------------

import types  # noqa: E402

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import synthetic  # noqa: E402


def test_attention_work_is_the_allowed_token_pairs():
    """Algorithmic flops = 4·d per allowed (query, key) token pair, counted here from the
    oracle's block mask at token level (ragged last block, spatial and temporal heads)."""
    wl = synthetic.WAN.with_(H=2, F=3, Hl=5, Wl=20)          # N = 300: blocks of 128, 128, 44
    nb = 3
    keeps = [np.array([[1, 0, 1], [1, 1, 0], [0, 1, 1]], bool), np.ones((nb, nb), bool)]
    kinds = [oracle.SPATIAL, oracle.TEMPORAL]
    idx = np.full((1, 2, nb, nb), -1, np.int32)
    cnt = np.zeros((1, 2, nb), np.int32)
    for h in range(2):
        i_, c_ = oracle.keep_to_lists(keeps[h], nb)
        idx[0, h], cnt[0, h] = i_, c_
    alg, exe, pairs = bench.attention_work(wl, np.array(kinds), idx, cnt)
    want = 0
    for h, kind in enumerate(kinds):
        blk = oracle.layout_slots(kind, wl.F, wl.Hl, wl.Wl) // wl.block
        want += int(keeps[h][blk[:, None], blk[None, :]].sum())
    assert alg == 4.0 * wl.d * want
    assert pairs == int(sum(k.sum() for k in keeps))
    assert exe == 4.0 * wl.d * 128 * 128 * pairs


def test_semantic_stage_work():
    """k-means: 2·d flop per (row, centroid) pair per round for Q and K; gathers read and
    write Q, K, V; the scatter reads and writes O."""
    wl = synthetic.WAN_SEMANTIC
    pipe = types.SimpleNamespace(nblk=256, max_kv=256)
    work, exp2 = bench.stage_work(wl, [1] * wl.H, pipe, pairs=1000)
    row = wl.d * 2
    assert work["profile"]["flops"] == wl.H * wl.kmeans_iters * 2 * wl.d * wl.N * sum(wl.clusters)
    assert work["permute"]["bytes"] == wl.H * 3 * 2 * wl.N * row
    assert work["unpermute"]["bytes"] == wl.H * 2 * wl.N * row
    assert work["mask"]["bytes"] == wl.H * 256 * (8 + 256 + 1) * 4
    assert exp2 == 1000 * 128 * 128
    roof = bench.stage_roofline(work, {"profile": 4.0, "permute": 0.1, "mask": 0.2, "unpermute": 0.05}, 6538.3,
                                1631.1)
    # the k-means distances run on the tensor cores: algorithmic and executed (two bf16 halves)
    # rates against the bf16 peak
    assert roof["profile"]["bound"] == "tensor" and roof["profile"]["peak"] == 1631.1
    assert abs(roof["profile"]["frac"] - work["profile"]["flops"] / 4e-3 / 1e12 / 1631.1) < 1e-12
    assert work["profile"]["executed_flops"] == 2 * work["profile"]["flops"]
    assert abs(roof["permute"]["achieved"] - work["permute"]["bytes"] / 1e-4 / 1e9) < 1e-6


@pytest.mark.parametrize("F,Hl,Wl,block,w_s,w_t,r", [(6, 8, 16, 128, 1, 40, 37), (7, 5, 9, 64, 2, 7, 10),
                                                     (21, 30, 52, 128, 2, 140, 328)])
def test_profile_allowed_keys_matches_masks(F, Hl, Wl, block, w_s, w_t, r):
    """The profiling stage's algorithmic work counts, per sampled row, the keys each pattern's
    block mask allows (counted here from the oracle's masks and layouts)."""
    wl = synthetic.Workload("p", 1, 1, F, Hl, Wl, 64, block, "bf16", "profiled")
    N = wl.N
    rows = [((2 * i + 1) * N) // (2 * r) for i in range(r)]
    want = 0
    for kind, w in ((oracle.SPATIAL, w_s), (oracle.TEMPORAL, w_t)):
        keep = oracle.pattern_keep(kind, F, Hl, Wl, block, w)
        blk = oracle.layout_slots(kind, F, Hl, Wl) // block
        want += int(keep[blk[rows]][:, blk].sum())
    assert bench.profile_allowed_keys(wl, r, w_s, w_t) == want
