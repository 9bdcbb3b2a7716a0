"""Host-side pieces of bench.py that need no GPU: the clock sampler's parsing and
time-window filter, and the algorithmic work count of a layer (against brute force)."""
import datetime
import sys
import os

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


class _FakeProc:
    def __init__(self, text):
        self.text = text

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return self.text, ""


def _line(t, mhz, power, cap):
    ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    reasons = ["Not Active", "Not Active", "Not Active", "Active" if cap else "Not Active"]
    return ", ".join([ts, "0", f"{mhz}", "1965", f"{power}", "0x0"] + reasons)


def _clocks(lines):
    c = bench.Clocks.__new__(bench.Clocks)
    c.proc = _FakeProc("\n".join(lines) + "\n")
    return c


def test_clock_samples_are_filtered_to_the_timed_window():
    t0 = 1_800_000_000.0
    lines = [_line(t0 - 0.5, 1965, 250, False),      # before the window: ignored
             _line(t0 + 0.01, 1965, 400, False),
             _line(t0 + 0.03, 1650, 900, True),
             _line(t0 + 0.05, 1700, 950, True),
             _line(t0 + 0.50, 1200, 999, True)]      # after the window: ignored
    r = _clocks(lines).stop(t0, t0 + 0.1)
    assert r["samples"] == 3
    assert r["sm_mhz"] == 1700.0 and r["sm_mhz_min"] == 1650.0 and r["sm_max_mhz"] == 1965.0
    assert r["power_w_max"] == 950.0
    assert r["reasons"] == ["sw_power_cap"]


def test_clock_samples_without_window_and_malformed_lines():
    t0 = 1_800_000_000.0
    lines = [_line(t0, 1965, 300, False), "garbage", "", _line(t0 + 1, 1900, 310, False)]
    r = _clocks(lines).stop()
    assert r["samples"] == 2 and r["reasons"] == []


def _brute_work(seqlens, kept_cnt, kept_idx, hq, hkv, d=128, bs=128):
    """Count causal (query, key) pairs on kept blocks and (row, pruned block) terms by
    enumerating rows."""
    G = hq // hkv
    pairs = corr = 0
    t = 0
    for L in seqlens:
        nb = (L + bs - 1) // bs
        for i in range(nb):
            for g in range(hkv):
                kept = set(int(j) for j in kept_idx[t, g, :kept_cnt[t, g]])
                for r in range(i * bs, min(L, (i + 1) * bs)):
                    for j in range(i + 1):
                        if j in kept:
                            pairs += G * len([c for c in range(j * bs, min(L, (j + 1) * bs)) if c <= r])
                        elif j < i:
                            corr += G
            t += 1
    return 4 * d * pairs, 4 * d * corr


def test_layer_work_matches_brute_force():
    rng = np.random.default_rng(3)
    seqlens = [300, 129, 1]
    hq, hkv = 4, 2
    nbs = [(L + 127) // 128 for L in seqlens]
    tot = sum(nbs)
    kept_cnt = np.zeros((tot, hkv), np.int32)
    kept_idx = np.zeros((tot, hkv, max(nbs)), np.int32)
    t = 0
    for nb in nbs:
        for i in range(nb):
            for g in range(hkv):
                js = sorted(set(rng.choice(i + 1, size=rng.integers(0, i + 1), replace=False).tolist()) | {i})
                kept_cnt[t, g] = len(js)
                kept_idx[t, g, :len(js)] = js
            t += 1
    assert bench.layer_work(seqlens, kept_cnt, kept_idx, hq, hkv) == _brute_work(seqlens, kept_cnt, kept_idx, hq, hkv)


def test_dense_flops_equal_layer_work_with_every_block_kept():
    """The comparators' dense work and the layer's kept-pair work agree when
    nothing is pruned (the diagonal block counted causally)."""
    seqlens = [1, 127, 128, 129, 700, 1000]
    hq, hkv = 8, 2
    nbs = [(L + 127) // 128 for L in seqlens]
    nb_max = max(nbs)
    rows = sum(nbs)
    cnt = np.zeros((rows, hkv), np.int32)
    idx = np.full((rows, hkv, nb_max), -1, np.int32)
    t = 0
    for nb in nbs:
        for i in range(nb):
            cnt[t] = i + 1
            idx[t, :, :i + 1] = np.arange(i + 1)
            t += 1
    flops, corr = bench.layer_work(seqlens, cnt, idx, hq, hkv)
    assert corr == 0.0
    assert flops == bench.dense_causal_flops(seqlens, hq)


def test_mufu_bound():
    """16 exp2/clk/SM x 148 SMs x 1965 MHz, 512 flops per exp2 (d = 128)."""
    assert abs(bench.mufu_bound_tflops(148, 1965.0) - 2382.40) < 0.01
