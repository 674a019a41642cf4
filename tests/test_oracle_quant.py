"""Pins for the oracle's cluster parameters, quantizer and dequantizer.

Sources: RPTQ article (基于重排序的新量化方法RPTQ…), worked example between Fig. 1 and Fig. 2 and
the text after Fig. 2 (one s and z per cluster); quantization-basics article, sections 一
(scale = float range / integer range), 1.1 (clamp to the profiled range), 1.3 (zero point,
dequantization s*(q - z)) and 1.4 (per-tensor / per-channel granularity).
"""
import os

import numpy as np
import pytest

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _worked_rows():
    rows = []
    with open(os.path.join(GOLD, "worked_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            b, lo, hi, s, z, half, mse = line.split()
            rows.append((int(b), float(lo), float(hi), float(s), int(z), float(half), float(mse)))
    return rows


WORKED = _worked_rows()


def _two_channel_batch(n=4097, seed=0):
    """Tokens of the two worked-example channels, endpoints included so the calibrated
    ranges are exactly [-100, -50] and [80, 100]."""
    rng = np.random.default_rng(seed)
    a = rng.uniform(-100.0, -50.0, n).astype(np.float32)
    b = rng.uniform(80.0, 100.0, n).astype(np.float32)
    a[:2] = [-100.0, -50.0]
    b[:2] = [80.0, 100.0]
    return np.stack([a, b], axis=1)


@pytest.mark.parametrize("row", WORKED, ids=lambda r: f"b{r[0]}[{r[1]},{r[2]}]")
def test_cluster_params_closed_form(orc, row):
    bits, lo, hi, s_ref, z_ref, _, _ = row
    s, z = orc.cluster_params([hi], [lo], [0], 1, bits)
    assert s[0] == np.float32(s_ref)
    assert z[0] == z_ref


@pytest.mark.parametrize("bits", [3, 4])
def test_worked_example_per_cluster_beats_per_tensor(orc, bits):
    """Per-cluster quantization of the two channels is far more accurate than one shared range
    ("far below": at least 10x lower MSE on BOTH channels; the closed forms give 16x / 100x)."""
    x = _two_channel_batch()
    mx, mn = orc.minmax(x)
    assert list(mx) == [-50.0, 100.0] and list(mn) == [-100.0, 80.0]
    errs = {}
    for g in (1, 2):
        cal = orc.calibrate(mx, mn, g, 10, bits)
        ref = [r for r in WORKED if r[0] == bits]
        if g == 1:
            assert cal["scale"][0] == np.float32(ref[0][3]) and cal["zero"][0] == ref[0][4]
        else:
            # cluster 0 is the lower (max, min) point, i.e. the [-100, -50] channel
            assert list(cal["R"]) == [0, 1]
            assert cal["scale"][0] == np.float32(ref[1][3]) and cal["zero"][0] == ref[1][4]
            assert cal["scale"][1] == np.float32(ref[2][3]) and cal["zero"][1] == ref[2][4]
        # quantize in stored order, dequantize, compare with the inputs gathered the same way
        xs = x[:, cal["R"]]
        q = orc.quantize(xs, cal["col_cluster"], cal["scale"], cal["zero"], bits)
        deq = orc.dequant(q, cal["col_cluster"], cal["scale"], cal["zero"])
        err = (deq.astype(np.float64) - xs.astype(np.float64))
        errs[g] = (np.mean(err ** 2, axis=0), np.max(np.abs(err), axis=0))
        for j, k in enumerate(cal["col_cluster"]):
            assert errs[g][1][j] <= cal["scale"][k] / 2 * (1 + 1e-6) + 2.0 ** -22 * 100
    mse_tensor, mse_cluster = errs[1][0], errs[2][0]
    assert np.all(mse_cluster * 10 <= mse_tensor), (mse_cluster, mse_tensor)
    # and the measured MSEs sit near the uniform-distribution closed form s^2/12
    ref = [r for r in WORKED if r[0] == bits]
    assert mse_tensor[0] == pytest.approx(ref[0][6], rel=0.15)
    assert mse_cluster[0] == pytest.approx(ref[1][6], rel=0.15)
    assert mse_cluster[1] == pytest.approx(ref[2][6], rel=0.15)


@pytest.mark.parametrize("bits", [3, 4])
def test_half_step_bound_inside_range_and_clamp_outside(orc, bits):
    rng = np.random.default_rng(1)
    qmax = 2 ** bits - 1
    g = 16
    lo = rng.normal(0, 5, g).astype(np.float32)
    hi = (lo + rng.lognormal(0, 1, g)).astype(np.float32)
    hi[3] = lo[3] + 1e-3  # a very narrow cluster (large |z|)
    lo[5], hi[5] = np.float32(2.0), np.float32(2.0)  # degenerate cluster
    s, z = orc.cluster_params(hi, lo, np.arange(g), g, bits)
    # closed forms of the degenerate reading: s = |m| / qmax, z = -qmax for a positive constant
    assert s[5] == np.float32(2.0) / np.float32(qmax) and z[5] == -qmax
    n = 2000
    u = rng.random((n, g)).astype(np.float32)
    y = (lo + (hi - lo) * u).astype(np.float32)
    y[0], y[1] = lo, hi
    cc = np.arange(g, dtype=np.int32)
    q = orc.quantize(y, cc, s, z, bits)
    assert q.max() <= qmax
    deq = orc.dequant(q, cc, s, z).astype(np.float64)
    err = np.abs(deq - y.astype(np.float64))
    # exact arithmetic gives err <= s/2; in fp32 the divide y/s and the product s*(q - z) each
    # round once, which can add half an ulp of |y| and of |deq| (visible when |z| is large)
    slack = 2.0 ** -23 * (np.abs(y) + np.abs(deq))
    assert np.all(err <= s.astype(np.float64) / 2 * (1 + 1e-6) + slack)
    # out of range: clamp to the ends of the code range (static quantization)
    # (beyond the whole code grid s*(q - z), q in [0, qmax], which for the degenerate cluster
    # spans [m, m + qmax*s] rather than [m, M])
    below = (lo - (qmax + 1) * s - 1).astype(np.float32)[None, :]
    above = (hi + (qmax + 1) * s + 1).astype(np.float32)[None, :]
    assert np.all(orc.quantize(below, cc, s, z, bits) == 0)
    assert np.all(orc.quantize(above, cc, s, z, bits) == qmax)


def test_round_half_to_even_and_integer_zero_point(orc):
    # s = 1: y/s is exact, so the code is rint(y) + z, ties to even, z added after rounding
    s = np.array([1.0], np.float32)
    z = np.array([3], np.int32)
    y = np.array([[-3.5, -2.5, -0.5, 0.5, 1.5, 2.5, 11.5]], np.float32)
    q = orc.quantize(y, [0] * 7, s, z, 4)
    assert list(q[0]) == [0, 1, 3, 3, 5, 5, 15]


def test_granularity_g1_is_per_tensor_and_gC_is_per_channel(orc):
    rng = np.random.default_rng(2)
    C, T, bits = 24, 300, 4
    center = rng.normal(0, 2, C)
    hw = rng.lognormal(0, 1, C)
    x = (center + hw * (2 * rng.random((T, C)) - 1)).astype(np.float32)
    mx, mn = orc.minmax(x)
    # g = 1: every channel shares the whole-tensor range
    one = orc.calibrate(mx, mn, 1, 5, bits)
    s_t, z_t = orc.cluster_params([x.max()], [x.min()], [0], 1, bits)
    assert one["scale"][0] == s_t[0] and one["zero"][0] == z_t[0]
    assert list(one["R"]) == list(range(C))
    # g = C: each channel is its own cluster with its own range
    allc = orc.calibrate(mx, mn, C, 5, bits)
    assert sorted(allc["labels"]) == list(range(C))
    for j in range(C):
        c = allc["R"][j]
        k = allc["col_cluster"][j]
        s_c, z_c = orc.cluster_params([mx[c]], [mn[c]], [0], 1, bits)
        assert allc["scale"][k] == s_c[0] and allc["zero"][k] == z_c[0]


def test_dequant_closed_form(orc):
    s = np.array([0.5, 2.0], np.float32)
    z = np.array([3, -60], np.int32)
    q = np.array([[0, 0], [7, 15]], np.uint8)
    out = orc.dequant(q, [0, 1], s, z)
    assert out.tolist() == [[-1.5, 120.0], [2.0, 150.0]]
