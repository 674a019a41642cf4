"""Property checks of the oracle on random small inputs (hypothesis): packing round trips and
its byte layout, the invariants of the offline chain (R a permutation, stable counting sort,
cluster ranges), the final labels being a nearest-centroid assignment of the final centroids,
and the quantizer's error bound inside a cluster's range with clamping outside it."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle

SETTINGS = settings(max_examples=40, deadline=None)


@SETTINGS
@given(rows=st.integers(1, 4), groups=st.integers(1, 12), bits=st.sampled_from([3, 4]), seed=st.integers(0, 2**31))
def test_pack_round_trip_and_layout(rows, groups, bits, seed):
    rng = np.random.default_rng(seed)
    C = 8 * groups
    q = rng.integers(0, 2**bits, (rows, C)).astype(np.uint8)
    p = oracle.pack(q, bits)
    assert p.shape == (rows, C * bits // 8)
    assert np.array_equal(oracle.unpack(p, C, bits), q)
    # the layout by hand: code k of each group of 8 at bits [b*k, b*k + b) of a little-endian word
    words = np.zeros((rows, groups), np.uint64)
    for k in range(8):
        words |= q[:, k::8].astype(np.uint64) << np.uint64(bits * k)
    by_hand = np.stack([(words >> np.uint64(8 * i)) & np.uint64(255) for i in range(bits)], axis=2)
    assert np.array_equal(p.reshape(rows, groups, bits), by_hand.astype(np.uint8))


def _stats(rng, C):
    mx = rng.normal(0, 2, C).astype(np.float32)
    mn = (mx - rng.lognormal(0, 1, C)).astype(np.float32)
    return mx, mn


@SETTINGS
@given(C=st.integers(1, 160), gfrac=st.floats(0.0, 1.0), iters=st.integers(0, 8), bits=st.sampled_from([3, 4]),
       seed=st.integers(0, 2**31))
def test_offline_chain_invariants(C, gfrac, iters, bits, seed):
    rng = np.random.default_rng(seed)
    mx, mn = _stats(rng, C)
    g = 1 + int(gfrac * (C - 1))
    cal = oracle.calibrate(mx, mn, g, iters, bits)
    lab, R, cc, off = cal["labels"], cal["R"], cal["col_cluster"], cal["offsets"]
    assert np.array_equal(np.sort(R), np.arange(C))                 # a permutation
    assert np.array_equal(cc, lab[R])                                # stored column -> its cluster
    assert np.all(np.diff(cc) >= 0)                                  # clusters in label order
    for k in range(g):
        members = R[off[k]:off[k + 1]]
        assert np.all(lab[members] == k) and np.all(np.diff(members) > 0)  # stable: ascending channels
    assert off[0] == 0 and off[g] == C
    # the final labels are a nearest-centroid assignment of the final centroids (fp64, dx*dx + dy*dy,
    # ties to the lowest index)
    P = np.stack([mx, mn], 1).astype(np.float64)
    cent = cal["centroids"]
    dx = P[:, None, 0] - cent[None, :, 0]
    dy = P[:, None, 1] - cent[None, :, 1]
    d = dx * dx + dy * dy
    assert np.array_equal(lab, np.argmin(d, axis=1).astype(np.int32))
    # every cluster's scale is positive and finite; a non-empty cluster's range is covered
    s, z = cal["scale"], cal["zero"]
    qmax = 2**bits - 1
    assert np.all(np.isfinite(s)) and np.all(s > 0)
    for k in range(g):
        m = lab == k
        if not m.any():
            continue
        lo, hi = mn[m].min(), mx[m].max()
        # the range's ends land on codes inside [0, qmax] up to one rounding step
        assert -1 <= np.rint(lo / s[k]) + z[k] <= 1 and qmax - 1 <= np.rint(hi / s[k]) + z[k] <= qmax + 1 \
            or lo == hi


@SETTINGS
@given(C=st.integers(8, 96).map(lambda c: c - c % 8), rows=st.integers(1, 6), bits=st.sampled_from([3, 4]),
       seed=st.integers(0, 2**31))
def test_quantizer_error_bound_and_clamping(C, rows, bits, seed):
    rng = np.random.default_rng(seed)
    mx, mn = _stats(rng, C)
    cal = oracle.calibrate(mx, mn, max(1, C // 8), 5, bits)
    R, cc, s, z = cal["R"], cal["col_cluster"], cal["scale"], cal["zero"]
    qmax = 2**bits - 1
    # values inside each stored column's cluster range [m_k, M_k]
    lab = cal["labels"]
    g = s.size
    lo = np.array([mn[lab == k].min() if (lab == k).any() else 0 for k in range(g)], np.float32)
    hi = np.array([mx[lab == k].max() if (lab == k).any() else 0 for k in range(g)], np.float32)
    u = rng.random((rows, C)).astype(np.float32)
    y = (lo[cc] + u * (hi[cc] - lo[cc])).astype(np.float32)
    q = oracle.quantize(y, cc, s, z, bits)
    assert q.max() <= qmax
    back = oracle.dequant(q, cc, s, z).astype(np.float64)
    err = np.abs(back - y.astype(np.float64))
    bound = s[cc].astype(np.float64) / 2 * (1 + 1e-5) + 2**-22 * np.abs(y).astype(np.float64) + 1e-30
    assert np.all(err <= bound)
    # far outside the range: clamped to the end codes
    far_hi = (hi[cc] + 10 * s[cc] + 1).astype(np.float32)[None, :]
    far_lo = (lo[cc] - 10 * s[cc] - 1).astype(np.float32)[None, :]
    assert np.all(oracle.quantize(far_hi, cc, s, z, bits) == qmax)
    assert np.all(oracle.quantize(far_lo, cc, s, z, bits) == 0)
