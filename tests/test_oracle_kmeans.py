"""Pins for the oracle's KMeans, reorder index and calibration chain (RPTQ article, text after
Fig. 2: KMeans into g clusters on the per-channel (max, min) points, then same-cluster channels
placed next to each other)."""
import itertools

import numpy as np
import pytest

from post_activation_quantization_b200 import synthetic


def _sse(P, labels, cent):
    return float(sum(((P[c] - cent[labels[c]]) ** 2).sum() for c in range(len(P))))


def _partitions(n, g):
    """All labelings of n items into exactly g non-empty groups (canonical: first use order)."""
    def rec(i, labels, used):
        if i == n:
            if used == g:
                yield list(labels)
            return
        for k in range(min(used + 1, g)):
            labels.append(k)
            yield from rec(i + 1, labels, max(used, k + 1))
            labels.pop()
    yield from rec(0, [], 0)


def test_assign_ties_go_to_lowest_index(orc):
    cent = np.array([[0.0, 0.0], [2.0, 0.0], [1.0, 1.0]])
    lab, _ = orc.kmeans_assign([1.0, 1.0], [0.0, 1.0], cent)
    # (1,0) is at distance 1 from clusters 0, 1 and 2 -> 0; (1,1) sits on centroid 2
    assert list(lab) == [0, 2]


def test_quantile_init_positions(orc):
    rng = np.random.default_rng(0)
    C, g = 37, 5
    mx = rng.normal(0, 1, C).astype(np.float32)
    mn = (mx - rng.random(C)).astype(np.float32)
    order = sorted(range(C), key=lambda c: (mx[c], mn[c], c))
    cent = orc.kmeans_init(mx, mn, g)
    for k in range(g):
        c = order[((2 * k + 1) * C) // (2 * g)]
        assert tuple(cent[k]) == (float(mx[c]), float(mn[c]))
    # equal max values are ordered by min, then by index
    mx2 = np.array([1, 1, 1, 0], np.float32)
    mn2 = np.array([0.5, 0.2, 0.5, 0], np.float32)
    cent2 = orc.kmeans_init(mx2, mn2, 4)
    f = lambda v: float(np.float32(v))
    assert cent2.tolist() == [[0, 0], [1, f(0.2)], [1, 0.5], [1, 0.5]]


@pytest.mark.parametrize("seed", range(6))
def test_lloyd_tiny_fixed_point_and_brute_force(orc, seed):
    rng = np.random.default_rng(seed)
    n = 8
    g = 2 + seed % 2
    mx = rng.normal(0, 3, n).astype(np.float32)
    mn = (mx - rng.lognormal(0, 1, n)).astype(np.float32)
    P = np.stack([mx, mn], 1).astype(np.float64)
    labels, cent = orc.kmeans(mx, mn, g, 100)
    # centroids are the member means (non-empty clusters), labels are nearest-centroid
    for k in range(g):
        mem = P[labels == k]
        if len(mem):
            assert np.allclose(cent[k], mem.mean(0), rtol=1e-14, atol=1e-14)
    d = ((P[:, None, :] - cent[None]) ** 2).sum(-1)
    assert np.all(d[np.arange(n), labels] <= d.min(1))
    # fixed point of (update, assign)
    cent2 = orc.kmeans_update(mx, mn, labels, cent)
    lab2, changed = orc.kmeans_assign(mx, mn, cent2, labels)
    assert changed == 0 and np.array_equal(lab2, labels)
    # Lloyd is a local method: its SSE is never below the exhaustive optimum
    best = min(_sse(P, lab, np.array([P[np.array(lab) == k].mean(0) for k in range(g)]))
               for lab in _partitions(n, g))
    assert _sse(P, labels, cent) >= best - 1e-9


def test_g1_centroid_is_mean_and_gC_is_identity(orc):
    rng = np.random.default_rng(3)
    C = 50
    mx = rng.normal(0, 3, C).astype(np.float32)
    mn = (mx - rng.lognormal(0, 1, C)).astype(np.float32)
    lab, cent = orc.kmeans(mx, mn, 1, 3)
    assert np.all(lab == 0)
    import math
    assert cent[0, 0] == pytest.approx(math.fsum(mx.astype(float)) / C, rel=1e-14)
    assert cent[0, 1] == pytest.approx(math.fsum(mn.astype(float)) / C, rel=1e-14)
    lab, cent = orc.kmeans(mx, mn, C, 0)
    rank = sorted(range(C), key=lambda c: (mx[c], mn[c], c))
    assert [rank.index(c) for c in range(C)] == list(lab)


def test_two_blobs_recovered(orc):
    rng = np.random.default_rng(4)
    C = 400
    blob = rng.random(C) < 0.3
    mx = np.where(blob, 100 + rng.normal(0, 1, C), rng.normal(0, 1, C)).astype(np.float32)
    mn = np.where(blob, 80 + rng.normal(0, 1, C), -rng.lognormal(0, 0.3, C)).astype(np.float32)
    lab, _ = orc.kmeans(mx, mn, 2, 10)
    assert np.array_equal(lab == 1, blob)  # the blob has the larger max -> cluster 1


@pytest.mark.parametrize("C,g,iters,seed", [(768, 8, 10, 0), (4096, 32, 20, 1), (2000, 16, 30, 2)])
def test_matches_sklearn_lloyd_from_same_init(orc, C, g, iters, seed):
    """sklearn's Lloyd (a library routine), started from the same centroids, reaches the same
    labels; centroids agree to rounding."""
    from sklearn.cluster import KMeans
    m = synthetic.channel_model(C, seed)
    x = synthetic.activations(512, m, seed, dtype="f32")
    gamma, beta = synthetic.ln_params(C, seed)
    mx, mn = orc.minmax_ln(x.numpy(), gamma, beta)
    labels, cent = orc.kmeans(mx, mn, g, iters)
    assert np.bincount(labels, minlength=g).min() > 0  # sklearn relocates empty clusters
    P = np.stack([mx, mn], 1).astype(np.float64)
    km = KMeans(n_clusters=g, init=orc.kmeans_init(mx, mn, g), n_init=1, max_iter=iters, tol=0.0,
                algorithm="lloyd").fit(P)
    assert np.array_equal(km.labels_, labels)
    assert np.allclose(km.cluster_centers_, cent, rtol=1e-9, atol=1e-9)


def test_reorder_invariants_and_stable_argsort(orc):
    rng = np.random.default_rng(5)
    C, g = 1000, 13
    labels = rng.integers(0, g, C).astype(np.int32)
    labels[labels == 4] = 5  # an empty cluster
    R, cc, off = orc.reorder(labels, g)
    assert sorted(R) == list(range(C))
    assert np.array_equal(R, np.argsort(labels, kind="stable"))
    assert np.array_equal(cc, labels[R]) and np.all(np.diff(cc) >= 0)
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(labels, minlength=g))]))
    for k in range(g):
        seg = R[off[k]:off[k + 1]]
        assert np.all(np.diff(seg) > 0) and np.all(labels[seg] == k)
